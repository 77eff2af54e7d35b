// Device helpers shared by the kernels of the W4 g32 MoE layer (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "layout.h"

namespace lingmoe {

// ---------------------------------------------------------------- loads
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ldg_stream64(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ unsigned short ldg_stream16(const void* p) {
  unsigned short v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
// Data written earlier in the same launch by other CTAs: read from L2.
__device__ __forceinline__ float ldcg_f32(const float* p) { return __ldcg(p); }
__device__ __forceinline__ float4 ldcg_f4(const float4* p) { return __ldcg(p); }

// Bulk prefetch of a contiguous byte range into L2 (size multiple of 16,
// address 16-byte aligned).  Fire and forget.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(unsigned short v) {
  return __uint_as_float(((uint32_t)v) << 16);
}

// int4 -> fp32 without a conversion instruction: with the code stored as an
// offset-binary nibble n = q + 8 in 0..15, the bit pattern 0x3F000000 | n<<16
// is the float 0.5 + n/256 exactly.  One byte permute per element places the
// nibble (already masked to the low half of its byte) into bits 16..19 under
// the exponent byte 0x3F.  So for a group of 32 codes and inputs x:
//   sum_k q_k x_k = 256 * (sum_k f_k x_k - (136/256) * sum_k x_k)
// which the kernels evaluate as an fp32 FMA chain started at
// c_G = -0.53125 * sum_k x_k, multiplied by 256 once per row at the end.
// Each product f_k * x_k is exact in fp32 (f has 8 significant bits, x a
// bf16-or-fp32 activation), so only the running sums round.
__device__ __forceinline__ void dequant8(uint32_t w, float f[8]) {
  const uint32_t lo = w & 0x0F0F0F0Fu;
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t m = 0x3F000000u;
  f[0] = __uint_as_float(__byte_perm(lo, m, 0x7054));
  f[1] = __uint_as_float(__byte_perm(hi, m, 0x7054));
  f[2] = __uint_as_float(__byte_perm(lo, m, 0x7154));
  f[3] = __uint_as_float(__byte_perm(hi, m, 0x7154));
  f[4] = __uint_as_float(__byte_perm(lo, m, 0x7254));
  f[5] = __uint_as_float(__byte_perm(hi, m, 0x7254));
  f[6] = __uint_as_float(__byte_perm(lo, m, 0x7354));
  f[7] = __uint_as_float(__byte_perm(hi, m, 0x7354));
}
constexpr float kBiasCoef = -0.53125f;  // -(136/256)
constexpr float kCodeScale = 256.0f;

__device__ __forceinline__ float silu_mul(float g, float u) {
  // SiLU(g) * u = g / (1 + e^-g) * u
  return g / (1.0f + expf(-g)) * u;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- grid barrier
// Counters only ever increase: a launch reads the counter once at its start
// (before it has arrived itself), so gen = value / nctas is this launch's
// generation and the barrier opens at (gen + 1) * nctas.  Every wait is
// bounded by a time limit read from %globaltimer; when it runs out the CTA
// sets the sticky error word and the caller returns.
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// All threads of the CTA call this after their writes; thread 0 arrives.
__device__ __forceinline__ void grid_arrive(unsigned long long* ctr, bool skip) {
  __syncthreads();
  if (threadIdx.x == 0 && !skip) {
    __threadfence();
    atomicAdd(ctr, 1ull);
  }
}

// All threads call; returns false (for every thread) if the wait gave up.
__device__ __forceinline__ bool grid_wait(const unsigned long long* ctr, unsigned long long target,
                                          unsigned long long limit_ns, unsigned int* err,
                                          int* s_flag) {
  if (threadIdx.x == 0) {
    int ok = 1;
    if (ld_acquire_u64(ctr) < target) {
      const unsigned long long t0 = globaltimer_ns();
      while (ld_acquire_u64(ctr) < target) {
        if (globaltimer_ns() - t0 > limit_ns) {
          atomicOr(err, 1u);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    *s_flag = ok;
  }
  __syncthreads();
  const int ok = *s_flag;
  __syncthreads();
  return ok != 0;
}

// ---------------------------------------------------------------- dot helpers
// bf16 chunk (8 weights) dot the matching 8 fp32 activations.
__device__ __forceinline__ float dot8_bf16(uint4 w, float4 a, float4 b, float acc) {
  acc = fmaf(bf16lo(w.x), a.x, acc);
  acc = fmaf(bf16hi(w.x), a.y, acc);
  acc = fmaf(bf16lo(w.y), a.z, acc);
  acc = fmaf(bf16hi(w.y), a.w, acc);
  acc = fmaf(bf16lo(w.z), b.x, acc);
  acc = fmaf(bf16hi(w.z), b.y, acc);
  acc = fmaf(bf16lo(w.w), b.z, acc);
  acc = fmaf(bf16hi(w.w), b.w, acc);
  return acc;
}

// 8 dequantised codes (0.5 + n/256 form) dot 8 activations.
__device__ __forceinline__ float dot8_f(const float f[8], float4 a, float4 b, float acc) {
  acc = fmaf(f[0], a.x, acc);
  acc = fmaf(f[1], a.y, acc);
  acc = fmaf(f[2], a.z, acc);
  acc = fmaf(f[3], a.w, acc);
  acc = fmaf(f[4], b.x, acc);
  acc = fmaf(f[5], b.y, acc);
  acc = fmaf(f[6], b.z, acc);
  acc = fmaf(f[7], b.w, acc);
  return acc;
}

// ---------------------------------------------------------------- top-k
// Order-preserving key: larger logit first, then smaller index.
__device__ __forceinline__ unsigned long long topk_key(float v, int idx) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)idx);
}

// One warp: top-k of logits[0..E) by (value desc, index asc) and the
// renormalised softmax weights of the kept logits.
__device__ __forceinline__ void warp_topk(const float* logits, int E, int k, int* out_i, float* out_w) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = kMaxExperts / 32;
  unsigned long long key[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int e = lane + 32 * j;
    key[j] = (e < E) ? topk_key(ldcg_f32(logits + e), e) : 0ull;
  }
  float val[kMaxTopK];
  int idx[kMaxTopK];
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    val[r] = 0.f;
    idx[r] = 0;
    if (r < k) {
      unsigned long long best = 0ull;
#pragma unroll
      for (int j = 0; j < kPer; ++j) best = key[j] > best ? key[j] : best;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
        best = other > best ? other : best;
      }
      const int e = (int)(0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull));
#pragma unroll
      for (int j = 0; j < kPer; ++j)
        if (e == lane + 32 * j) key[j] = 0ull;
      idx[r] = e;
      val[r] = ldcg_f32(logits + e);
    }
  }
  if (lane == 0) {
    const float m = val[0];
    float sum = 0.f;
    float ex[kMaxTopK];
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r) {
      ex[r] = (r < k) ? expf(val[r] - m) : 0.f;
      sum += ex[r];
    }
    const float inv = 1.0f / sum;
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r)
      if (r < k) { out_i[r] = idx[r]; out_w[r] = ex[r] * inv; }
  }
}

// ---------------------------------------------------------------- smem layouts
// x as fp32 in two planes of 4-float chunks (chunk c = elements 8c..8c+7;
// plane 0 holds 8c..8c+3, plane 1 holds 8c+4..8c+7), one pad chunk after
// every 80 chunks so that the 4 K-quarters of the gate/up units fall in
// different banks.
constexpr int kXChunks = kH / 8;                       // 320
constexpr int kXPlane = (kXChunks + kXChunks / 80) * 4;  // 1296 floats
constexpr int kXTok = 2 * kXPlane;                     // 2592 floats
constexpr int kXGroups = kH / kGroup;                  // 80
// Routed intermediate activations h (fp32), padded by 4 floats per 96.
constexpr int kHpStride = kI + 4 * (kI / 96);          // 800 floats
constexpr int kHGroups = kI / kGroup;                  // 24
// Shared-expert h in two planes of 4-float chunks.
constexpr int kHsPlane = (kI / 8) * 4;                 // 384 floats
constexpr int kHsTok = 2 * kHsPlane;
// fp32 x of token t, chunk c (8 elements) -> the two float4 planes.
__device__ __forceinline__ int xoff(int c) { return 4 * (c + c / 80); }

__device__ __forceinline__ float scale_of(uint2 s4, int jj) {
  const uint32_t w = (jj < 2) ? s4.x : s4.y;
  return (jj & 1) ? bf16hi(w) : bf16lo(w);
}

}  // namespace lingmoe
