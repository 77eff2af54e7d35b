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

// ---------------------------------------------------------------- mbarrier + bulk copy
// Non-multicast TMA bulk copies (global -> this CTA's shared memory) completing
// on an mbarrier.  Addresses 16-byte aligned, sizes multiples of 16.
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
// The thread sleeps (up to kMbarSuspendNs) until the phase completes instead
// of returning at once, so waiting warps leave the issue slots to the warps
// that compute.
constexpr uint32_t kMbarSuspendNs = 20000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(kMbarSuspendNs) : "memory");
  return ok != 0;
}
// Bounded wait for phase `parity` of the barrier; false (and the sticky error
// word set) if it did not complete within limit_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned long long limit_ns,
                                          unsigned int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(err, 2u);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ float4 ldsf4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// ---------------------------------------------------------------- mixed-precision FMA
// d = a * b + c with a, b taken from one half (lo = 0, hi = 1) of packed
// 16-bit pairs and c, d in fp32; the product of two 16-bit values is exact in
// fp32, so only the accumulation rounds.
#define LING_MIXED_FMA_ASM(TYPE, A, B)                                   \
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"                                  \
      "mov.b32 {al, ah}, %1;\n\t"                                           \
      "mov.b32 {bl, bh}, %2;\n\t"                                           \
      "fma.rn.f32." TYPE " %0, " A ", " B ", %3;\n\t}"                       \
      : "=f"(d) : "r"(a2), "r"(b2), "f"(c))
template <int AH, int BH>
__device__ __forceinline__ float fma_bf16h(uint32_t a2, uint32_t b2, float c) {
  float d;
  if constexpr (AH == 0 && BH == 0) LING_MIXED_FMA_ASM("bf16", "al", "bl");
  else if constexpr (AH == 0 && BH == 1) LING_MIXED_FMA_ASM("bf16", "al", "bh");
  else if constexpr (AH == 1 && BH == 0) LING_MIXED_FMA_ASM("bf16", "ah", "bl");
  else LING_MIXED_FMA_ASM("bf16", "ah", "bh");
  return d;
}
template <int AH, int BH>
__device__ __forceinline__ float fma_f16h(uint32_t a2, uint32_t b2, float c) {
  float d;
  if constexpr (AH == 0 && BH == 0) LING_MIXED_FMA_ASM("f16", "al", "bl");
  else if constexpr (AH == 0 && BH == 1) LING_MIXED_FMA_ASM("f16", "al", "bh");
  else if constexpr (AH == 1 && BH == 0) LING_MIXED_FMA_ASM("f16", "ah", "bl");
  else LING_MIXED_FMA_ASM("f16", "ah", "bh");
  return d;
}

// 8 bf16 weights (one 16-byte chunk) dot 8 bf16 activations, fp32 accumulate.
__device__ __forceinline__ float dot8_bf16_bf16(uint4 w, uint4 x, float acc) {
  acc = fma_bf16h<0, 0>(w.x, x.x, acc);
  acc = fma_bf16h<1, 1>(w.x, x.x, acc);
  acc = fma_bf16h<0, 0>(w.y, x.y, acc);
  acc = fma_bf16h<1, 1>(w.y, x.y, acc);
  acc = fma_bf16h<0, 0>(w.z, x.z, acc);
  acc = fma_bf16h<1, 1>(w.z, x.z, acc);
  acc = fma_bf16h<0, 0>(w.w, x.w, acc);
  acc = fma_bf16h<1, 1>(w.w, x.w, acc);
  return acc;
}

// int4 -> fp16 with one LOP3 per two codes.  For a 32-bit word holding 8
// offset-binary nibbles n_0..n_7 (n = q + 8, nibble i at bits 4i..4i+3,
// element i of the word), (w & 0x000F000F) | 0x64006400 is the fp16 pair
// (1024 + n_0, 1024 + n_4) and (w & 0x00F000F0) | 0x64006400 is
// (1024 + 16 n_1, 1024 + 16 n_5); the same on w >> 8 gives elements 2, 6
// and 3, 7.  Even elements carry 1024 + n, odd ones 1024 + 16 n, so for a
// group of 32 codes with activations x (fp16):
//   sum_k q_k x_k = (A_even - 1032 S_even) + (A_odd - 1152 S_odd) / 16
// with A the fp32 FMA sums of the fp16 products and S the sums of x over the
// even / odd positions.  Each fp16 x fp16 product is exact in fp32.
struct Pairs4 { uint32_t p0, p1, p2, p3; };
__device__ __forceinline__ Pairs4 dequant_f16x2(uint32_t w) {
  Pairs4 r;
  const uint32_t w8 = w >> 8;
  asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(r.p0) : "r"(w));
  asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xEA;" : "=r"(r.p1) : "r"(w));
  asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(r.p2) : "r"(w8));
  asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xEA;" : "=r"(r.p3) : "r"(w8));
  return r;
}
// Exact codes from a fragment word (offset-binary nibbles): the pair of
// nibbles (0, 4) as fp16 (q0, q4) = (1024 + n) - 1032, and the pair (1, 5)
// as 16 q = (1024 + 16 n) - 1152; w >> 8 gives the pairs (2, 6) and (3, 7).
__device__ __forceinline__ uint32_t deq_q_even(uint32_t w) {
  uint32_t v, r;
  asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(v) : "r"(w));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(0x64086408u));  // 1032
  return r;
}
__device__ __forceinline__ uint32_t deq_q_odd16(uint32_t w) {
  uint32_t v, r;
  asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xEA;" : "=r"(v) : "r"(w));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(0x64806480u));  // 1152
  return r;
}
// D = A B + C for one m16n8k16 tile: A 16x16 fp16 (row-major fragment),
// B 16x8 fp16 (column-major fragment), C and D fp32.
__device__ __forceinline__ void mma_16816(float& d0, float& d1, float& d2, float& d3, uint32_t a0, uint32_t a1,
                                          uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1, float c0, float c1,
                                          float c2, float c3) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d0), "=f"(d1), "=f"(d2), "=f"(d3)
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2), "f"(c3));
}

constexpr float kEvenBias = -1032.0f;
constexpr float kOddBias = -1152.0f;
// acc_e += even products, acc_o += odd products of one word (8 codes) with
// the 8 fp16 activations x = (x0..x7) packed in a uint4.
__device__ __forceinline__ void dot8_q_f16(const Pairs4& P, uint4 x, float& ae, float& ao) {
  ae = fma_f16h<0, 0>(P.p0, x.x, ae);  // e0 * x0
  ae = fma_f16h<1, 0>(P.p0, x.z, ae);  // e4 * x4
  ae = fma_f16h<0, 0>(P.p2, x.y, ae);  // e2 * x2
  ae = fma_f16h<1, 0>(P.p2, x.w, ae);  // e6 * x6
  ao = fma_f16h<0, 1>(P.p1, x.x, ao);  // e1 * x1
  ao = fma_f16h<1, 1>(P.p1, x.z, ao);  // e5 * x5
  ao = fma_f16h<0, 1>(P.p3, x.y, ao);  // e3 * x3
  ao = fma_f16h<1, 1>(P.p3, x.w, ao);  // e7 * x7
}

// ---------------------------------------------------------------- top-k
// Order-preserving 32-bit key of a float: larger float, larger key.
__device__ __forceinline__ uint32_t f32_order_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float f32_from_order_key(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// One warp: top-k (k <= 8) of lg[0..E) (E <= 512) by (value desc, index asc)
// and the renormalised softmax weights of the kept logits.
// Lane l holds entries l, l + 32, ... as order keys (0 marks a removed or
// absent entry).  Each lane keeps its best entry (largest key, lowest index
// among equal keys) from a 4-level comparison tree.  A round takes the
// warp-wide largest key with redux.sync, then the lowest index among the
// lanes holding it (a second redux.sync on 0xFFFF - index); the owner
// removes the entry and rebuilds its tree.  Lane r keeps the result of
// round r.  Lane r < k writes slot r and exp(l_r - l_0) / sum_s exp(l_s - l_0).
__device__ __forceinline__ void lane_best16(const uint32_t key[16], uint32_t& bk, int& bj) {
  uint32_t k8[8];
  int j8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = key[2 * i + 1] > key[2 * i];
    k8[i] = hi ? key[2 * i + 1] : key[2 * i];
    j8[i] = hi ? 2 * i + 1 : 2 * i;
  }
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1) {
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const bool hi = k8[2 * i + 1] > k8[2 * i];
      k8[i] = hi ? k8[2 * i + 1] : k8[2 * i];
      j8[i] = hi ? j8[2 * i + 1] : j8[2 * i];
    }
  }
  bk = k8[0];
  bj = j8[0];
}
__device__ __forceinline__ void warp_topk_fast(const float* lg, int E, int k, int* out_i, float* out_w) {
  const int lane = threadIdx.x & 31;
  uint32_t key[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int e = lane + 32 * j;
    key[j] = (e < E) ? f32_order_key(lg[e]) : 0u;
  }
  uint32_t bk;
  int bj;
  lane_best16(key, bk, bj);
  uint32_t mine_k = 0u;
  int mine_i = 0;
#pragma unroll 1
  for (int r = 0; r < k; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t cand = (bk == m) ? 0xFFFFu - (uint32_t)(lane + 32 * bj) : 0u;
    const uint32_t c = __reduce_max_sync(0xffffffffu, cand);
    const int idx = (int)(0xFFFFu - c);
    if (lane == r) {
      mine_k = m;
      mine_i = idx;
    }
    const int kj = (lane == (idx & 31)) ? (idx >> 5) : -1;  // the owner's entry
#pragma unroll
    for (int j = 0; j < 16; ++j) key[j] = (j == kj) ? 0u : key[j];
    if (kj >= 0) lane_best16(key, bk, bj);
  }
  const float vmax = f32_from_order_key(__shfl_sync(0xffffffffu, mine_k, 0));
  const float vr = f32_from_order_key(mine_k);
  const float ex = (lane < k) ? expf(vr - vmax) : 0.f;
  float s = ex;
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane < k) {
    out_i[lane] = mine_i < E ? mine_i : 0;  // only a NaN logit could select past the end
    out_w[lane] = ex / s;
  }
  __syncwarp();
}

// Two-accumulator variants (even / odd elements) to halve dependent chains.
__device__ __forceinline__ void dot8_bf16_bf16_2(uint4 w, uint4 x, float& a, float& b) {
  a = fma_bf16h<0, 0>(w.x, x.x, a);
  b = fma_bf16h<1, 1>(w.x, x.x, b);
  a = fma_bf16h<0, 0>(w.y, x.y, a);
  b = fma_bf16h<1, 1>(w.y, x.y, b);
  a = fma_bf16h<0, 0>(w.z, x.z, a);
  b = fma_bf16h<1, 1>(w.z, x.z, b);
  a = fma_bf16h<0, 0>(w.w, x.w, a);
  b = fma_bf16h<1, 1>(w.w, x.w, b);
}
__device__ __forceinline__ void dot8_f_2(const float f[8], float4 x0, float4 x1, float& a, float& b) {
  a = fmaf(f[0], x0.x, a);
  b = fmaf(f[1], x0.y, b);
  a = fmaf(f[2], x0.z, a);
  b = fmaf(f[3], x0.w, b);
  a = fmaf(f[4], x1.x, a);
  b = fmaf(f[5], x1.y, b);
  a = fmaf(f[6], x1.z, a);
  b = fmaf(f[7], x1.w, b);
}
__device__ __forceinline__ void dot8_bf16_2(uint4 w, float4 x0, float4 x1, float& a, float& b) {
  a = fmaf(bf16lo(w.x), x0.x, a);
  b = fmaf(bf16hi(w.x), x0.y, b);
  a = fmaf(bf16lo(w.y), x0.z, a);
  b = fmaf(bf16hi(w.y), x0.w, b);
  a = fmaf(bf16lo(w.z), x1.x, a);
  b = fmaf(bf16hi(w.z), x1.y, b);
  a = fmaf(bf16lo(w.w), x1.z, a);
  b = fmaf(bf16hi(w.w), x1.w, b);
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned int* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

}  // namespace lingmoe
