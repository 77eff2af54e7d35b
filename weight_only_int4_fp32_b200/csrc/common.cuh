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

__device__ __forceinline__ float silu_mul(float g, float u) {
  // SiLU(g) * u = g / (1 + e^-g) * u
  return g / (1.0f + expf(-g)) * u;
}
// The same for a token carried at scale 2^-sigma: g and u are the scaled
// gate and up values (true values s g, s u with s = 2^sigma) and the result is
// SiLU(s g) (s u) / s^2 = g u sigmoid(s g), which stays finite wherever g and
// u are.  With s = 1 it is silu_mul bit for bit.
__device__ __forceinline__ float silu_mul_scaled(float g, float u, float s) {
  return g / (1.0f + expf(-(g * s))) * u;
}
// Largest |x| of a token as bf16 magnitude bits (0..0x7F80 for finite x) ->
// the exponent sigma of its power-of-two scale: 0 while that |x| lies in
// [2^-3, 16) (the range the fixed scales of h are laid out for), otherwise
// the exponent that brings it into [2, 4), limited to [-100, 126] (a token
// whose largest |x| is below 2^-99 has an output below bf16's smallest
// subnormal either way).
__device__ __forceinline__ int token_sigma(uint32_t bf16_mag_bits) {
  if (bf16_mag_bits == 0u) return 0;
  const int e = (int)(bf16_mag_bits >> 7) - 127;  // subnormals count as 2^-127
  if (e >= -3 && e <= 3) return 0;
  return max(-100, min(126, e - 1));
}
// 2^e for e in [-126, 127]
__device__ __forceinline__ float pow2_int(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

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

// ---------------------------------------------------------------- smem layouts
// x as fp32 in two planes of 4-float chunks (chunk c = elements 8c..8c+7;
// plane 0 holds 8c..8c+3, plane 1 holds 8c+4..8c+7), one pad chunk after
// every 80 chunks so that the 4 K-quarters of the gate/up units fall in
// different banks.
constexpr int kXChunks = kH / 8;                       // 320
constexpr int kXPlane = (kXChunks + kXChunks / 80) * 4;  // 1296 floats
constexpr int kXTok = 2 * kXPlane;                     // 2592 floats
// Shared-expert h in two planes of 4-float chunks.
constexpr int kHsPlane = (kI / 8) * 4;                 // 384 floats
constexpr int kHsTok = 2 * kHsPlane;
// fp32 x of token t, chunk c (8 elements) -> the two float4 planes.
__device__ __forceinline__ int xoff(int c) { return 4 * (c + c / 80); }

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
// L2 eviction priorities for bulk copies: bytes read once (evict first) and
// bytes prefetched for a later read that should outlast other traffic
// (evict last).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy) : "memory");
}
__device__ __forceinline__ void prefetch_l2_bulk_hint(const void* p, uint32_t bytes, uint64_t policy) {
  asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;" :: "l"(p), "r"(bytes), "l"(policy)
               : "memory");
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
// The same, with one answer for the whole warp (for waits in front of
// warp-wide instructions: mma.sync, full-mask shuffles).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, unsigned long long limit_ns,
                                               unsigned int* err) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, limit_ns, err));
}
__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

// ---------------------------------------------------------------- cp.async (global -> shared, per thread)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" :: "r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" :: "r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
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
// ---------------------------------------------------------------- routed-weight codecs (layout.h)
// The E2M1 codes at bits P..P+3 and P+16..P+19 of a fragment word as the
// fp16 pair (value * 2^-14, exactly): with its magnitude bits E1 E0 M at
// fp16 bits 11..9 and its sign at bit 15, an fp16 is 2^(E - 15) (1 + M / 2)
// for E > 0 and the subnormal M 2^-15 for E = 0, i.e. the E2M1 value times
// 2^-14.  (The 2^14 is folded into the stored scale.)
template <int P>
__device__ __forceinline__ uint32_t deq_e2m1(uint32_t w) {
  static_assert(P >= 0 && P <= 12, "nibble position");
  uint32_t mag, sgn;
  if constexpr (P <= 9) mag = (w << (9 - P)) & 0x0E000E00u;
  else mag = (w >> (P - 9)) & 0x0E000E00u;
  sgn = (w << (12 - P)) & 0x80008000u;
  return mag | sgn;
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

// Exact codes of the pair of nibbles (1, 5) without the factor 16:
// (1024 + 16 n) / 16 - 72 = n - 8 = q, one rounding of an exact value.
__device__ __forceinline__ uint32_t deq_q_odd(uint32_t w) {
  uint32_t v, r;
  asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xEA;" : "=r"(v) : "r"(w));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(v), "r"(0x2C002C00u), "r"(0xD480D480u));  // 1/16, -72
  return r;
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- routed down on mma.sync
// The down units (layout.h) are the B operand of m16n8k16 MMAs whose 8
// columns are a unit's output rows.  The A operand is h: rows 0..7 of the A
// tile are up to 8 tokens' h * 2^-8 as fp16 (hi), rows 8..15 the remainders
// lo = fp16(h * 2^-8 - hi) of the same tokens, so one MMA takes both terms
// (~22 significant bits of h) and the accumulator rows g and g + 8 add up.
// A token's fragments in shared memory: for chunk j (128 K), group-in-chunk
// gg and K block b, lane class c = lane % 4 owns the 16 bytes
// (hi[k], hi[k+1]), (lo[k], lo[k+1]), (hi[k+8], hi[k+9]), (lo[k+8], lo[k+9])
// with k = 128 j + 32 gg + 16 b + 2 c, at byte ((8 j + 2 gg + b) * 4 + c) * 16.
constexpr int kHShift = 8;                       // h is scaled by 2^-8 before the split
constexpr int kHfTokBytes = kDnChunks * 512;     // 3072
constexpr int kHfStride = kHfTokBytes + 64;      // consecutive tokens in opposite bank halves
__device__ __forceinline__ int hf_off(int k) {   // byte of (hi[k], hi[k+1]) for even k
  const int G = k >> 5, b = (k >> 4) & 1, kk = k & 15;
  return ((8 * (G >> 2) + 2 * (G & 3) + b) * 4 + ((kk & 7) >> 1)) * 16 + (kk >= 8 ? 8 : 0);
}
// (hi pair, lo pair) of two consecutive h values
__device__ __forceinline__ uint2 h_split2(float h0, float h1) {
  const float a = h0 * (1.0f / (float)(1 << kHShift)), b = h1 * (1.0f / (float)(1 << kHShift));
  const __half2 hi = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(hi);
  const __half2 lo = __floats2half2_rn(a - hf.x, b - hf.y);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&hi), *reinterpret_cast<const uint32_t*>(&lo));
}
// One down unit (kDnUnitBytes in shared memory) against the h of up to 8
// tokens.  Lane (g = lane / 4, c = lane % 4) returns token g's sums for the
// unit's rows 2c and 2c + 1, times 2^-8, over chunks j0 .. j1 - 1 of K
// (default: all of K).  hf points at this lane's token's fragments plus 16 c.
// A lane without a token of its own points at any valid token (its
// accumulator row is discarded): the loads stay unconditional, so the MMAs
// of different groups can overlap.  Every lane of the warp must call it.
// C: the codec of the unit's codes (the scales already carry its factor).
template <int C = kCodecInt4>
__device__ __forceinline__ void dn_unit_mma(const unsigned char* unit, const unsigned char* hf, int lane, float& r0,
                                            float& r1, int j0 = 0, int j1 = kDnChunks) {
  const int c = lane & 3;
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 2
  for (int j = j0; j < j1; ++j) {
    const uint4 w = lds128(unit + j * 512 + 16 * lane);
    const uint4 s = lds128(unit + kDnScaleOff + j * 64 + 16 * c);
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w}, sv[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
    for (int gg = 0; gg < 4; ++gg) {
      const uint4 a0 = lds128(hf + (8 * j + 2 * gg) * 64);
      const uint4 a1 = lds128(hf + (8 * j + 2 * gg + 1) * 64);
      float d0, d1, d2, d3;
      if constexpr (C == kCodecMxfp4) {
        mma_16816(d0, d1, d2, d3, a0.x, a0.y, a0.z, a0.w, deq_e2m1<0>(wv[gg]), deq_e2m1<4>(wv[gg]), 0.f, 0.f, 0.f,
                  0.f);
        mma_16816(d0, d1, d2, d3, a1.x, a1.y, a1.z, a1.w, deq_e2m1<8>(wv[gg]), deq_e2m1<12>(wv[gg]), d0, d1, d2, d3);
      } else {
        mma_16816(d0, d1, d2, d3, a0.x, a0.y, a0.z, a0.w, deq_q_even(wv[gg]), deq_q_odd(wv[gg]), 0.f, 0.f, 0.f,
                  0.f);
        mma_16816(d0, d1, d2, d3, a1.x, a1.y, a1.z, a1.w, deq_q_even(wv[gg] >> 8), deq_q_odd(wv[gg] >> 8), d0, d1,
                  d2, d3);
      }
      acc0 = fmaf(bf16lo(sv[gg]), d0 + d2, acc0);
      acc1 = fmaf(bf16hi(sv[gg]), d1 + d3, acc1);
    }
  }
  r0 = acc0;
  r1 = acc1;
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
// lg may hold logits divided by a power of two s (a rescaled token): the
// weights then take wscale = s, exp(s (l_r - l_0)).
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
__device__ __forceinline__ void warp_topk_fast(const float* lg, int E, int k, int* out_i, float* out_w,
                                               float wscale = 1.0f) {
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
  const float ex = (lane < k) ? expf((vr - vmax) * wscale) : 0.f;
  float s = ex;
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane < k) {
    out_i[lane] = (unsigned)mine_i < (unsigned)E ? mine_i : 0;  // always in [0, E)
    out_w[lane] = ex / s;
  }
  __syncwarp();
}

// The same selection with fewer dependent steps (one warp, k <= 8,
// E <= 512): keys are 64-bit (order key of the logit, then 0xFFFF - index),
// all distinct, so (logit desc, index asc) is plain key order.  The k-th
// largest lane maximum (found by redux.sync rounds over the 32-bit order
// keys, lanes that tie dropping out together) bounds the k-th largest key
// from below, so every selected key is a candidate; the few candidates are
// gathered in shared memory and each one's rank among them is counted.  With
// more than 32 candidates (heavy ties) the round-by-round selection above
// takes over.  scratch: 40 x 8 bytes of this warp's shared memory.
// Returns the same indices and weights as warp_topk_fast.
__device__ __forceinline__ void warp_topk_thresh(const float* lg, int E, int k, unsigned long long* scratch,
                                                 int* out_i, float* out_w, float wscale = 1.0f) {
  const int lane = threadIdx.x & 31;
  unsigned long long key[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int e = lane + 32 * j;
    key[j] = e < E ? ((unsigned long long)f32_order_key(lg[e]) << 32) | (unsigned long long)(0xFFFF - e) : 0ull;
  }
  uint32_t mx = 0u;
#pragma unroll
  for (int j = 0; j < 16; ++j) mx = max(mx, (uint32_t)(key[j] >> 32));
  uint32_t cur = mx, tau32 = 0u;
  int counted = 0;
#pragma unroll 1
  for (int r = 0; r < 32 && counted < k; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, cur);
    counted += __popc(__ballot_sync(0xffffffffu, cur == m));
    tau32 = m;
    cur = cur == m ? 0u : cur;
  }
  const unsigned long long tau = (unsigned long long)tau32 << 32;
  unsigned int mask = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) mask |= (key[j] >= tau && key[j] != 0ull ? 1u : 0u) << j;
  const int cnt = __popc(mask);
  int off = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, off, o);
    if (lane >= o) off += v;
  }
  const int total = __shfl_sync(0xffffffffu, off, 31);
  off -= cnt;
  if (total > 32) {
    warp_topk_fast(lg, E, k, out_i, out_w, wscale);
    return;
  }
  unsigned long long* cand = scratch;
  unsigned long long* sel = scratch + 32;
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (mask >> j & 1u) cand[off++] = key[j];
  __syncwarp();
  const unsigned long long mine = lane < total ? cand[lane] : 0ull;
  int r = 0;
  for (int o = 0; o < total; ++o) r += cand[o] > mine;
  __syncwarp();
  if (lane < total && r < k) sel[r] = mine;  // the r-th selection
  __syncwarp();
  const unsigned long long s_l = lane < k ? sel[lane] : 0ull;
  const float v0 = f32_from_order_key((uint32_t)(sel[0] >> 32));
  const float vr = f32_from_order_key((uint32_t)(s_l >> 32));
  const float ex = lane < k ? expf((vr - v0) * wscale) : 0.f;
  float s = ex;
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane < k) {
    const int e = 0xFFFF - (int)(s_l & 0xFFFFu);
    out_i[lane] = (unsigned)e < (unsigned)E ? e : 0;  // always in [0, E)
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
