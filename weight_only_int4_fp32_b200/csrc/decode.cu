// Decode / verify path (1 <= T <= kMaxDecodeT) of the W4 g32 MoE layer.
//
// One persistent launch per call, one CTA per SM, co-resident (cooperative
// launch), specialised at compile time for the token count T.  The work is a
// chain router -> top-k -> routed gate/up -> down, so the CTAs meet at
// bounded grid barriers:
//
//   phase 1+2  router logits (bf16 GEMV, fp32) and shared-expert
//              gate/up + SiLU*up (bf16)                        -> barriers A, B
//   phase 3    wait A; every CTA selects the top-k itself; routed gate/up
//              (W4 g32, dequantised in registers) + SiLU*up     -> barrier C
//   phase 4    routed down (W4 g32, mma.sync with h as fp16 hi + lo) weighted
//              by the routing weights and shared down (bf16), summed in a
//              fixed order, one bf16 rounding.
//
// Weight bytes move HBM -> shared memory by non-multicast TMA bulk copies,
// one private buffer and mbarrier per warp; each warp issues the copy of its
// next item before it waits, and the compute loops read the staged bytes with
// conflict-free 16-byte shared loads.  Bytes that do not depend on the
// routing (shared expert) are requested first.  A routed gate/up unit is
// copied in four pieces with one mbarrier each, so its dot products start
// when the first piece lands.  For one token the CTA's routed down units are
// copied into a dedicated shared-memory region as soon as the CTA's own
// gate/up work is done (they land while the grid exchanges h); otherwise
// they are prefetched into L2 once the routing is known and copied in
// batches while the CTA waits at the last grid barrier.  A CTA owns whole
// 8-row down units (the granularity of the routed down layout), so its
// output rows need no exchange with other CTAs.
//
// Layer definition: vLLM recipe page "inclusionAI/Ling-3.0-flash" (Overview;
// "Single-GPU int4": symmetric W4, group 32, routed experts only) and the
// bpdata article "Harom optimalizacio a Ling-3.0-flash MoE inferenciajanak"
// ("Modell es kiindulo konfiguracio": 8 of 512 routed experts + 1 shared).
#include <type_traits>

#include "common.cuh"
#include "decode.h"

namespace lingmoe {

// Optional phase timestamps (compile with -DLING_MOE_TRACE): thread 0 of
// every CTA records %globaltimer at each phase boundary.
#ifdef LING_MOE_TRACE
__device__ float g_sink;
__device__ __forceinline__ void g_clk_sink(float v) { if (v == 12345.f) g_sink = v; }
__device__ unsigned long long g_trace[1024][16];
__device__ long long g_clk[16];
#define LING_CLK(slot) \
  do { if (blockIdx.x == 0 && threadIdx.x == 0) g_clk[slot] = clock64(); } while (0)
#else
#define LING_CLK(slot) do { } while (0)
__device__ __forceinline__ void g_clk_sink(float) {}
#endif
#ifdef LING_MOE_TRACE
#define LING_TRACE(slot) \
  do { if (threadIdx.x == 0) g_trace[blockIdx.x][slot] = globaltimer_ns(); } while (0)
#else
#define LING_TRACE(slot) do { } while (0)
#endif

constexpr int kWarps = kDecodeWarps;
constexpr int kBufA = kGuHalfBytes;                 // per-warp buffer, phases 1-3 (one K half of a unit)
constexpr int kShDnBytes = 4 * kI * 2;              // 4 shared-down rows (half a row-block)
// routed down units per copy batch (one above 4 tokens: shared memory goes to
// h), and the per-warp phase-4 buffer (a batch or a shared-down block)
template <int T> __host__ __device__ constexpr int dn_batch() { return T > 4 ? 1 : 2; }
template <int T> __host__ __device__ constexpr int dn_buf() { return T > 4 ? kShDnBytes : 2 * kDnUnitBytes; }
// Routed h staged in shared memory as fp16 hi + lo A fragments: every pair up
// to 4 tokens (indexed by pair); above, at most kHfCapBig pairs at a time,
// experts taken in union order, so that phase 4 runs in at most two passes
// (the first takes more than kHfCapBig - 8 pairs, leaving at most 33 of 64).
constexpr int kHfCapBig = 38;
template <int T> __host__ __device__ constexpr int hf_cap() { return T > 4 ? kHfCapBig : T * kMaxTopK; }
constexpr int kMaxBlkPerCta = 4;                    // 8-row down blocks per CTA (>= 320 / nctas, nctas >= 80)
constexpr int kDnPrefBlk = 3;                       // T = 1: routed down units kept in shared memory
                                                    // when the CTA has <= 3 row-blocks (>= 107 CTAs)
constexpr int kGuPiece = kGuHalfCodes / 4;          // 2560 B: 5 chunks of a gate/up half-unit
constexpr int kPairs = kDecodeWarps / 2;            // phase-3 warp pairs (one K half each)
constexpr int kRowBytes = kH * 2;                   // one bf16 row of H
static_assert(dn_buf<8>() >= kShDnBytes && dn_buf<1>() >= kShDnBytes && dn_buf<8>() >= kDnUnitBytes,
              "phase-4 buffer holds a batch or a shared-down block");
static_assert(kBufA >= 2 * kRowBytes, "phase-1/2 buffer holds a gate and an up row");

struct __align__(128) SmemHeader {  // 128-byte multiple: the body starts on a full line
  uint64_t mbar[kWarps][4];
  uint64_t xbar;
  uint64_t dbar;
  uint32_t xmax[kMaxDecodeT];   // largest |x| of each token, bf16 magnitude bits
  float xscale[kMaxDecodeT];    // s_t = 2^sigma_t (1 for most tokens)
  float xinv[kMaxDecodeT];      // 1 / s_t
  int topi[kMaxDecodeT][kMaxTopK];
  float topw[kMaxDecodeT][kMaxTopK];
  int uniq_e[kMaxDecodeT * kMaxTopK];
  int uniq_cnt[kMaxDecodeT * kMaxTopK];
  int uniq_pair[kMaxDecodeT * kMaxTopK][kMaxDecodeT];
  int uniq_slot[kMaxDecodeT * kMaxTopK];  // T > 4: the expert's first h row in its pass
  int slot_pair[2][kHfCapBig];            // T > 4: pair id of each h row, per pass
  int nslot[2];                           // T > 4: h rows per pass
  int u_split;                            // T > 4: experts [0, u_split) form the first pass
  int nuniq;
  int dcopies;  // T = 1: routed down copies into the dedicated region were issued
  unsigned long long epoch;  // launch index (see the arrival counters)
  int abort;
  int pad[3];
};
static_assert(sizeof(SmemHeader) % 128 == 0, "header keeps the body 128-byte aligned");

// x is kept twice: the bf16 input as staged (router and shared rows read it
// with mixed-precision FMAs) and an fp16 copy in MMA B-fragment order for the
// routed gate/up.  A token whose largest |x| lies outside [2^-3, 16) is first
// divided by its power-of-two scale s_t in place (exact); everything after
// that runs on x / s_t: the router adds b / s_t and weighs by exp(s_t (l -
// l_0)), h is kept as h / s_t^2 (silu_mul_scaled) and the output is
// multiplied by s_t twice before its bf16 rounding.  Per chunk of 64 K, per lane
// class m = lane % 4, per K block w, the pair (x[c], x[c+1]) and the pair
// (x[c+8], x[c+9]) / 16 with c = 16 kb + 2 m (the /16 matches the 16 q form
// in which the upper half of a block's codes is dequantised).
constexpr int kXbTok = kH * 2;                   // bytes per token, bf16
constexpr int kXfTok = (kH / 64) * 128;          // 5120 bytes per token

// Shared-memory plan (byte offsets into the body).  Region A (phases 1-3)
// and region B (phase 4) overlap: B is used only after the CTA's own phase 3,
// and so is region D (T = 1), which follows B.
template <int T>
struct Plan {
  static constexpr int P = T * kMaxTopK;
  static constexpr size_t xb = 0;                                           // [T][kXbTok]
  static constexpr size_t xf = xb + (size_t)T * kXbTok;                     // [T][kXfTok]
  static constexpr size_t comb = xf + (size_t)T * kXfTok;                   // float [pairs][2][32][4]
  static constexpr size_t bufA = comb + (size_t)kPairs * 2 * 32 * 16;       // [warps][kBufA]
  static constexpr size_t endA = bufA + (size_t)kWarps * kBufA;
  static constexpr size_t hf = 0;                                           // [hf_cap][kHfStride] h as MMA A fragments
  static constexpr size_t hs = hf + (size_t)hf_cap<T>() * kHfStride;        // float [T][kHsTok]
  static constexpr size_t part = hs + (size_t)T * kHsTok * 4;               // float [blk][P + T][8]
  static constexpr size_t bufB = part + (size_t)kMaxBlkPerCta * (P + T) * 32;
  static constexpr size_t endB = bufB + (size_t)kWarps * dn_buf<T>();
  // T = 1: the CTA's routed down units, [expert slot][row-block] x kDnUnitBytes
  static constexpr size_t dn = endB;
  static constexpr size_t endD = dn + (T == 1 ? (size_t)kMaxTopK * kDnPrefBlk * kDnUnitBytes : 0);
  static constexpr size_t body = endA > endD ? endA : endD;
  static constexpr size_t bytes = sizeof(SmemHeader) + body;
  static_assert(xf % 16 == 0 && comb % 16 == 0 && bufA % 16 == 0 && bufB % 16 == 0 && hs % 16 == 0 &&
                part % 16 == 0 && dn % 16 == 0, "16-byte aligned regions");
  static_assert(bytes <= 227 * 1024, "decode smem over budget");
};

size_t decode_smem_bytes(int T) {
  switch (T) {
    case 1: return Plan<1>::bytes;
    case 2: return Plan<2>::bytes;
    case 3: return Plan<3>::bytes;
    case 4: return Plan<4>::bytes;
    case 5: return Plan<5>::bytes;
    case 6: return Plan<6>::bytes;
    case 7: return Plan<7>::bytes;
    default: return Plan<8>::bytes;
  }
}

__device__ __forceinline__ bool aborted(const SmemHeader& hd) {
  return *reinterpret_cast<const volatile int*>(&hd.abort) != 0;
}

// ---------------------------------------------------------------- arrival counters
// Publish: the calling thread's earlier stores (and, after a warp or CTA
// barrier, those of the other threads) become visible before the count.
// The counters only grow (64-bit): launch L waits for (L + 1) x its per-launch
// total, so nothing has to be reset between launches.
__device__ __forceinline__ void arrive(unsigned long long* ctr) {
  __threadfence();
  atomicAdd(ctr, 1ull);
}
// Bounded poll until *ctr >= target.  On time-out sets the error word and the
// CTA's abort flag; returns false.
__device__ __forceinline__ bool wait_count(const unsigned long long* ctr, unsigned long long target,
                                           unsigned long long limit_ns, unsigned int* err, int* abort) {
  if (ld_acquire_u64(ctr) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (ld_acquire_u64(ctr) < target) {
    if (*reinterpret_cast<volatile int*>(abort) || globaltimer_ns() - t0 > limit_ns) {
      atomicOr(err, 1u);
      *reinterpret_cast<volatile int*>(abort) = 1;
      return false;
    }
  }
  return true;
}

// C: the codec of the routed weights (kCodecInt4 or kCodecMxfp4).  EP: the
// variant that honours an expert range, shared_on and out_f32 (expert-parallel
// handles and fp32 partial outputs); the ordinary variant computes every
// expert and the shared expert into a bf16 out, with none of that code.
template <int T, int C, bool EP>
__global__ void __launch_bounds__(kDecodeThreads, 1) moe_decode_kernel(const DecodeParams p) {
  using PL = Plan<T>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  SmemHeader& hd = *reinterpret_cast<SmemHeader*>(smem_raw);
  unsigned char* body = smem_raw + sizeof(SmemHeader);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cta = blockIdx.x, ncta = gridDim.x;
  const int E = p.E, K = p.k;
  LING_TRACE(0);

  const bool withhold = (cta == p.skip_arrive_cta);

  // this CTA's slices
  const int r0 = (int)((long long)cta * E / ncta), r1 = (int)((long long)(cta + 1) * E / ncta);
  const int s0 = cta * kI / ncta, s1 = (cta + 1) * kI / ncta;
  const int b0 = cta * kDnUnits / ncta, b1 = (cta + 1) * kDnUnits / ncta;
  const int nblk = b1 - b0;
  const bool sh_on = !EP || p.shared_on;                   // the shared expert is computed here
  const int e0 = EP ? p.e0 : 0, e_local = EP ? p.e_local : E;  // the experts held here
  const bool ep = EP && e_local != E;
  const int nr = r1 - r0, n12 = nr + (sh_on ? s1 - s0 : 0);

  uint64_t* barA = &hd.mbar[warp][0];  // phases 1-2 items, piece 0 of a gate/up unit, phase-4 copies
  uint32_t pha = 0, phq = 0;           // phq: parity of pieces 1-3 (always used together)
  const bool use_d = (T == 1) && nblk <= kDnPrefBlk;
  unsigned char* bufA = body + PL::bufA + (size_t)warp * kBufA;
  unsigned char* bufB = body + PL::bufB + (size_t)warp * dn_buf<T>();
  unsigned char* xb = body + PL::xb;
  unsigned char* xf = body + PL::xf;
  if (tid < kMaxDecodeT) {
    hd.xmax[tid] = 0u;
    hd.xscale[tid] = 1.0f;
    hd.xinv[tid] = 1.0f;
  }
  // Launch index of this call: every CTA of the earlier launches on the
  // stream has counted itself out, and no CTA of this one can before all
  // have passed the router barrier (which comes after this read).
  // (the load is issued here; its value is first needed at the routing)
  const unsigned long long done_ctas = (tid == 0) ? ld_acquire_u64(p.sync + 3) : 0ull;
  if (tid == 0) {
    hd.abort = 0;
    hd.dcopies = 0;
    hd.nslot[1] = 0;  // one phase-4 pass unless the union sets a second
    mbar_init(&hd.xbar, 1);
    mbar_init(&hd.dbar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&hd.xbar, T * kXbTok);
    bulk_g2s(xb, p.x, T * kXbTok, &hd.xbar);
  }
  if (lane == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&hd.mbar[warp][i], 1);
    fence_mbar_init();
  }
  __syncthreads();  // barriers initialised before anyone waits on them

  // phase-1/2 item `it`: router row (it < nr) or shared gate+up rows
  auto issue12 = [&](int it) {
    if (lane == 0) {
      if (it < nr) {
        mbar_arrive_expect_tx(barA, kRowBytes);
        bulk_g2s(bufA, p.router_w + (size_t)(r0 + it) * kH, kRowBytes, barA);
      } else {
        const int i = s0 + it - nr;
        mbar_arrive_expect_tx(barA, 2 * kRowBytes);
        bulk_g2s(bufA, p.sh_gate + (size_t)i * kH, kRowBytes, barA);
        bulk_g2s(bufA + kRowBytes, p.sh_up + (size_t)i * kH, kRowBytes, barA);
      }
    }
  };
  if (warp < n12) issue12(warp);

  // L2 prefetch of the shared down rows this CTA will need
  if (sh_on && warp == kWarps - 1 && lane == 0 && nblk > 0)
    prefetch_l2_bulk(p.sh_down + (size_t)b0 * kDnUnitRows * kI, (uint32_t)nblk * 2 * kShDnBytes);

  // x (bf16) lands in shared memory; every warp waits for it once
  if (!mbar_wait(&hd.xbar, 0, p.wait_limit_ns, p.err)) hd.abort = 1;
  LING_TRACE(1);
  // fp16 copy of x in B-fragment order, built as soon as x lands (the first
  // weight rows are still in flight), together with each token's largest |x|.
  // A warp's 32 items never straddle two tokens (640 items per token).
  auto build_xh = [&](bool track) {
    for (int v = tid; v < T * (kH / 4); v += kDecodeThreads) {
      const int t = v / (kH / 4), r = v - t * (kH / 4), kb = r >> 2, m = r & 3;
      const int c = 16 * kb + 2 * m;
      const uint32_t lo = *reinterpret_cast<const uint32_t*>(xb + t * kXbTok + 2 * c);
      const uint32_t hi = *reinterpret_cast<const uint32_t*>(xb + t * kXbTok + 2 * (c + 8));
      const __half2 h0 = __floats2half2_rn(bf16lo(lo), bf16hi(lo));
      // int4: the upper half meets codes dequantised as 16 q, so it carries 1/16
      constexpr float kHiFactor = C == kCodecInt4 ? 0.0625f : 1.0f;
      const __half2 h1 = __floats2half2_rn(bf16lo(hi) * kHiFactor, bf16hi(hi) * kHiFactor);
      if (track) {
        const uint32_t mag = __vmaxu2(lo & 0x7FFF7FFFu, hi & 0x7FFF7FFFu);
        const uint32_t wm = __reduce_max_sync(0xffffffffu, max(mag & 0xFFFFu, mag >> 16));
        if (lane == 0) atomicMax(&hd.xmax[t], wm);
      }
      *reinterpret_cast<uint2*>(xf + t * kXfTok + (kb >> 2) * 128 + m * 32 + (kb & 3) * 8) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
    }
  };
  build_xh(true);
  __syncthreads();
  {
    int sig[T];
    bool any = false;
#pragma unroll
    for (int t = 0; t < T; ++t) {
      sig[t] = token_sigma(hd.xmax[t]);
      any |= sig[t] != 0;
    }
    if (any) {
      // rare: a token outside the direct range; x / s_t in place, then the
      // fp16 copy again
      if (tid < T) {
        const int st = token_sigma(hd.xmax[tid]);
        hd.xscale[tid] = pow2_int(st);
        hd.xinv[tid] = pow2_int(-st);
      }
      for (int v = tid; v < T * kXChunks; v += kDecodeThreads) {
        const int t = v / kXChunks, c = v - t * kXChunks;
        int st = 0;
#pragma unroll
        for (int q = 0; q < T; ++q)
          if (q == t) st = sig[q];
        if (st == 0) continue;
        const float inv = pow2_int(-st);
        uint4 w = lds128(xb + t * kXbTok + 16 * c);
        uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          const __nv_bfloat162 r2 = __floats2bfloat162_rn(bf16lo(wv[o]) * inv, bf16hi(wv[o]) * inv);
          wv[o] = *reinterpret_cast<const uint32_t*>(&r2);
        }
        *reinterpret_cast<uint4*>(xb + t * kXbTok + 16 * c) = w;
      }
      __syncthreads();
      build_xh(false);
      __syncthreads();
    }
  }
  LING_TRACE(15);

  // ---- phases 1+2: router rows (published at once) and shared gate/up rows
  for (int it = warp; it < n12; it += kWarps) {
    if (it != warp) issue12(it);
    if (!mbar_wait(barA, pha, p.wait_limit_ns, p.err)) { hd.abort = 1; break; }
    pha ^= 1;
    const bool router = it < nr;
    float a0[T], a1[T];
    // tokens [T0, T0 + TG): one pass over the staged row(s); more than 4
    // tokens take two passes, so the accumulators stay those of 4 tokens
    auto dots = [&](auto t0c, auto tgc) {
      constexpr int T0 = decltype(t0c)::value, TG = decltype(tgc)::value;
      float g0[TG], g1[TG], g2[TG], g3[TG], u0_[TG], u1_[TG], u2_[TG], u3_[TG];
#pragma unroll
      for (int t = 0; t < TG; ++t) g0[t] = g1[t] = g2[t] = g3[t] = u0_[t] = u1_[t] = u2_[t] = u3_[t] = 0.f;
#pragma unroll
      for (int m = 0; m < kXChunks / 32; m += 2) {
        const int c0 = lane + 32 * m, c1 = c0 + 32;
        const uint4 w00 = lds128(bufA + 16 * c0), w01 = lds128(bufA + 16 * c1);
        const uint4 w10 = router ? w00 : lds128(bufA + kRowBytes + 16 * c0);
        const uint4 w11 = router ? w01 : lds128(bufA + kRowBytes + 16 * c1);
#pragma unroll
        for (int t = 0; t < TG; ++t) {
          const uint4 xv0 = lds128(xb + (T0 + t) * kXbTok + 16 * c0), xv1 = lds128(xb + (T0 + t) * kXbTok + 16 * c1);
          dot8_bf16_bf16_2(w00, xv0, g0[t], g1[t]);
          dot8_bf16_bf16_2(w01, xv1, g2[t], g3[t]);
          if (!router) {
            dot8_bf16_bf16_2(w10, xv0, u0_[t], u1_[t]);
            dot8_bf16_bf16_2(w11, xv1, u2_[t], u3_[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        a0[T0 + t] = (g0[t] + g1[t]) + (g2[t] + g3[t]);
        a1[T0 + t] = (u0_[t] + u1_[t]) + (u2_[t] + u3_[t]);
      }
    };
    if constexpr (T <= 4) {
      dots(std::integral_constant<int, 0>{}, std::integral_constant<int, T>{});
    } else {
      dots(std::integral_constant<int, 0>{}, std::integral_constant<int, 4>{});
      dots(std::integral_constant<int, 4>{}, std::integral_constant<int, T - 4>{});
    }
#pragma unroll
    for (int t = 0; t < T; ++t) {
      const float g = warp_sum(a0[t]);
      if (router) {
        if (lane == 0)
          p.logits[(size_t)t * E + r0 + it] = g + (p.router_bias ? p.router_bias[r0 + it] * hd.xinv[t] : 0.f);
      } else {
        const float u = warp_sum(a1[t]);
        if (lane == 0) p.h_s[(size_t)t * kI + s0 + it - nr] = silu_mul_scaled(g, u, hd.xscale[t]);
      }
    }
    if (lane == 0 && !(router && withhold)) arrive(p.sync + (router ? 0 : 1));
    __syncwarp();
  }
  LING_TRACE(2);

  LING_TRACE(10);
  // All warps leave phases 1-2 together, so that the selecting warps run
  // alone: with other warps still streaming shared-memory dot products, the
  // shuffle/reduction-bound selection was measured ~3x slower.  The shared
  // rows finish before the router counter completes, so this costs nothing.
  if (tid == 0) hd.epoch = done_ctas / (unsigned long long)ncta;
  __syncthreads();
  // ---- routing: every CTA selects the top-k itself from the published logits
  if (warp < T && !aborted(hd)) {
    float* lg = reinterpret_cast<float*>(bufA);  // scratch: this warp's buffer is idle here
    bool ok = true;
    if (lane == 0) ok = wait_count(p.sync + 0, (hd.epoch + 1) * (unsigned long long)E, p.wait_limit_ns, p.err, &hd.abort);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (warp == 0) LING_TRACE(11);
    if (warp == 0) LING_CLK(0);
    if (ok) {
      // all 16 loads in flight before the first shared store (the compiler
      // cannot tell the two pointers apart and would otherwise serialise them)
      const float* src = p.logits + (size_t)warp * E;
      float v[kMaxExperts / 32];
#pragma unroll
      for (int j = 0; j < kMaxExperts / 32; ++j) v[j] = (lane + 32 * j < E) ? ldcg_f32(src + lane + 32 * j) : 0.f;
#pragma unroll
      for (int j = 0; j < kMaxExperts / 32; ++j)
        if (lane + 32 * j < E) lg[lane + 32 * j] = v[j];
    }
    __syncwarp();
    if (warp == 0) LING_TRACE(12);
    if (warp == 0) { LING_CLK(1); if (lane == 0) g_clk_sink(lg[0] + lg[E - 1]); LING_CLK(2); }
    warp_topk_thresh(lg, E, K, reinterpret_cast<unsigned long long*>(bufA + kMaxExperts * 4), hd.topi[warp],
                     hd.topw[warp], hd.xscale[warp]);
    // the phase-3 bulk copies overwrite this scratch: order these generic
    // writes before them
    fence_async_smem();
    if (warp == 0) LING_CLK(3);

  }
  __syncthreads();
  LING_TRACE(3);
  if (T == 1 && !ep) {
    // one token: the selected experts are already distinct
    if (tid < K) {
      hd.uniq_e[tid] = hd.topi[0][tid];
      hd.uniq_cnt[tid] = 1;
      hd.uniq_pair[tid][0] = tid;
      if (cta == 0) {
        if (p.topk_idx_out) p.topk_idx_out[tid] = hd.topi[0][tid];
        if (p.topk_w_out) p.topk_w_out[tid] = hd.topw[0][tid];
      }
    }
    if (tid == 0) hd.nuniq = K;
  } else if (T <= 4 && warp == 0 && !aborted(hd)) {
    // union of the selected experts held here, in first-occurrence order
    // (t-major), as indices into the local weights
    const int npairs = T * K;
    const int pe = (lane < npairs) ? hd.topi[lane / K][lane % K] : -1 - lane;
    bool first = lane < npairs && (unsigned)(pe - e0) < (unsigned)e_local;
    for (int j = 0; j < npairs; ++j) {
      const int ej = __shfl_sync(0xffffffffu, pe, j);
      if (j < lane && ej == pe) first = false;
    }
    const unsigned fm = __ballot_sync(0xffffffffu, first);
    const int myu = first ? __popc(fm & ((1u << lane) - 1u)) : -1;
    if (first) hd.uniq_e[myu] = pe - e0;
    int cnt = 0;
    for (int j = 0; j < npairs; ++j) {
      const int ej = __shfl_sync(0xffffffffu, pe, j);
      if (first && ej == pe) hd.uniq_pair[myu][cnt++] = j;
    }
    if (first) hd.uniq_cnt[myu] = cnt;
    if (lane == 0) hd.nuniq = __popc(fm);
    if (cta == 0 && lane < npairs) {
      const int t = lane / K, s = lane % K;
      if (p.topk_idx_out) p.topk_idx_out[lane] = hd.topi[t][s];
      if (p.topk_w_out) p.topk_w_out[lane] = hd.topw[t][s];
    }
  } else if (T > 4 && warp == 0 && !aborted(hd)) {
    // the same union over up to 64 pairs (lane l holds pairs l and l + 32),
    // then the h rows of phase 4: experts in union order fill passes of at
    // most kHfCapBig pairs
    const int npairs = T * K;
    int pe[2];
    bool first[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int j = lane + 32 * hh;
      pe[hh] = j < npairs ? hd.topi[j / K][j % K] : -1 - j;
      first[hh] = j < npairs && (unsigned)(pe[hh] - e0) < (unsigned)e_local;
    }
    for (int j = 0; j < npairs; ++j) {
      const int ej = __shfl_sync(0xffffffffu, j < 32 ? pe[0] : pe[1], j & 31);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        if (j < lane + 32 * hh && ej == pe[hh]) first[hh] = false;
    }
    const unsigned fm0 = __ballot_sync(0xffffffffu, first[0]), fm1 = __ballot_sync(0xffffffffu, first[1]);
    const unsigned below = (1u << lane) - 1u;
    const int myu[2] = {first[0] ? __popc(fm0 & below) : -1, first[1] ? __popc(fm0) + __popc(fm1 & below) : -1};
    int cnt[2] = {0, 0};
    for (int j = 0; j < npairs; ++j) {
      const int ej = __shfl_sync(0xffffffffu, j < 32 ? pe[0] : pe[1], j & 31);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        if (first[hh] && ej == pe[hh]) hd.uniq_pair[myu[hh]][cnt[hh]++] = j;
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
      if (first[hh]) {
        hd.uniq_e[myu[hh]] = pe[hh] - e0;
        hd.uniq_cnt[myu[hh]] = cnt[hh];
      }
    const int nu = __popc(fm0) + __popc(fm1);
    if (lane == 0) hd.nuniq = nu;
    __syncwarp();
    if (lane == 0) {
      int pass = 0, rows = 0;
      hd.u_split = nu;
      for (int u = 0; u < nu; ++u) {
        const int c = hd.uniq_cnt[u];
        if (pass == 0 && rows + c > kHfCapBig) {
          hd.nslot[0] = rows;
          hd.u_split = u;
          pass = 1;
          rows = 0;
        }
        hd.uniq_slot[u] = rows;
        for (int g = 0; g < c; ++g) hd.slot_pair[pass][rows + g] = hd.uniq_pair[u][g];
        rows += c;
      }
      hd.nslot[pass] = rows;
      if (pass == 0) hd.nslot[1] = 0;
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int j = lane + 32 * hh;
      if (cta == 0 && j < npairs) {
        if (p.topk_idx_out) p.topk_idx_out[j] = hd.topi[j / K][j % K];
        if (p.topk_w_out) p.topk_w_out[j] = hd.topw[j / K][j % K];
      }
    }
  }
  __syncthreads();
  const int U = aborted(hd) ? 0 : hd.nuniq;

  // ---- phase 3: routed gate/up, whole units [u0, u1) of 8 intermediate rows
  // (gate and up).  Warp pair p takes units u0 + p, u0 + p + kPairs, ...; warp
  // 2p computes the first K half, warp 2p+1 the second, each copied in four
  // pieces (the half's scales travel with piece 0).  Per 16-K block one
  // fragment word per lane is dequantised to the exact codes q (LOP3 + HSUB2)
  // and fed to one m16n8k16 MMA whose columns are the expert's tokens; per
  // 32-K group the fp32 result is scaled by the group's bf16 scale.
  const int n3 = U * kGuUnits;
  const int u0 = (int)((long long)cta * n3 / ncta), u1 = (int)((long long)(cta + 1) * n3 / ncta);
  const int pair = warp >> 1, half = warp & 1;
  auto issue3 = [&](int unit) {
    if (lane == 0) {
      const int u = unit / kGuUnits, b = unit - u * kGuUnits;
      const uint8_t* src = p.gu + ((size_t)hd.uniq_e[u] * kGuUnits + b) * kGuUnitBytes;
      mbar_arrive_expect_tx(barA, kGuPiece + kGuHalfScales);
      if (T > 4) {  // read once: evict first (see the down-unit prefetch)
        const uint64_t once = l2_evict_first_policy();
        bulk_g2s_hint(bufA + kGuHalfCodes, src + kGuScaleOff + half * kGuHalfScales, kGuHalfScales, barA, once);
        bulk_g2s_hint(bufA, src + half * kGuHalfCodes, kGuPiece, barA, once);
        for (int pc = 1; pc < 4; ++pc) {
          mbar_arrive_expect_tx(&hd.mbar[warp][pc], kGuPiece);
          bulk_g2s_hint(bufA + pc * kGuPiece, src + half * kGuHalfCodes + pc * kGuPiece, kGuPiece,
                        &hd.mbar[warp][pc], once);
        }
      } else {
        bulk_g2s(bufA + kGuHalfCodes, src + kGuScaleOff + half * kGuHalfScales, kGuHalfScales, barA);
        bulk_g2s(bufA, src + half * kGuHalfCodes, kGuPiece, barA);
        for (int pc = 1; pc < 4; ++pc) {
          mbar_arrive_expect_tx(&hd.mbar[warp][pc], kGuPiece);
          bulk_g2s(bufA + pc * kGuPiece, src + half * kGuHalfCodes + pc * kGuPiece, kGuPiece, &hd.mbar[warp][pc]);
        }
      }
    }
  };
  const bool first_issued = u0 + pair < u1 && __shfl_sync(0xffffffffu, !aborted(hd), 0);  // one view per warp
  if (first_issued) issue3(u0 + pair);
  // routed down units of this CTA (contiguous per expert) into L2 as soon as
  // the routing is known.  Above 4 tokens the union's weights (~200 MB at 8
  // tokens) outgrow L2: the gate/up units, read once, stream with an
  // evict-first hint and these with evict-last, so that they are still there
  // at phase 4 (without the hints: 1.24x the algorithmic DRAM reads at 8
  // tokens).
  if (!use_d && warp == kWarps - 1 && nblk > 0) {
    const uint64_t keep = T > 4 ? l2_evict_last_policy() : 0;
    for (int u = lane; u < U; u += 32) {
      const uint8_t* src = p.dn + ((size_t)hd.uniq_e[u] * kDnUnits + b0) * kDnUnitBytes;
      if (T > 4) prefetch_l2_bulk_hint(src, (uint32_t)nblk * kDnUnitBytes, keep);
      else prefetch_l2_bulk(src, (uint32_t)nblk * kDnUnitBytes);
    }
  }

  {
    float* comb = reinterpret_cast<float*>(body + PL::comb) + (size_t)pair * (2 * 32 * 4);
    const int n = lane >> 2, m = lane & 3;  // B column (token of the expert) / lane class
    int par = 0;
    bool issued = first_issued;
    for (int unit = u0 + pair; unit < u1; unit += kPairs, par ^= 1) {
      if (unit != u0 + pair) {
        issued = __shfl_sync(0xffffffffu, !aborted(hd), 0);
        if (issued) issue3(unit);
      }
      const int u = unit / kGuUnits, b = unit - u * kGuUnits;
      const int cnt = hd.uniq_cnt[u];
      const bool bval = n < cnt;
      // a column without a token reads token 0's x (its results are dropped),
      // so that the loads below need no branch
      const unsigned char* xrow = xf + (hd.uniq_pair[u][bval ? n : 0] / K) * kXfTok + m * 32 +
                                  half * (kGuChunks / 2) * 128;
      float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
      bool ok = issued && mbar_wait_warp(barA, pha, p.wait_limit_ns, p.err);
      const uint32_t pa0 = pha;
      int pc_next = ok ? 1 : 0;  // first piece not yet seen complete
      if (issued) pha ^= 1;
      if (warp == 0 && unit == u0) { LING_TRACE(13); LING_CLK(6); }
#pragma unroll 1
      for (int pc = 0; pc < 4 && ok; ++pc) {
        if (pc > 0) {
          ok = mbar_wait_warp(&hd.mbar[warp][pc], phq, p.wait_limit_ns, p.err);
          if (!ok) break;
          pc_next = pc + 1;
          if (warp == 0 && unit == u0) LING_CLK(6 + pc);
        }
#pragma unroll
        for (int jj = 0; jj < kGuChunks / 8; ++jj) {
          const int jl = pc * (kGuChunks / 8) + jj;  // chunk within the half
          const uint4 wv = lds128(bufA + jl * 512 + 16 * lane);
          const uint4 xa = lds128(xrow + jl * 128);
          const uint4 xc = lds128(xrow + jl * 128 + 16);
          const uint32_t s01 = *reinterpret_cast<const uint32_t*>(bufA + kGuHalfCodes + (2 * jl) * 32 + 4 * n);
          const uint32_t s23 = *reinterpret_cast<const uint32_t*>(bufA + kGuHalfCodes + (2 * jl + 1) * 32 + 4 * n);
          const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
          const uint32_t bx[8] = {xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w};
          float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t a0, a1, a2, a3;
            if constexpr (C == kCodecMxfp4) {
              a0 = deq_e2m1<0>(wd[w]);
              a2 = deq_e2m1<4>(wd[w]);
              a1 = deq_e2m1<8>(wd[w]);
              a3 = deq_e2m1<12>(wd[w]);
            } else {
              a0 = deq_q_even(wd[w]);
              a2 = deq_q_odd16(wd[w]);
              a1 = deq_q_even(wd[w] >> 8);
              a3 = deq_q_odd16(wd[w] >> 8);
            }
            if (w & 1) {
              mma_16816(d0, d1, d2, d3, a0, a1, a2, a3, bx[2 * w], bx[2 * w + 1], d0, d1, d2, d3);
              const uint32_t sw = (w == 1) ? s01 : s23;
              const float sg = bf16lo(sw), su = bf16hi(sw);
              acc0 = fmaf(sg, d0, acc0);
              acc1 = fmaf(sg, d1, acc1);
              acc2 = fmaf(su, d2, acc2);
              acc3 = fmaf(su, d3, acc3);
            } else {
              mma_16816(d0, d1, d2, d3, a0, a1, a2, a3, bx[2 * w], bx[2 * w + 1], 0.f, 0.f, 0.f, 0.f);
            }
          }
        }
      }
      if (issued) phq ^= 1;
      if (!ok && issued) {
        // a wait ran out: the unit's pieces still in flight land (bounded
        // waits) before the buffer is reused or the CTA exits
        hd.abort = 1;
        if (lane == 0)
          for (int pc = pc_next; pc < 4; ++pc)
            mbar_wait(pc == 0 ? barA : &hd.mbar[warp][pc], pc == 0 ? pa0 : (phq ^ 1u), p.wait_limit_ns, p.err);
        __syncwarp();
      }
      // combine the two K halves: the second half's partials go through
      // shared memory (double-buffered by unit parity, one barrier per unit)
      float* cb = comb + par * (32 * 4) + lane * 4;
      if (half == 1) *reinterpret_cast<float4*>(cb) = make_float4(acc0, acc1, acc2, acc3);
      asm volatile("bar.sync %0, %1;" :: "r"(1 + pair), "r"(64) : "memory");
      if (half == 0 && !aborted(hd)) {
        const float4 o = *reinterpret_cast<const float4*>(cb);
        acc0 += o.x;
        acc1 += o.y;
        acc2 += o.z;
        acc3 += o.w;
        const int i = 8 * b + n;  // intermediate row of this lane
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int col = 2 * m + cc;  // the expert's token column
          if (col < cnt) {
            const int pr = hd.uniq_pair[u][col];
            p.h_pair[(size_t)pr * kI + i] = silu_mul_scaled(cc ? acc1 : acc0, cc ? acc3 : acc2, hd.xscale[pr / K]);
          }
        }
      }
      if (warp == 0 && unit == u0) { LING_TRACE(14); LING_CLK(10); }
    }
  }
  __syncthreads();
  if (tid == 0) arrive(p.sync + 2);  // this CTA's h values are published
  if (use_d && warp == kWarps - 1 && U > 0 && !aborted(hd)) {
    // T = 1: this CTA's routed down units, one contiguous copy per expert,
    // requested now so that they stream in during the h exchange (during the
    // gate/up phase they would only share its bandwidth).  Region D overlays
    // the phase 1-3 buffers, read until the barrier above.
    fence_async_smem();
    const uint32_t per = (uint32_t)nblk * kDnUnitBytes;
    if (lane == 0) mbar_arrive_expect_tx(&hd.dbar, per * (uint32_t)U);
    __syncwarp();
    if (lane < U)
      bulk_g2s(body + PL::dn + (size_t)lane * per,
               p.dn + ((size_t)hd.uniq_e[lane] * kDnUnits + b0) * kDnUnitBytes, per, &hd.dbar);
    if (lane == 0) hd.dcopies = 1;
  }
  LING_TRACE(5);

  // ---- phase 4: down projections and the output
  // Region A is free now; start this warp's first phase-4 copy before waiting.
  constexpr int kDnBatch = dn_batch<T>();
  const int npairs = T * K;
  const int nitems = nblk * U;
  // above 4 tokens the items of the first pass's experts come first (pass-major,
  // then row-block, then expert); a copy batch is one item there
  const int npass = (T > 4 && hd.nslot[1] > 0) ? 2 : 1;  // the same value in every thread
  const int U1 = npass == 2 ? hd.u_split : U, n1 = nblk * U1;
  auto item_bu = [&](int it, int& blk, int& u) {
    if (it < n1) {
      blk = it / U1;
      u = it - blk * U1;
    } else {
      const int i2 = it - n1, U2 = U - U1;
      blk = i2 / U2;
      u = U1 + (i2 - blk * U2);
    }
  };
  const int nbatch = use_d ? 0 : (nitems + kDnBatch - 1) / kDnBatch;
  const int nmine_r = warp < nbatch ? (nbatch - warp + kWarps - 1) / kWarps : 0;
  const int sh_first = kWarps - 1 - warp;  // shared down: half-blocks of 4 rows
  const int nsub = 2 * nblk;
  const int nmine_s = (sh_on && !aborted(hd) && sh_first < nsub) ? (nsub - sh_first + kWarps - 1) / kWarps : 0;
  auto issue4 = [&](int s) {
    if (lane == 0) {
      if (s < nmine_r) {
        const int bi = warp + s * kWarps;
        const int it0 = bi * kDnBatch, n = min(kDnBatch, nitems - it0);
        mbar_arrive_expect_tx(barA, (uint32_t)n * kDnUnitBytes);
        for (int bI = 0; bI < n; ++bI) {
          int blk, u;
          item_bu(it0 + bI, blk, u);
          bulk_g2s(bufB + bI * kDnUnitBytes,
                   p.dn + ((size_t)hd.uniq_e[u] * kDnUnits + b0 + blk) * kDnUnitBytes, kDnUnitBytes, barA);
        }
      } else {
        const int sb = sh_first + (s - nmine_r) * kWarps;
        mbar_arrive_expect_tx(barA, kShDnBytes);
        bulk_g2s(bufB, p.sh_down + ((size_t)2 * b0 + sb) * 4 * kI, kShDnBytes, barA);
      }
    }
  };
  const int nseq = nmine_r + nmine_s;
  fence_async_smem();  // region B overlays buffers read through the generic proxy
  if (nseq > 0) issue4(0);

  unsigned char* hfb = body + PL::hf;
  float* hsm = reinterpret_cast<float*>(body + PL::hs);
  float* part = reinterpret_cast<float*>(body + PL::part);
  if (tid == 0 && !aborted(hd)) {
    const unsigned long long ep1 = hd.epoch + 1;
    if (!sh_on || wait_count(p.sync + 1, ep1 * (unsigned long long)kI, p.wait_limit_ns, p.err, &hd.abort))
      wait_count(p.sync + 2, ep1 * (unsigned long long)ncta, p.wait_limit_ns, p.err, &hd.abort);
  }
  __syncthreads();
  // routed h as fp16 hi + lo A fragments (h row r: pair r up to 4 tokens;
  // above, row r of the pass, pair slot_pair[pass][r]) and, with the first
  // pass, the shared h per token; in batches whose loads are all in flight
  // before the first shared store
  auto stage = [&](int pass) {
    constexpr int kB = 5;
    const int nrow = T <= 4 ? npairs : hd.nslot[pass];
    const int nh = nrow * (kI / 4), nall = nh + (pass == 0 && sh_on ? T * (kI / 4) : 0);
    for (int v0 = tid; v0 < nall; v0 += kB * kDecodeThreads) {
      float4 hv[kB];
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int v = v0 + b * kDecodeThreads;
        if (v < nh) {
          const int row = v / (kI / 4);
          const int pr = T <= 4 ? row : hd.slot_pair[pass][row];
          hv[b] = ldcg_f4(reinterpret_cast<const float4*>(p.h_pair) + (size_t)pr * (kI / 4) + (v - row * (kI / 4)));
        } else if (v < nall) {
          hv[b] = ldcg_f4(reinterpret_cast<const float4*>(p.h_s) + (v - nh));
        }
      }
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int v = v0 + b * kDecodeThreads;
        if (v < nh) {
          // h * 2^-8 as fp16 hi + lo in MMA A-fragment order
          const int row = v / (kI / 4), k = 4 * (v - row * (kI / 4));
          unsigned char* dst = hfb + (size_t)row * kHfStride + hf_off(k);
          *reinterpret_cast<uint2*>(dst) = h_split2(hv[b].x, hv[b].y);
          *reinterpret_cast<uint2*>(dst + 16) = h_split2(hv[b].z, hv[b].w);
        } else if (v < nall) {
          const int t = (v - nh) / (kI / 4), c4 = (v - nh) - t * (kI / 4), c = c4 >> 1, pl = c4 & 1;
          *reinterpret_cast<float4*>(hsm + (size_t)t * kHsTok + pl * kHsPlane + 4 * c) = hv[b];
        }
      }
    }
  };
  if (!aborted(hd)) stage(0);
  __syncthreads();
  LING_TRACE(6);
  // one routed down unit (8 output rows of expert slot u, row-block blk) on
  // the tensor cores: per pair, the partial sums times the routing weight go
  // to part[]
  auto down_item = [&](const unsigned char* base, int blk, int u) {
    const int g = lane >> 2, c = lane & 3;
    const bool act = g < hd.uniq_cnt[u];
    const int pr = hd.uniq_pair[u][act ? g : 0];
    const int hrow = T <= 4 ? pr : hd.uniq_slot[u] + (act ? g : 0);
    float v0, v1;
    dn_unit_mma<C>(base, hfb + (size_t)hrow * kHfStride + 16 * c, lane, v0, v1);
    if (act) {
      const float f = (float)(1 << kHShift) * hd.topw[pr / K][pr % K];
      *reinterpret_cast<float2*>(part + ((size_t)blk * (PL::P + T) + pr) * 8 + 2 * c) = make_float2(v0 * f, v1 * f);
    }
  };
  if (use_d && !aborted(hd) && warp < nitems) {
    // T = 1: routed units straight from the dedicated region
    if (!mbar_wait(&hd.dbar, 0, p.wait_limit_ns, p.err)) {
      hd.abort = 1;
    } else {
      LING_TRACE(7);
      if (warp == 0) LING_CLK(4);
      for (int it = warp; it < nitems; it += kWarps) {
        const int blk = it / U, u = it - blk * U;
        down_item(body + PL::dn + ((size_t)u * nblk + blk) * kDnUnitBytes, blk, u);
        if (warp == 0 && it == 0) LING_CLK(5);
      }
      if (warp == 0) { LING_CLK(15); LING_TRACE(4); }
    }
  }
  {
    const int r = lane & 3, q = lane >> 2;
    const bool run = !aborted(hd);
    int issued = nseq > 0 ? 1 : 0;  // copies requested: item sequence 0 went out above
    // one step of this warp's sequence; false when its wait ran out
    auto step = [&](int s) -> bool {
      if (s >= issued) {
        issue4(s);
        issued = s + 1;
      }
      if (!mbar_wait(barA, pha, p.wait_limit_ns, p.err)) {
        hd.abort = 1;
        return false;
      }
      pha ^= 1;
      if (!run) return true;
      if (s < nmine_r) {
        const int it0 = (warp + s * kWarps) * kDnBatch, n = min(kDnBatch, nitems - it0);
#pragma unroll 1
        for (int bI = 0; bI < n; ++bI) {
          int blk, u;
          item_bu(it0 + bI, blk, u);
          down_item(bufB + bI * kDnUnitBytes, blk, u);
        }
      } else {
        const int sb = sh_first + (s - nmine_r) * kWarps;
        float acc[T];
        {
          float a0[T], a1[T], a2[T], a3[T];
#pragma unroll
          for (int t = 0; t < T; ++t) a0[t] = a1[t] = a2[t] = a3[t] = 0.f;
#pragma unroll 2
          for (int m = 0; m < kI / 64; m += 2) {
            const int c0 = q + 8 * m, c1 = c0 + 8;
            const uint4 w0 = lds128(bufB + r * (kI * 2) + 16 * c0);
            const uint4 w1 = lds128(bufB + r * (kI * 2) + 16 * c1);
#pragma unroll
            for (int t = 0; t < T; ++t) {
              const float* ht = hsm + (size_t)t * kHsTok;
              dot8_bf16_2(w0, ldsf4(ht + 4 * c0), ldsf4(ht + kHsPlane + 4 * c0), a0[t], a1[t]);
              dot8_bf16_2(w1, ldsf4(ht + 4 * c1), ldsf4(ht + kHsPlane + 4 * c1), a2[t], a3[t]);
            }
          }
#pragma unroll
          for (int t = 0; t < T; ++t) acc[t] = (a0[t] + a1[t]) + (a2[t] + a3[t]);
        }
#pragma unroll
        for (int t = 0; t < T; ++t) {
          float v = acc[t];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          if (q == 0) part[((size_t)(sb >> 1) * (PL::P + T) + PL::P + t) * 8 + 4 * (sb & 1) + r] = v;
        }
      }
      __syncwarp();
      return true;
    };
    // this warp's items of the first pass (with one pass: its whole sequence)
    const int s_p0 = npass == 2 ? min(nmine_r, n1 > warp ? (n1 - warp + kWarps - 1) / kWarps : 0) : nseq;
    int s = 0;
    for (; s < s_p0; ++s)
      if (!step(s)) {
        s = nseq;
        break;
      }
    if (npass == 2) {
      // the second pass's h rows replace the first's once every warp is done
      // with them; this warp's next copy is requested before the barrier
      if (s < nseq && s >= issued) {
        issue4(s);
        issued = s + 1;
      }
      __syncthreads();
      if (!aborted(hd)) stage(1);
      __syncthreads();
    }
    for (; s < nseq; ++s)
      if (!step(s)) break;
  }
  __syncthreads();
  LING_TRACE(8);
  if (!aborted(hd)) {
    // fixed-order sum: routed slots 0..k-1 (those computed here), then the
    // shared expert (if computed here)
    for (int v = tid; v < nblk * T * kDnUnitRows; v += kDecodeThreads) {
      const int blk = v / (T * kDnUnitRows), rem = v - blk * T * kDnUnitRows, t = rem >> 3, r = rem & 7;
      const float* pb = part + (size_t)blk * (PL::P + T) * 8;
      float v8[kMaxTopK];  // all loads in flight first, then the sum in slot order
#pragma unroll
      for (int sl = 0; sl < kMaxTopK; ++sl)
        v8[sl] = sl < K && (!ep || (unsigned)(hd.topi[t][sl] - e0) < (unsigned)e_local) ? pb[(t * K + sl) * 8 + r]
                                                                                        : 0.f;
      const float vs = sh_on ? pb[(PL::P + t) * 8 + r] : 0.f;
      float s = 0.f;
#pragma unroll
      for (int sl = 0; sl < kMaxTopK; ++sl)
        if (sl < K) s += v8[sl];
      s += vs;
      const float st = hd.xscale[t];  // back from x / s_t: the output scales as s_t^2
      const size_t o = (size_t)t * kH + kDnUnitRows * (b0 + blk) + r;
      if (EP && p.out_f32) p.out_f32[o] = s * st * st;
      else p.out[o] = __float2bfloat16_rn(s * st * st);
    }
  }
  // every CTA (aborted or not) counts itself out: the next launch's index
  __syncthreads();
  // no copy left in flight (without an abort the phase-4 warps waited for them)
  if (tid == 0 && hd.dcopies && aborted(hd)) mbar_wait(&hd.dbar, 0, p.wait_limit_ns, p.err);
  if (tid == 0) atomicAdd(p.sync + 3, 1ull);  // read by later launches only: no fence needed
  LING_TRACE(9);
}

#ifdef LING_MOE_TRACE
extern "C" int ling_moe_clk_read(long long* host) { return (int)cudaMemcpyFromSymbol(host, g_clk, sizeof(g_clk)); }
extern "C" int ling_moe_trace_read(unsigned long long* host, int nctas) {
  return (int)cudaMemcpyFromSymbol(host, g_trace, (size_t)nctas * 16 * sizeof(unsigned long long));
}
#endif

template <int T, int C, bool EP>
static cudaError_t launch_t(const DecodeParams& p, int nctas, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = Plan<T>::bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe_decode_kernel<T, C, EP>, p);
}

template <int C, bool EP>
static cudaError_t launch_c(const DecodeParams& p, int nctas, cudaStream_t stream) {
  switch (p.T) {
    case 1: return launch_t<1, C, EP>(p, nctas, stream);
    case 2: return launch_t<2, C, EP>(p, nctas, stream);
    case 3: return launch_t<3, C, EP>(p, nctas, stream);
    case 4: return launch_t<4, C, EP>(p, nctas, stream);
    case 5: return launch_t<5, C, EP>(p, nctas, stream);
    case 6: return launch_t<6, C, EP>(p, nctas, stream);
    case 7: return launch_t<7, C, EP>(p, nctas, stream);
    case 8: return launch_t<8, C, EP>(p, nctas, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode(const DecodeParams& p, int nctas, cudaStream_t stream) {
  const bool ep = p.e0 != 0 || p.e_local != p.E || !p.shared_on || p.out_f32 != nullptr;
  if (p.codec == kCodecMxfp4)
    return ep ? launch_c<kCodecMxfp4, true>(p, nctas, stream) : launch_c<kCodecMxfp4, false>(p, nctas, stream);
  if (p.codec == kCodecInt4)
    return ep ? launch_c<kCodecInt4, true>(p, nctas, stream) : launch_c<kCodecInt4, false>(p, nctas, stream);
  return cudaErrorInvalidValue;
}

template <int T, int C, bool EP>
static cudaError_t set_smem() {
  return cudaFuncSetAttribute(moe_decode_kernel<T, C, EP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)Plan<T>::bytes);
}

template <int T>
static cudaError_t setup_t() {
  cudaError_t e;
  if ((e = set_smem<T, kCodecInt4, false>()) != cudaSuccess) return e;
  if ((e = set_smem<T, kCodecInt4, true>()) != cudaSuccess) return e;
  if ((e = set_smem<T, kCodecMxfp4, false>()) != cudaSuccess) return e;
  return set_smem<T, kCodecMxfp4, true>();
}

cudaError_t setup_decode() {
  cudaError_t e;
  if ((e = setup_t<1>()) != cudaSuccess) return e;
  if ((e = setup_t<2>()) != cudaSuccess) return e;
  if ((e = setup_t<3>()) != cudaSuccess) return e;
  if ((e = setup_t<4>()) != cudaSuccess) return e;
  if ((e = setup_t<5>()) != cudaSuccess) return e;
  if ((e = setup_t<6>()) != cudaSuccess) return e;
  if ((e = setup_t<7>()) != cudaSuccess) return e;
  return setup_t<8>();
}

int decode_max_ctas_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, moe_decode_kernel<8, kCodecInt4, true>, kDecodeThreads,
                                                    Plan<8>::bytes) != cudaSuccess)
    return 0;
  return n;
}

}  // namespace lingmoe
