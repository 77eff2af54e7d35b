// Token-grouped path (T > kMaxDecodeT): prefill chunks and large verify
// batches of the W4 g32 MoE layer.
//
//   route        logits[t, e] = x_t . Wr_e (+ b_e), bf16 products summed in
//                fp32 on the tensor cores (mma.sync), tiles of 32 tokens x 64
//                experts
//   top-k        per token (ties to the lower index) and the renormalised
//                softmax weights; pairs per expert counted on the fly
//   plan         exclusive scan of the counts, tile lists for both GEMMs
//                (N-tiles of <= 128 positions, the costly ones first)
//   scatter      each pair gets a position in its expert's run; x is written
//                in fp16 by position (8 routed copies + 1 shared row per token)
//   gate/up      tcgen05 tiles over the routed experts with more than
//                kGvMaxTok tokens and the shared expert; a GEMV kernel
//                (mma.sync on streamed weights) for the experts with fewer
//   down         the same split: y[position] = w * Wd h[position]
//   combine      out[t] = sum_slot y[position of (t, slot)] + y[shared row t],
//                one bf16 rounding, slots summed in a fixed order
//
// Chunked prefill feeds this path (vLLM recipe page "inclusionAI/Ling-3.0-flash",
// "Launching the Server": --enable-chunked-prefill); a verify window of
// several tokens touches the union of their experts (bpdata article, section
// "Optimalizacio 3": four tokens can activate up to 32 experts).
#include <algorithm>

#include "common.cuh"
#include "grouped.h"
#include "grouped_gemv.h"

namespace lingmoe {

constexpr int kPlanThreads = 1024;
constexpr int kRowThreads = kH / 8;  // 320: one thread per 8 columns of a row

const char* grouped_describe() {
  return "router GEMM (bf16 mma.sync, fp32 sums) + top-k + counting scatter by expert + tcgen05 grouped GEMMs "
         "(M=256 weight rows x N<=128 positions; routed int4 dequantised to exact fp16 in shared memory, "
         "shared expert as fp16 tiles via TMA; activations via TMA; fp32 accumulators in double-buffered TMEM) "
         "+ fixed-order combine";
}

cudaError_t grouped_alloc(GroupedWorkspace* ws, int E, int k, int max_T, const AllocFn& alloc) {
  ws->max_T = max_T;
  const size_t P = (size_t)max_T * k;
  ws->rows = (size_t)max_T * (k + 1);
  const size_t nt = tc_max_ntiles((int)P, max_T, E);
  cudaError_t e;
  struct A { void** p; size_t n; } plan[] = {
      {(void**)&ws->logits, (size_t)max_T * E * sizeof(float)},
      {(void**)&ws->topk_idx, P * sizeof(int32_t)},
      {(void**)&ws->topk_w, P * sizeof(float)},
      {(void**)&ws->cnt, (size_t)E * sizeof(int32_t)},
      {(void**)&ws->fill, (size_t)E * sizeof(int32_t)},
      {(void**)&ws->off, (size_t)(E + 1) * sizeof(int32_t)},
      {(void**)&ws->perm, P * sizeof(int32_t)},
      {(void**)&ws->inv, P * sizeof(int32_t)},
      {(void**)&ws->xscale, (size_t)max_T * sizeof(float)},
      {(void**)&ws->xg, ws->rows * kH * sizeof(__half)},
      {(void**)&ws->h16, ws->rows * 2 * kI * sizeof(__half)},
      {(void**)&ws->y, ws->rows * kH * sizeof(float)},
      {(void**)&ws->shgu16, (size_t)2 * kI * kH * sizeof(__half)},
      {(void**)&ws->shdn16, (size_t)kH * kI * sizeof(__half)},
      {(void**)&ws->sh_scale, 4 * sizeof(float)},
      {(void**)&ws->amax, 4 * sizeof(unsigned int)},
      {(void**)&ws->gu_tiles, nt * kTcMTilesGu * sizeof(int4)},
      {(void**)&ws->dn_tiles, nt * kTcMTilesDn * sizeof(int4)},
      {(void**)&ws->ntiles, 4 * sizeof(int32_t)},
      {(void**)&ws->small, (size_t)E * sizeof(int4)},
      {(void**)&ws->nsmall, 4 * sizeof(int32_t)},
  };
  for (auto& a : plan)
    if ((e = alloc(a.p, a.n)) != cudaSuccess) return e;
  return cudaSuccess;
}

cudaError_t grouped_prepare(GroupedWorkspace* ws, int E, const __nv_bfloat16* sh_gate, const __nv_bfloat16* sh_up,
                            const __nv_bfloat16* sh_down, cudaStream_t stream) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(ws->cnt, 0, (size_t)E * sizeof(int32_t), stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(ws->fill, 0, (size_t)E * sizeof(int32_t), stream)) != cudaSuccess) return e;
  // rows of the B operands that no call writes still reach the MMA as padding
  // columns (whose results are discarded); keep them finite
  if ((e = cudaMemsetAsync(ws->xg, 0, ws->rows * kH * sizeof(__half), stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(ws->h16, 0, ws->rows * 2 * kI * sizeof(__half), stream)) != cudaSuccess) return e;
  // (no shared expert on this handle: its fp16 copies are never read)
  if (sh_gate && (e = launch_tc_prep_shared(sh_gate, sh_up, sh_down, ws->shgu16, ws->shdn16, ws->sh_scale, ws->amax,
                                            stream)) != cudaSuccess)
    return e;
  return tc_encode_maps(&ws->maps, ws->xg, ws->h16, (int)ws->rows, ws->shgu16, ws->shdn16);
}

// ---------------------------------------------------------------- route
// logits[t, e] = x_t . Wr_e (+ b_e): the bf16 x bf16 products are exact in
// fp32 and are summed in fp32 by mma.sync m16n8k16 (bf16 inputs).  CTA tile:
// 32 tokens x 64 experts, 4 warps of 16 tokens x 32 experts; K streams
// through shared memory in stages of 128 (cp.async, double-buffered), the
// fragments come from ldmatrix.  Rows past T or E repeat the last valid row;
// their results are not stored.
constexpr int kRmTok = 32, kRmExp = 64, kRmK = 128, kRmThreads = 128;
constexpr int kRmRow = kRmK * 2 + 16;                    // 272 B: 8 rows hit 8 distinct 16-byte bank groups
constexpr int kRmStage = (kRmTok + kRmExp) * kRmRow;     // 26112
constexpr size_t kRmSmem = 2 * (size_t)kRmStage;
static_assert(kH % kRmK == 0, "K stages tile the hidden size");

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kRmThreads) grp_route_kernel(GroupedParams p, float* logits) {
  extern __shared__ __align__(128) unsigned char rsm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kRmTok, e0 = blockIdx.y * kRmExp;
  const int wm = warp & 1, wn = warp >> 1;  // 16-token half, 32-expert half
  auto load_stage = [&](int kc, int buf) {
    unsigned char* base = rsm + buf * kRmStage;
    for (int v = tid; v < (kRmTok + kRmExp) * (kRmK / 8); v += kRmThreads) {
      const int row = v >> 4, pc = v & 15;
      const __nv_bfloat16* src = row < kRmTok ? p.x + (size_t)min(t0 + row, p.T - 1) * kH
                                              : p.router_w + (size_t)min(e0 + row - kRmTok, p.E - 1) * kH;
      cp_async16(smem_u32(base + row * kRmRow + pc * 16), src + kc * kRmK + pc * 8);
    }
    cp_async_commit();
  };
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  constexpr int NKC = kH / kRmK;
  load_stage(0, 0);
#pragma unroll 1
  for (int kc = 0; kc < NKC; ++kc) {
    if (kc + 1 < NKC) {
      load_stage(kc + 1, (kc + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t base = smem_u32(rsm + (kc & 1) * kRmStage);
    // A (x rows): lanes 0-15 address rows 0-15 at k 0, lanes 16-31 the same rows at k 8
    const uint32_t arow = base + (wm * 16 + (lane & 15)) * kRmRow + (lane >> 4) * 16;
    // B (router rows, K contiguous): matrix lane/8 = (expert octet lane/16, k half (lane/8)%2)
    const uint32_t brow = base + (kRmTok + wn * 32 + (lane >> 4) * 8 + (lane & 7)) * kRmRow + ((lane >> 3) & 1) * 16;
#pragma unroll
    for (int ks = 0; ks < kRmK / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(arow + ks * 32, a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(brow + np * 16 * kRmRow + ks * 32, b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();  // the buffer is refilled two stages on
  }
  // accumulator (token g / g + 8, experts 2c, 2c + 1 of each 8-expert tile)
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const int e = e0 + wn * 32 + nt * 8 + 2 * c;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int t = t0 + wm * 16 + g + 8 * hh;
      if (t >= p.T) continue;
#pragma unroll
      for (int q = 0; q < 2; ++q)
        if (e + q < p.E)
          logits[(size_t)t * p.E + e + q] = acc[nt][2 * hh + q] + (p.router_bias ? p.router_bias[e + q] : 0.f);
    }
  }
}

// One warp per token: top-k of its logits, the renormalised weights, and
// one count per selected expert.  The router GEMM sums bf16 products in fp32
// on the tensor cores, which is exact to fp32 rounding while every product
// that matters is a normal fp32 number and no sum overflows: for a token whose
// largest |x| lies in [2^-60, 2^101) (with |Wr| < 2^20 per row sum).  A token
// outside that window, or with a logit that is not finite, has its logits
// recomputed here from x / s_t (the decode path's power-of-two token scale)
// with fp32 FMAs: keys l / s_t + b / s_t, weights exp(s_t (l - l_0)).
__global__ void __launch_bounds__(256) grp_topk_kernel(GroupedParams p, const float* logits, int32_t* ti,
                                                       float* tw, int32_t* cnt) {
  __shared__ float lg[8][kMaxExperts];
  __shared__ int s_idx[8][kMaxTopK];
  __shared__ float s_w[8][kMaxTopK];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + warp;
  if (t >= p.T) return;
  bool bad = false;
  for (int e = lane; e < p.E; e += 32) {
    const float v = logits[(size_t)t * p.E + e];
    bad |= !isfinite(v);
    lg[warp][e] = v;
  }
  const uint4* xr = reinterpret_cast<const uint4*>(p.x + (size_t)t * kH);
  uint32_t mag = 0u;
  for (int c = lane; c < kH / 8; c += 32) {
    const uint4 w = xr[c];
    mag = __vmaxu2(mag, __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu),
                                 __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu)));  // per half
  }
  mag = __reduce_max_sync(0xffffffffu, max(mag & 0xFFFFu, mag >> 16));
  const int ex = (int)(mag >> 7) - 127;
  bad |= mag != 0u && (ex < -60 || ex > 100);
  float wscale = 1.0f;
  if (__any_sync(0xffffffffu, bad)) {
    const int st = token_sigma(mag);
    const float inv = pow2_int(-st);
    wscale = pow2_int(st);
    for (int e = 0; e < p.E; ++e) {
      const uint4* wr = reinterpret_cast<const uint4*>(p.router_w + (size_t)e * kH);
      float a = 0.f;
      for (int c = lane; c < kH / 8; c += 32) {
        const uint4 xv = xr[c], wv = wr[c];
        const uint32_t xa[4] = {xv.x, xv.y, xv.z, xv.w}, wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          a = fmaf(bf16lo(xa[o]) * inv, bf16lo(wa[o]), a);
          a = fmaf(bf16hi(xa[o]) * inv, bf16hi(wa[o]), a);
        }
      }
      a = warp_sum(a);
      if (lane == 0) lg[warp][e] = a + (p.router_bias ? p.router_bias[e] * inv : 0.f);
    }
  }
  __syncwarp();
  warp_topk_fast(lg[warp], p.E, p.k, s_idx[warp], s_w[warp], wscale);
  if (lane < p.k) {
    const int e = s_idx[warp][lane];
    const float w = s_w[warp][lane];
    // the pair's expert as an index into the local weights, -1 if not held here
    const int el = (unsigned)(e - p.e0) < (unsigned)p.e_local ? e - p.e0 : -1;
    ti[t * p.k + lane] = el;
    tw[t * p.k + lane] = w;
    if (p.topk_idx_out) p.topk_idx_out[t * p.k + lane] = e;
    if (p.topk_w_out) p.topk_w_out[t * p.k + lane] = w;
    if (el >= 0) atomicAdd(&cnt[el], 1);
  }
}

// ---------------------------------------------------------------- plan
// One CTA, thread e <= E (e == E is the shared expert over all T tokens).
// Routed experts with 1..kGvMaxTok tokens go to the GEMV list (small), the
// others and the shared expert to the tile lists.
// Position runs: off[e] = exclusive scan of the pair counts.  N-tiles of
// <= 128 positions: the full ones and each expert's remainder, bucketed by
// MMA width (16..128 in steps of 16) and listed widest first, so that the
// round-robin over CTAs hands out the costly tiles first.  Each N-tile
// expands into its M-tiles (6 for gate/up, 10 for down) consecutively.
// Leaves cnt and fill at zero for the next call.
__device__ __forceinline__ void write_ntile(int idx, int e, int pos0, int n, int4* gu_tiles, int4* dn_tiles) {
  for (int mt = 0; mt < kTcMTilesGu; ++mt) gu_tiles[idx * kTcMTilesGu + mt] = make_int4(e, mt, pos0, n);
  for (int mt = 0; mt < kTcMTilesDn; ++mt) dn_tiles[idx * kTcMTilesDn + mt] = make_int4(e, mt, pos0, n);
}

// The shared expert's rows are positions Pall + t (Pall = T * k, where the
// scatter writes them), whether or not every routed pair is held here.
__global__ void __launch_bounds__(kPlanThreads) grp_plan_kernel(int T, int E, int shared_on, int Pall, int32_t* cnt,
                                                                int32_t* fill,
                                                                int32_t* off, int4* gu_tiles, int4* dn_tiles,
                                                                int32_t* ntiles, int4* small, int32_t* nsmall) {
  constexpr int NV = 10;  // [0] pairs, [1 + b] N-tiles of width bucket b, [9] GEMV experts
  __shared__ int wtot[kPlanThreads / 32][NV];
  __shared__ int wbase[kPlanThreads / 32][NV];
  __shared__ int total[NV];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int c = t < E ? cnt[t] : (t == E && shared_on ? T : 0);
  const bool gemv = t < E && c > 0 && c <= kGvMaxTok;
  const int full = gemv ? 0 : c / kTcTileN, rem = gemv ? 0 : c % kTcTileN;
  const int pb = rem > 0 ? (rem + 15) / 16 - 1 : -1;
  int v[NV];
  v[0] = t < E ? c : 0;
#pragma unroll
  for (int b = 0; b < 8; ++b) v[1 + b] = (b == 7 ? full : 0) + (pb == b ? 1 : 0);
  v[9] = gemv ? 1 : 0;
  // block exclusive scan of the 9 values
  int incl[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    int s = v[i];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    incl[i] = s;
    if (lane == 31) wtot[warp][i] = s;
  }
  __syncthreads();
  if (t < NV) {
    int a = 0;
    for (int w = 0; w < kPlanThreads / 32; ++w) {
      wbase[w][t] = a;
      a += wtot[w][t];
    }
    total[t] = a;
  }
  __syncthreads();
  int excl[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) excl[i] = wbase[warp][i] + incl[i] - v[i];
  // bucket b starts after all wider buckets
  int bstart[8];
  {
    int a = 0;
#pragma unroll
    for (int b = 7; b >= 0; --b) {
      bstart[b] = a;
      a += total[1 + b];
    }
    if (t == 0) {
      ntiles[0] = a * kTcMTilesGu;
      ntiles[1] = a * kTcMTilesDn;
      nsmall[0] = total[9];
    }
  }
  const int P = total[0];
  if (t < E) off[t] = excl[0];
  if (t == E) off[E] = P;
  if (gemv) small[excl[9]] = make_int4(t, excl[0], c, 0);
  if (t <= E && !gemv) {
    const int pos_base = t < E ? excl[0] : Pall;
    const int i7 = bstart[7] + excl[8];
    for (int q = 0; q < full; ++q) write_ntile(i7 + q, t, pos_base + kTcTileN * q, kTcTileN, gu_tiles, dn_tiles);
    if (pb >= 0) {
      int ib = 0, eb = 0;
#pragma unroll
      for (int b = 0; b < 8; ++b)
        if (pb == b) {
          ib = bstart[b];
          eb = excl[1 + b];
        }
      write_ntile(ib + eb + (pb == 7 ? full : 0), t, pos_base + kTcTileN * full, rem, gu_tiles, dn_tiles);
    }
  }
  if (t < E) {
    cnt[t] = 0;
    fill[t] = 0;
  }
}

// ---------------------------------------------------------------- scatter
// One CTA per token: each of its k pairs takes the next position in its
// expert's run; x_t is scaled by 2^-sigma_t (max |x_t| * 2^-sigma_t in
// [2^14, 2^15), so fp16 holds every value of the row down to 2^-24 of its
// largest exactly), converted to fp16 and written to its k positions and to
// the shared-expert row P + t.  sigma_t runs from -100 (a token whose largest
// |x| is below 2^-86 has an output below bf16's smallest subnormal either
// way) to 113 (bf16's largest finite value).
__global__ void __launch_bounds__(kRowThreads) grp_scatter_kernel(const __nv_bfloat16* x, int k, int P, int shared_on,
                                                                  const int32_t* ti, const int32_t* off,
                                                                  int32_t* fill, int32_t* perm, int32_t* inv,
                                                                  __half* xg, float* xscale) {
  const int t = blockIdx.x, c = threadIdx.x;
  __shared__ int spos[kMaxTopK + 1];
  __shared__ unsigned int smax;
  if (c == 0) smax = 0;
  if (c < k) {
    const int pp = t * k + c;
    const int e = ti[pp];  // -1: an expert not held here (no position)
    const int pos = e >= 0 ? off[e] + atomicAdd(&fill[e], 1) : -1;
    if (pos >= 0) perm[pos] = pp;
    inv[pp] = pos;
    spos[c] = pos;
  }
  if (c == k) spos[k] = shared_on ? P + t : -1;
  __syncthreads();
  const uint4 w = *reinterpret_cast<const uint4*>(x + (size_t)t * kH + 8 * c);
  const float f[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                      bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
  float m = 0.f;
#pragma unroll
  for (int o = 0; o < 8; ++o) m = fmaxf(m, fabsf(f[o]));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((c & 31) == 0) atomicMax(&smax, __float_as_uint(fminf(m, 3.0e38f)));
  __syncthreads();
  const int ex = (int)(smax >> 23) - 127;
  const int sigma = smax == 0 ? 0 : max(-100, ex - 14);  // ex <= 127: at most 113
  const float inv_s = __uint_as_float((uint32_t)(127 - sigma) << 23);
  if (c == 0) xscale[t] = __uint_as_float((uint32_t)(127 + sigma) << 23);
  __half h[8];
#pragma unroll
  for (int o = 0; o < 8; ++o) h[o] = __float2half_rn(f[o] * inv_s);
  const uint4 hv = *reinterpret_cast<const uint4*>(h);
  for (int i = 0; i <= k; ++i)
    if (spos[i] >= 0) *reinterpret_cast<uint4*>(xg + (size_t)spos[i] * kH + 8 * c) = hv;
}

// ---------------------------------------------------------------- combine
__global__ void __launch_bounds__(kRowThreads) grp_combine_kernel(const float* y, const int32_t* inv, int k, int P,
                                                                  int shared_on, const float* xscale,
                                                                  __nv_bfloat16* out, float* out_f32) {
  const int t = blockIdx.x, c = threadIdx.x;
  float s[8];
#pragma unroll
  for (int o = 0; o < 8; ++o) s[o] = 0.f;
  for (int i = 0; i <= k; ++i) {
    const int pos = i < k ? inv[t * k + i] : (shared_on ? P + t : -1);
    if (pos < 0) continue;  // an expert (or the shared expert) not computed here
    const float4 a = ldcg_f4(reinterpret_cast<const float4*>(y + (size_t)pos * kH + 8 * c));
    const float4 b = ldcg_f4(reinterpret_cast<const float4*>(y + (size_t)pos * kH + 8 * c + 4));
    s[0] += a.x; s[1] += a.y; s[2] += a.z; s[3] += a.w;
    s[4] += b.x; s[5] += b.y; s[6] += b.z; s[7] += b.w;
  }
  // y is kept as y / c_t^2: back to the token's scale, c_t = 2^(sigma_t + 13)
  // in [2^-87, 2^126], then one bf16 rounding (exact products unless the
  // result leaves fp32's range, where bf16 rounds the same way)
  const float ct = xscale[t] * (float)(1 << kGrpUnitShift);
  if (out_f32) {
    const float4 a = make_float4(s[0] * ct * ct, s[1] * ct * ct, s[2] * ct * ct, s[3] * ct * ct);
    const float4 b = make_float4(s[4] * ct * ct, s[5] * ct * ct, s[6] * ct * ct, s[7] * ct * ct);
    *reinterpret_cast<float4*>(out_f32 + (size_t)t * kH + 8 * c) = a;
    *reinterpret_cast<float4*>(out_f32 + (size_t)t * kH + 8 * c + 4) = b;
    return;
  }
  __nv_bfloat162 r[4];
#pragma unroll
  for (int o = 0; o < 4; ++o) r[o] = __floats2bfloat162_rn(s[2 * o] * ct * ct, s[2 * o + 1] * ct * ct);
  *reinterpret_cast<uint4*>(out + (size_t)t * kH + 8 * c) = *reinterpret_cast<const uint4*>(r);
}

cudaError_t setup_grouped() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(grp_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRmSmem)) !=
      cudaSuccess)
    return e;
  if ((e = setup_grouped_gemv()) != cudaSuccess) return e;
  return setup_grouped_tc();
}

cudaError_t launch_grouped(const GroupedParams& p, const GroupedWorkspace& ws, cudaStream_t s, int* nlaunch,
                           cudaEvent_t* marks) {
  int nl = 0;
  cudaError_t e = cudaSuccess;
  auto mark = [&](int i) {
    if (marks) cudaEventRecord(marks[i], s);
  };
  const int P = p.T * p.k;
  mark(0);
  grp_route_kernel<<<dim3((p.T + kRmTok - 1) / kRmTok, (p.E + kRmExp - 1) / kRmExp), kRmThreads, kRmSmem, s>>>(
      p, ws.logits);
  ++nl;
  mark(1);
  grp_topk_kernel<<<(p.T + 7) / 8, 256, 0, s>>>(p, ws.logits, ws.topk_idx, ws.topk_w, ws.cnt);
  ++nl;
  mark(2);
  grp_plan_kernel<<<1, kPlanThreads, 0, s>>>(p.T, p.e_local, p.shared_on, P, ws.cnt, ws.fill, ws.off, ws.gu_tiles,
                                             ws.dn_tiles, ws.ntiles, ws.small, ws.nsmall);
  ++nl;
  mark(3);
  grp_scatter_kernel<<<p.T, kRowThreads, 0, s>>>(p.x, p.k, P, p.shared_on, ws.topk_idx, ws.off, ws.fill, ws.perm,
                                                 ws.inv, ws.xg, ws.xscale);
  ++nl;
  TcParams tp{};
  tp.gu = p.gu;
  tp.dn = p.dn;
  tp.xscale = ws.xscale;
  tp.h16 = ws.h16;
  tp.y = ws.y;
  tp.perm = ws.perm;
  tp.topk_w = ws.topk_w;
  tp.sh_scale = ws.sh_scale;
  tp.k = p.k;
  tp.E = p.e_local;  // tiles of expert e_local are the shared expert's
  tp.P = P;
  tp.gu_tiles = ws.gu_tiles;
  tp.dn_tiles = ws.dn_tiles;
  tp.ntiles = ws.ntiles;
  tp.err = ws.err;
  tp.xg = ws.xg;
  tp.shgu16 = ws.shgu16;
  tp.shdn16 = ws.shdn16;
  tp.codec = p.codec;
  GvParams gv{};
  gv.gu = p.gu;
  gv.dn = p.dn;
  gv.xg = ws.xg;
  gv.xscale = ws.xscale;
  gv.perm = ws.perm;
  gv.topk_w = ws.topk_w;
  gv.k = p.k;
  gv.h16 = ws.h16;
  gv.y = ws.y;
  gv.small = ws.small;
  gv.nsmall = ws.nsmall;
  gv.err = ws.err;
  gv.wait_limit_ns = 2000000000ull;
  gv.codec = p.codec;
  mark(4);
  if ((e = launch_gemv_gu(gv, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  mark(5);
  if ((e = launch_tc_gemm(0, ws.maps, tp, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  mark(6);
  if ((e = launch_gemv_dn(gv, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  mark(7);
  if ((e = launch_tc_gemm(1, ws.maps, tp, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  mark(8);
  grp_combine_kernel<<<p.T, kRowThreads, 0, s>>>(ws.y, ws.inv, p.k, P, p.shared_on, ws.xscale, p.out, p.out_f32);
  ++nl;
  mark(kGroupedKernels);
  e = cudaGetLastError();
  *nlaunch = nl;
  return e;
}

}  // namespace lingmoe
