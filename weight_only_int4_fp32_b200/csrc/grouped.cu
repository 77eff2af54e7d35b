// Token-grouped path (T > kMaxDecodeT): prefill chunks and large verify
// batches of the W4 g32 MoE layer.
//
//   route        logits[t, e] = x_t . Wr_e (+ b_e) in fp32 on CUDA cores, tiles
//                of <= 16 tokens x 64 experts
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

constexpr int kRtThreads = 256;
constexpr int kRtWarps = kRtThreads / 32;
constexpr int kRtPass = 8;      // tokens per pass (register tile: 8 experts x 8 tokens per lane)
constexpr int kRtMaxTok = 16;   // tokens per CTA
constexpr int kRtExperts = 8 * kRtWarps;  // experts per CTA: 8 per warp
constexpr size_t kRtSmem = (size_t)kRtPass * kXTok * sizeof(float);
constexpr int kPlanThreads = 1024;
constexpr int kRowThreads = kH / 8;  // 320: one thread per 8 columns of a row

const char* grouped_describe() {
  return "fp32 router GEMM + top-k + counting scatter by expert + tcgen05 grouped GEMMs "
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
  if ((e = launch_tc_prep_shared(sh_gate, sh_up, sh_down, ws->shgu16, ws->shdn16, ws->sh_scale, ws->amax,
                                 stream)) != cudaSuccess)
    return e;
  return tc_encode_maps(&ws->maps, ws->xg, ws->h16, (int)ws->rows, ws->shgu16, ws->shdn16);
}

// Block-cooperative: x rows toks[0..n) (bf16) -> fp32 planes (first and
// second halves of each 8-column chunk in separate planes, padded every 80
// chunks) so that a warp reading consecutive chunks hits distinct banks.
__device__ void stage_x_rows(const __nv_bfloat16* x, const int* toks, int n, float* xs) {
  for (int v = threadIdx.x; v < n * kXChunks; v += blockDim.x) {
    const int m = v / kXChunks, c = v - m * kXChunks;
    const uint4 w = *reinterpret_cast<const uint4*>(x + (size_t)toks[m] * kH + 8 * c);
    float* d = xs + (size_t)m * kXTok + xoff(c);
    *reinterpret_cast<float4*>(d) = make_float4(bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y));
    *reinterpret_cast<float4*>(d + kXPlane) = make_float4(bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w));
  }
}

// ---------------------------------------------------------------- route
// Logits of NT <= 8 staged tokens (rows t0 ..) for the CTA's experts.  A warp
// takes 8 experts; each lane accumulates 8 experts x NT tokens over its
// K-chunks (every 32nd chunk of 8 columns), then a reduce-scatter across the
// warp leaves lane l with the sums for expert e0 + l/4 and tokens 2(l%4), +1.
template <int NT>
__device__ __forceinline__ void route_logits(const float* xs, const GroupedParams& p, int t0, int ebase,
                                             float* logits) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  {
    const int e0 = ebase + 8 * warp;
    if (e0 >= p.E) return;
    float acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0.f;
#pragma unroll 1
    for (int c = lane; c < kXChunks; c += 32) {
      float wf[8][8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = e0 + j;
        const uint4 w = e < p.E ? ldg_stream(p.router_w + (size_t)e * kH + 8 * c) : make_uint4(0, 0, 0, 0);
        wf[j][0] = bf16lo(w.x); wf[j][1] = bf16hi(w.x); wf[j][2] = bf16lo(w.y); wf[j][3] = bf16hi(w.y);
        wf[j][4] = bf16lo(w.z); wf[j][5] = bf16hi(w.z); wf[j][6] = bf16lo(w.w); wf[j][7] = bf16hi(w.w);
      }
      const int o = xoff(c);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float4 a = ldsf4(xs + t * kXTok + o);
        const float4 b = ldsf4(xs + t * kXTok + kXPlane + o);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float s = acc[8 * j + t];
          s = fmaf(wf[j][0], a.x, s); s = fmaf(wf[j][1], a.y, s);
          s = fmaf(wf[j][2], a.z, s); s = fmaf(wf[j][3], a.w, s);
          s = fmaf(wf[j][4], b.x, s); s = fmaf(wf[j][5], b.y, s);
          s = fmaf(wf[j][6], b.z, s); s = fmaf(wf[j][7], b.w, s);
          acc[8 * j + t] = s;
        }
      }
    }
    // reduce-scatter of the 64 partial sums: after the step with offset o,
    // lane bit o selects which half of the remaining values the lane keeps
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < 2 * o; ++i) {
        const float send = up ? acc[i] : acc[i + 2 * o];
        const float keep = up ? acc[i + 2 * o] : acc[i];
        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    const int e = e0 + (lane >> 2);
    if (e < p.E) {
      const float bias = p.router_bias ? p.router_bias[e] : 0.f;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int t = 2 * (lane & 3) + u;
        if (t < NT) logits[(size_t)(t0 + t) * p.E + e] = acc[u] + bias;
      }
    }
  }
}

// CTA (x, y): tokens [x tpc, x tpc + tpc) in passes of <= 8, experts
// [64 y, 64 y + 64).  Splitting the experts keeps every SM streaming router
// rows at small T too.
__global__ void __launch_bounds__(kRtThreads, 1) grp_route_kernel(GroupedParams p, int tpc, float* logits) {
  extern __shared__ __align__(16) float xs[];
  __shared__ int toks[kRtPass];
  const int t_begin = blockIdx.x * tpc, t_end = min(p.T, t_begin + tpc);
  const int ntok = t_end - t_begin;
  const int ebase = blockIdx.y * kRtExperts;
  if (ntok <= 0) return;
  const int npass = (ntok + kRtPass - 1) / kRtPass;
  const int per = (ntok + npass - 1) / npass;
#pragma unroll 1
  for (int t0 = t_begin; t0 < t_end; t0 += per) {
    const int nt = min(per, t_end - t0);
    if (threadIdx.x < kRtPass) toks[threadIdx.x] = t0 + min((int)threadIdx.x, nt - 1);
    __syncthreads();
    stage_x_rows(p.x, toks, nt, xs);
    __syncthreads();
    switch (nt) {
      case 1: route_logits<1>(xs, p, t0, ebase, logits); break;
      case 2: route_logits<2>(xs, p, t0, ebase, logits); break;
      case 3: route_logits<3>(xs, p, t0, ebase, logits); break;
      case 4: route_logits<4>(xs, p, t0, ebase, logits); break;
      case 5: route_logits<5>(xs, p, t0, ebase, logits); break;
      case 6: route_logits<6>(xs, p, t0, ebase, logits); break;
      case 7: route_logits<7>(xs, p, t0, ebase, logits); break;
      default: route_logits<8>(xs, p, t0, ebase, logits); break;
    }
    __syncthreads();
  }
}

// One warp per token: top-k of its logits, the renormalised weights, and
// one count per selected expert.
__global__ void __launch_bounds__(256) grp_topk_kernel(GroupedParams p, const float* logits, int32_t* ti,
                                                       float* tw, int32_t* cnt) {
  __shared__ float lg[8][kMaxExperts];
  __shared__ int s_idx[8][kMaxTopK];
  __shared__ float s_w[8][kMaxTopK];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + warp;
  if (t >= p.T) return;
  for (int e = lane; e < p.E; e += 32) lg[warp][e] = logits[(size_t)t * p.E + e];
  __syncwarp();
  warp_topk_fast(lg[warp], p.E, p.k, s_idx[warp], s_w[warp]);
  if (lane < p.k) {
    const int e = s_idx[warp][lane];
    const float w = s_w[warp][lane];
    ti[t * p.k + lane] = e;
    tw[t * p.k + lane] = w;
    if (p.topk_idx_out) p.topk_idx_out[t * p.k + lane] = e;
    if (p.topk_w_out) p.topk_w_out[t * p.k + lane] = w;
    atomicAdd(&cnt[e], 1);
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

__global__ void __launch_bounds__(kPlanThreads) grp_plan_kernel(int T, int E, int32_t* cnt, int32_t* fill,
                                                                int32_t* off, int4* gu_tiles, int4* dn_tiles,
                                                                int32_t* ntiles, int4* small, int32_t* nsmall) {
  constexpr int NV = 10;  // [0] pairs, [1 + b] N-tiles of width bucket b, [9] GEMV experts
  __shared__ int wtot[kPlanThreads / 32][NV];
  __shared__ int wbase[kPlanThreads / 32][NV];
  __shared__ int total[NV];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int c = t < E ? cnt[t] : (t == E ? T : 0);
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
    const int pos_base = t < E ? excl[0] : P;
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
// [2^14, 2^15), so fp16 holds every bf16 value of a normal-range row exactly),
// converted to fp16 and written to its k positions and to the shared-expert
// row P + t.
__global__ void __launch_bounds__(kRowThreads) grp_scatter_kernel(const __nv_bfloat16* x, int k, int P,
                                                                  const int32_t* ti, const int32_t* off,
                                                                  int32_t* fill, int32_t* perm, int32_t* inv,
                                                                  __half* xg, float* xscale) {
  const int t = blockIdx.x, c = threadIdx.x;
  __shared__ int spos[kMaxTopK + 1];
  __shared__ unsigned int smax;
  if (c == 0) smax = 0;
  if (c < k) {
    const int pp = t * k + c;
    const int e = ti[pp];
    const int pos = off[e] + atomicAdd(&fill[e], 1);
    perm[pos] = pp;
    inv[pp] = pos;
    spos[c] = pos;
  }
  if (c == k) spos[k] = P + t;
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
  const int sigma = smax == 0 ? 0 : max(-100, min(100, ex - 14));
  const float inv_s = __uint_as_float((uint32_t)(127 - sigma) << 23);
  if (c == 0) xscale[t] = __uint_as_float((uint32_t)(127 + sigma) << 23);
  __half h[8];
#pragma unroll
  for (int o = 0; o < 8; ++o) h[o] = __float2half_rn(f[o] * inv_s);
  const uint4 hv = *reinterpret_cast<const uint4*>(h);
  for (int i = 0; i <= k; ++i) *reinterpret_cast<uint4*>(xg + (size_t)spos[i] * kH + 8 * c) = hv;
}

// ---------------------------------------------------------------- combine
__global__ void __launch_bounds__(kRowThreads) grp_combine_kernel(const float* y, const int32_t* inv, int k, int P,
                                                                  __nv_bfloat16* out) {
  const int t = blockIdx.x, c = threadIdx.x;
  float s[8];
#pragma unroll
  for (int o = 0; o < 8; ++o) s[o] = 0.f;
  for (int i = 0; i <= k; ++i) {
    const int pos = i < k ? inv[t * k + i] : P + t;
    const float4 a = ldcg_f4(reinterpret_cast<const float4*>(y + (size_t)pos * kH + 8 * c));
    const float4 b = ldcg_f4(reinterpret_cast<const float4*>(y + (size_t)pos * kH + 8 * c + 4));
    s[0] += a.x; s[1] += a.y; s[2] += a.z; s[3] += a.w;
    s[4] += b.x; s[5] += b.y; s[6] += b.z; s[7] += b.w;
  }
  __nv_bfloat162 r[4];
#pragma unroll
  for (int o = 0; o < 4; ++o) r[o] = __floats2bfloat162_rn(s[2 * o], s[2 * o + 1]);
  *reinterpret_cast<uint4*>(out + (size_t)t * kH + 8 * c) = *reinterpret_cast<const uint4*>(r);
}

cudaError_t setup_grouped() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(grp_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRtSmem)) !=
      cudaSuccess)
    return e;
  if ((e = setup_grouped_gemv()) != cudaSuccess) return e;
  return setup_grouped_tc();
}

cudaError_t launch_grouped(const GroupedParams& p, const GroupedWorkspace& ws, cudaStream_t s, int* nlaunch) {
  int nl = 0;
  cudaError_t e = cudaSuccess;
  const int P = p.T * p.k;
  const int eblocks = (p.E + kRtExperts - 1) / kRtExperts;
  const int tpc = std::max(1, std::min(kRtMaxTok, (p.T * eblocks + 2 * p.num_sms - 1) / (2 * p.num_sms)));
  grp_route_kernel<<<dim3((p.T + tpc - 1) / tpc, (p.E + kRtExperts - 1) / kRtExperts), kRtThreads, kRtSmem, s>>>(
      p, tpc, ws.logits);
  ++nl;
  grp_topk_kernel<<<(p.T + 7) / 8, 256, 0, s>>>(p, ws.logits, ws.topk_idx, ws.topk_w, ws.cnt);
  ++nl;
  grp_plan_kernel<<<1, kPlanThreads, 0, s>>>(p.T, p.E, ws.cnt, ws.fill, ws.off, ws.gu_tiles, ws.dn_tiles, ws.ntiles,
                                             ws.small, ws.nsmall);
  ++nl;
  grp_scatter_kernel<<<p.T, kRowThreads, 0, s>>>(p.x, p.k, P, ws.topk_idx, ws.off, ws.fill, ws.perm, ws.inv, ws.xg,
                                                 ws.xscale);
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
  tp.E = p.E;
  tp.P = P;
  tp.gu_tiles = ws.gu_tiles;
  tp.dn_tiles = ws.dn_tiles;
  tp.ntiles = ws.ntiles;
  tp.err = ws.err;
  tp.xg = ws.xg;
  tp.shgu16 = ws.shgu16;
  tp.shdn16 = ws.shdn16;
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
  if ((e = launch_gemv_gu(gv, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  if ((e = launch_tc_gemm(0, ws.maps, tp, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  if ((e = launch_gemv_dn(gv, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  if ((e = launch_tc_gemm(1, ws.maps, tp, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  grp_combine_kernel<<<p.T, kRowThreads, 0, s>>>(ws.y, ws.inv, p.k, P, p.out);
  ++nl;
  e = cudaGetLastError();
  *nlaunch = nl;
  return e;
}

}  // namespace lingmoe
