// Token-grouped path (T > kMaxDecodeT): prefill chunks and large verify
// batches of the W4 g32 MoE layer.
//
//   router       logits[T, E] = x Wr^T (+ b)                     fp32
//   top-k        per token, ties to the lower index, renormalised softmax
//   grouping     count per expert, exclusive scan, stable scatter of the
//                (token, slot) pairs into expert order (pair id ascending)
//   gate/up      per expert, tcgen05 tiles of 128 weight rows x up to 128
//                of its tokens (grouped_tc.cu)
//   down         per expert tile: y[position] = w * Wd_e h[position]
//   shared       SiLU(Wg_s x) * (Wu_s x) for all tokens, then Wd_s h
//   combine      out[t] = sum_slot y[position of (t, slot)] + shared, one bf16
//                rounding, slots summed in a fixed order
//
// Chunked prefill feeds this path (vLLM recipe page "inclusionAI/Ling-3.0-flash",
// "Launching the Server": --enable-chunked-prefill); a verify window of
// several tokens touches the union of their experts (bpdata article, section
// "Optimalizacio 3": four tokens can activate up to 32 experts).
#include "common.cuh"
#include "grouped.h"
#include "grouped_tc.h"

namespace lingmoe {

constexpr int kTile = 16;                 // tokens per expert tile
constexpr int kGThreads = 384;
constexpr int kGWarps = kGThreads / 32;
constexpr size_t kOutSmem = (size_t)kTile * kHsTok * sizeof(float);
constexpr size_t kRouterSmem = (size_t)8 * kXTok * sizeof(float);

const char* grouped_describe() {
  return "router GEMV tiles + top-k + stable counting sort by expert + tcgen05 grouped GEMMs "
         "(M=128 weight rows x N<=128 tokens, int4 dequantised to exact fp16 in shared memory, "
         "fp32 TMEM accumulators) for routed gate/up and down + shared expert + fixed-order combine";
}

cudaError_t grouped_alloc(GroupedWorkspace* ws, int E, int k, int max_T, const AllocFn& alloc) {
  ws->max_T = max_T;
  const size_t P = (size_t)max_T * k;
  cudaError_t e;
  if ((e = alloc((void**)&ws->logits, (size_t)max_T * E * sizeof(float))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->topk_idx, P * sizeof(int32_t))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->topk_w, P * sizeof(float))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->cnt, (size_t)E * sizeof(int32_t))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->off, (size_t)(E + 1) * sizeof(int32_t))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->tile_off, (size_t)(E + 1) * sizeof(int32_t))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->perm, P * sizeof(int32_t))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->inv, P * sizeof(int32_t))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->y, P * kH * sizeof(float))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->hs, (size_t)max_T * kI * sizeof(float))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->x16, (size_t)max_T * kH * sizeof(__half))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->xscale, (size_t)max_T * sizeof(float))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->h16, P * 2 * kI * sizeof(__half))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->gu_tiles, tc_max_tiles_gu((int)P, E) * sizeof(int4))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->dn_tiles, tc_max_tiles_dn((int)P, E) * sizeof(int4))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->ntiles, 4 * sizeof(int32_t))) != cudaSuccess) return e;
  return cudaSuccess;
}

// Block-cooperative: x rows toks[0..n) (bf16) -> fp32 planes + group sums.
__device__ void stage_x_rows(const __nv_bfloat16* x, const int* toks, int n, float* xs, float* cx) {
  for (int v = threadIdx.x; v < n * kXChunks; v += blockDim.x) {
    const int m = v / kXChunks, c = v - m * kXChunks;
    const uint4 w = *reinterpret_cast<const uint4*>(x + (size_t)toks[m] * kH + 8 * c);
    float* d = xs + (size_t)m * kXTok + xoff(c);
    *reinterpret_cast<float4*>(d) = make_float4(bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y));
    *reinterpret_cast<float4*>(d + kXPlane) =
        make_float4(bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w));
  }
  __syncthreads();
  if (cx) {
    for (int v = threadIdx.x; v < n * kXGroups; v += blockDim.x) {
      const int m = v / kXGroups, G = v - m * kXGroups;
      const float* xt = xs + (size_t)m * kXTok;
      float s = 0.f;
      for (int i = 0; i < 4; ++i) {
        const int c = 4 * G + i;
        const float4 a = *reinterpret_cast<const float4*>(xt + xoff(c));
        const float4 b = *reinterpret_cast<const float4*>(xt + kXPlane + xoff(c));
        s += a.x + a.y + a.z + a.w + b.x + b.y + b.z + b.w;
      }
      cx[m * kXGroups + G] = kBiasCoef * s;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- router
__global__ void __launch_bounds__(256) grp_router_kernel(GroupedParams p, float* logits) {
  extern __shared__ __align__(16) float sm[];
  __shared__ int toks[8];
  const int t0 = blockIdx.x * 8;
  const int n = min(8, p.T - t0);
  if (threadIdx.x < 8) toks[threadIdx.x] = t0 + min((int)threadIdx.x, n - 1);
  __syncthreads();
  stage_x_rows(p.x, toks, n, sm, nullptr);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = warp; e < p.E; e += 8) {
    const __nv_bfloat16* wr = p.router_w + (size_t)e * kH;
    uint4 w[kXChunks / 32];
#pragma unroll
    for (int m = 0; m < kXChunks / 32; ++m) w[m] = ldg_stream(wr + 8 * (lane + 32 * m));
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
#pragma unroll
    for (int m = 0; m < kXChunks / 32; ++m) {
      const int o = xoff(lane + 32 * m);
#pragma unroll
      for (int t = 0; t < 8; ++t)
        if (t < n)
          acc[t] = dot8_bf16(w[m], *reinterpret_cast<const float4*>(sm + t * kXTok + o),
                             *reinterpret_cast<const float4*>(sm + t * kXTok + kXPlane + o), acc[t]);
    }
    const float bias = p.router_bias ? p.router_bias[e] : 0.f;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (t < n) {
        const float v = warp_sum(acc[t]);
        if (lane == 0) logits[(size_t)(t0 + t) * p.E + e] = v + bias;
      }
    }
  }
}

__global__ void __launch_bounds__(256) grp_topk_kernel(GroupedParams p, const float* logits,
                                                       int32_t* ti, float* tw) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + warp;
  if (t >= p.T) return;
  __shared__ int si[8][kMaxTopK];
  __shared__ float sw[8][kMaxTopK];
  warp_topk(logits + (size_t)t * p.E, p.E, p.k, si[warp], sw[warp]);
  __syncwarp();
  if (lane < p.k) {
    ti[t * p.k + lane] = si[warp][lane];
    tw[t * p.k + lane] = sw[warp][lane];
    if (p.topk_idx_out) p.topk_idx_out[t * p.k + lane] = si[warp][lane];
    if (p.topk_w_out) p.topk_w_out[t * p.k + lane] = sw[warp][lane];
  }
}

// ---------------------------------------------------------------- grouping
// One warp per expert: count (pass 0) or scatter (pass 1) its pairs in
// ascending pair-id order, so the permutation is deterministic.
__global__ void __launch_bounds__(256) grp_sort_kernel(const int32_t* ti, int P, int E, int pass,
                                                       int32_t* cnt, const int32_t* off,
                                                       int32_t* perm, int32_t* inv) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (e >= E) return;
  int pos = pass ? off[e] : 0;
  for (int base = 0; base < P; base += 32) {
    const int pp = base + lane;
    const bool hit = pp < P && ti[pp] == e;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (pass && hit) {
      const int at = pos + __popc(m & ((1u << lane) - 1u));
      perm[at] = pp;
      inv[pp] = at;
    }
    pos += __popc(m);
  }
  if (!pass && lane == 0) cnt[e] = pos;
}

__global__ void grp_scan_kernel(const int32_t* cnt, int E, int32_t* off, int32_t* tile_off) {
  if (threadIdx.x == 0) {
    int a = 0, b = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = a;
      tile_off[e] = b;
      a += cnt[e];
      b += (cnt[e] + kTile - 1) / kTile;
    }
    off[E] = a;
    tile_off[E] = b;
  }
}

// ---------------------------------------------------------------- shared expert
__global__ void __launch_bounds__(kGThreads, 1) grp_shared_gu_kernel(GroupedParams p, float* hs_out) {
  extern __shared__ __align__(16) float sm[];
  __shared__ int toks[kTile];
  const int t0 = blockIdx.x * kTile;
  const int n = min(kTile, p.T - t0);
  if (threadIdx.x < kTile) toks[threadIdx.x] = t0 + min((int)threadIdx.x, n - 1);
  __syncthreads();
  stage_x_rows(p.x, toks, n, sm, nullptr);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = warp; i < kI; i += kGWarps) {
    const __nv_bfloat16* wg = p.sh_gate + (size_t)i * kH;
    const __nv_bfloat16* wu = p.sh_up + (size_t)i * kH;
    uint4 g[kXChunks / 32], u[kXChunks / 32];
#pragma unroll
    for (int m = 0; m < kXChunks / 32; ++m) {
      g[m] = ldg_stream(wg + 8 * (lane + 32 * m));
      u[m] = ldg_stream(wu + 8 * (lane + 32 * m));
    }
    float ag[kTile], au[kTile];
#pragma unroll
    for (int t = 0; t < kTile; ++t) ag[t] = au[t] = 0.f;
#pragma unroll
    for (int m = 0; m < kXChunks / 32; ++m) {
      const int o = xoff(lane + 32 * m);
#pragma unroll
      for (int t = 0; t < kTile; ++t) {
        if (t < n) {
          const float4 a = *reinterpret_cast<const float4*>(sm + t * kXTok + o);
          const float4 b = *reinterpret_cast<const float4*>(sm + t * kXTok + kXPlane + o);
          ag[t] = dot8_bf16(g[m], a, b, ag[t]);
          au[t] = dot8_bf16(u[m], a, b, au[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kTile; ++t) {
      if (t < n) {
        const float vg = warp_sum(ag[t]);
        const float vu = warp_sum(au[t]);
        if (lane == (t & 31)) hs_out[(size_t)(t0 + t) * kI + i] = silu_mul(vg, vu);
      }
    }
  }
}

// shared down + weighted combine of the routed outputs -> bf16
__global__ void __launch_bounds__(kGThreads, 1)
grp_out_kernel(GroupedParams p, GroupedWorkspace ws) {
  extern __shared__ __align__(16) float sm[];
  const int t0 = blockIdx.x * kTile;
  const int n = min(kTile, p.T - t0);
  for (int v = threadIdx.x; v < n * (kI / 4); v += blockDim.x) {
    const int m = v / (kI / 4), c4 = v - m * (kI / 4);
    const float4 h = reinterpret_cast<const float4*>(ws.hs + (size_t)(t0 + m) * kI)[c4];
    const int c = c4 >> 1, pl = c4 & 1;
    *reinterpret_cast<float4*>(sm + (size_t)m * kHsTok + pl * kHsPlane + 4 * c) = h;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane & 3, q = lane >> 2;
  for (int vb = warp; vb < kDnUnits; vb += kGWarps) {
    const int nrow = 4 * vb + r;
    const __nv_bfloat16* wd = p.sh_down + (size_t)nrow * kI;
    uint4 w[kI / 64];
#pragma unroll
    for (int m = 0; m < kI / 64; ++m) w[m] = ldg_stream(wd + 8 * (q + 8 * m));
    float acc[kTile];
#pragma unroll
    for (int t = 0; t < kTile; ++t) acc[t] = 0.f;
#pragma unroll
    for (int m = 0; m < kI / 64; ++m) {
      const int c = q + 8 * m;
#pragma unroll
      for (int t = 0; t < kTile; ++t)
        if (t < n)
          acc[t] = dot8_bf16(w[m], *reinterpret_cast<const float4*>(sm + t * kHsTok + 4 * c),
                             *reinterpret_cast<const float4*>(sm + t * kHsTok + kHsPlane + 4 * c), acc[t]);
    }
#pragma unroll
    for (int t = 0; t < kTile; ++t) {
      if (t < n) {
        float v = acc[t];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        if (q == (t & 7)) {
          const int tok = t0 + t;
          float s = 0.f;
          for (int sl = 0; sl < p.k; ++sl) s += ws.y[(size_t)ws.inv[tok * p.k + sl] * kH + nrow];
          s += v;
          p.out[(size_t)tok * kH + nrow] = __float2bfloat16_rn(s);
        }
      }
    }
  }
}

cudaError_t setup_grouped() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(grp_router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kRouterSmem)) != cudaSuccess) return e;
  if ((e = setup_grouped_tc()) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(grp_shared_gu_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(kTile * kXTok * sizeof(float)))) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(grp_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kOutSmem)) != cudaSuccess) return e;
  return cudaSuccess;
}

cudaError_t launch_grouped(const GroupedParams& p, const GroupedWorkspace& ws, cudaStream_t s,
                           int* nlaunch) {
  int nl = 0;
  cudaError_t e = cudaSuccess;
  const int P = p.T * p.k;
  grp_router_kernel<<<(p.T + 7) / 8, 256, kRouterSmem, s>>>(p, ws.logits);
  ++nl;
  grp_topk_kernel<<<(p.T + 7) / 8, 256, 0, s>>>(p, ws.logits, ws.topk_idx, ws.topk_w);
  ++nl;
  grp_sort_kernel<<<(p.E + 7) / 8, 256, 0, s>>>(ws.topk_idx, P, p.E, 0, ws.cnt, ws.off, ws.perm, ws.inv);
  ++nl;
  grp_scan_kernel<<<1, 32, 0, s>>>(ws.cnt, p.E, ws.off, ws.tile_off);
  ++nl;
  grp_sort_kernel<<<(p.E + 7) / 8, 256, 0, s>>>(ws.topk_idx, P, p.E, 1, ws.cnt, ws.off, ws.perm, ws.inv);
  ++nl;
  if ((e = launch_tc_tiles(ws.cnt, ws.off, p.E, ws.gu_tiles, ws.dn_tiles, ws.ntiles, s)) != cudaSuccess) return e;
  ++nl;
  if ((e = launch_x16(p.x, p.T, ws.x16, ws.xscale, s)) != cudaSuccess) return e;
  ++nl;
  TcParams tp{};
  tp.gu = p.gu;
  tp.dn = p.dn;
  tp.x16 = ws.x16;
  tp.xscale = ws.xscale;
  tp.h16 = ws.h16;
  tp.y = ws.y;
  tp.perm = ws.perm;
  tp.topk_w = ws.topk_w;
  tp.k = p.k;
  tp.gu_tiles = ws.gu_tiles;
  tp.dn_tiles = ws.dn_tiles;
  tp.ntiles = ws.ntiles;
  tp.err = ws.err;
  if ((e = launch_tc_gemm(0, tp, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  if ((e = launch_tc_gemm(1, tp, p.num_sms, s)) != cudaSuccess) return e;
  ++nl;
  grp_shared_gu_kernel<<<(p.T + kTile - 1) / kTile, kGThreads, kTile * kXTok * sizeof(float), s>>>(p, ws.hs);
  ++nl;
  grp_out_kernel<<<(p.T + kTile - 1) / kTile, kGThreads, kOutSmem, s>>>(p, ws);
  ++nl;
  e = cudaGetLastError();
  *nlaunch = nl;
  return e;
}

}  // namespace lingmoe
