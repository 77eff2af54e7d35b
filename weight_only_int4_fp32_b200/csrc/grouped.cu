// Token-grouped path (T > kMaxDecodeT): prefill chunks and large verify
// batches of the W4 g32 MoE layer.
//
//   router       logits[T, E] = x Wr^T (+ b)                     fp32
//   top-k        per token, ties to the lower index, renormalised softmax
//   grouping     count per expert, exclusive scan, stable scatter of the
//                (token, slot) pairs into expert order (pair id ascending)
//   gate/up      per expert, tiles of up to 16 of its tokens: the expert's
//                weights are read once per tile and dequantised in registers
//   down         per expert tile: y[pair] = Wd_e h[pair]
//   shared       SiLU(Wg_s x) * (Wu_s x) for all tokens, then Wd_s h
//   combine      out[t] = sum_slot w[t,slot] y[t*k+slot] + shared, one bf16
//                rounding, slots summed in a fixed order
//
// Chunked prefill feeds this path (vLLM recipe page "inclusionAI/Ling-3.0-flash",
// "Launching the Server": --enable-chunked-prefill); a verify window of
// several tokens touches the union of their experts (bpdata article, section
// "Optimalizacio 3": four tokens can activate up to 32 experts).
#include "common.cuh"
#include "grouped.h"

namespace lingmoe {

constexpr int kTile = 16;                 // tokens per expert tile
constexpr int kGThreads = 384;
constexpr int kGWarps = kGThreads / 32;
constexpr size_t kGuSmem = (size_t)kTile * (kXTok + kXGroups) * sizeof(float) + 64 * sizeof(int);
constexpr size_t kDnSmem = (size_t)kTile * (kHpStride + kHGroups) * sizeof(float) + 64 * sizeof(int);
constexpr size_t kOutSmem = (size_t)kTile * kHsTok * sizeof(float);
constexpr size_t kRouterSmem = (size_t)8 * kXTok * sizeof(float);

const char* grouped_describe() {
  return "router GEMV tiles + top-k + stable counting sort by expert + per-expert 16-token "
         "tiles (W4 g32 dequant-in-register, fp32 accumulate) + shared expert + fixed-order combine";
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
  if ((e = alloc((void**)&ws->h_g, P * kI * sizeof(float))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->y, P * kH * sizeof(float))) != cudaSuccess) return e;
  if ((e = alloc((void**)&ws->hs, (size_t)max_T * kI * sizeof(float))) != cudaSuccess) return e;
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
                                                       int32_t* perm) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (e >= E) return;
  int pos = pass ? off[e] : 0;
  for (int base = 0; base < P; base += 32) {
    const int pp = base + lane;
    const bool hit = pp < P && ti[pp] == e;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (pass && hit) perm[pos + __popc(m & ((1u << lane) - 1u))] = pp;
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

// tile -> (expert, first position in perm, number of pairs)
__device__ __forceinline__ void tile_lookup(const int32_t* tile_off, const int32_t* off, int E, int tile,
                                            int* e_out, int* pos, int* n) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {  // largest e with tile_off[e] <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (tile_off[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  const int e = lo;
  const int lt = tile - tile_off[e];
  *e_out = e;
  *pos = off[e] + lt * kTile;
  *n = min(kTile, off[e + 1] - *pos);
}

// ---------------------------------------------------------------- routed gate/up
__global__ void __launch_bounds__(kGThreads, 1)
grp_gateup_kernel(GroupedParams p, GroupedWorkspace ws) {
  extern __shared__ __align__(16) float sm[];
  float* xs = sm;
  float* cx = sm + (size_t)kTile * kXTok;
  int* s_pair = reinterpret_cast<int*>(cx + kTile * kXGroups);
  int* s_tok = s_pair + kTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane & 7, q = lane >> 3;
  const int ntiles = ws.tile_off[p.E];
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    int e, pos, n;
    tile_lookup(ws.tile_off, ws.off, p.E, tile, &e, &pos, &n);
    __syncthreads();
    if (threadIdx.x < kTile) {
      const int m = min((int)threadIdx.x, n - 1);
      s_pair[threadIdx.x] = ws.perm[pos + m];
      s_tok[threadIdx.x] = ws.perm[pos + m] / p.k;
    }
    __syncthreads();
    stage_x_rows(p.x, s_tok, n, xs, cx);
    const float* xq = xs + 324 * q;
    const float* cq = cx + q * kGuChunks;
    for (int b = warp; b < kGuUnits; b += kGWarps) {
      const uint8_t* base = p.gu + ((size_t)e * kGuUnits + b) * kGuUnitBytes;
      uint4 wq[kGuChunks];
      uint2 sc[kGuChunks / 4];
#pragma unroll
      for (int j = 0; j < kGuChunks; ++j) wq[j] = ldg_stream(base + j * 512 + 16 * lane);
#pragma unroll
      for (int j = 0; j < kGuChunks / 4; ++j) sc[j] = ldg_stream64(base + kGuScaleOff + j * 256 + 8 * lane);
      float acc[kTile];
#pragma unroll
      for (int m = 0; m < kTile; ++m) acc[m] = 0.f;
#pragma unroll
      for (int j = 0; j < kGuChunks; ++j) {
        float part[kTile];
#pragma unroll
        for (int m = 0; m < kTile; ++m) part[m] = (m < n) ? cq[m * kXGroups + j] : 0.f;
        const uint32_t wj[4] = {wq[j].x, wq[j].y, wq[j].z, wq[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float f[8];
          dequant8(wj[i], f);
#pragma unroll
          for (int m = 0; m < kTile; ++m) {
            if (m < n) {
              const float* xp = xq + m * kXTok + 16 * j + 4 * i;
              part[m] = dot8_f(f, *reinterpret_cast<const float4*>(xp),
                               *reinterpret_cast<const float4*>(xp + kXPlane), part[m]);
            }
          }
        }
        const float s = scale_of(sc[j >> 2], j & 3);
#pragma unroll
        for (int m = 0; m < kTile; ++m) acc[m] = fmaf(s, part[m], acc[m]);
      }
#pragma unroll
      for (int m = 0; m < kTile; ++m) {
        if (m < n) {
          float v = acc[m];
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          const float up = __shfl_sync(0xffffffffu, v, (lane & ~7) | ((r + 4) & 7));
          if (r < 4 && q == (m & 3))
            ws.h_g[(size_t)s_pair[m] * kI + 4 * b + r] = silu_mul(kCodeScale * v, kCodeScale * up);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- routed down
__global__ void __launch_bounds__(kGThreads, 1)
grp_down_kernel(GroupedParams p, GroupedWorkspace ws) {
  extern __shared__ __align__(16) float sm[];
  float* hp = sm;
  float* chp = sm + (size_t)kTile * kHpStride;
  int* s_pair = reinterpret_cast<int*>(chp + kTile * kHGroups);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane & 3, q = lane >> 2;
  const int ntiles = ws.tile_off[p.E];
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    int e, pos, n;
    tile_lookup(ws.tile_off, ws.off, p.E, tile, &e, &pos, &n);
    __syncthreads();
    if (threadIdx.x < kTile) s_pair[threadIdx.x] = ws.perm[pos + min((int)threadIdx.x, n - 1)];
    __syncthreads();
    for (int v = threadIdx.x; v < n * (kI / 4); v += blockDim.x) {
      const int m = v / (kI / 4), c4 = v - m * (kI / 4);
      const float4 h = reinterpret_cast<const float4*>(ws.h_g + (size_t)s_pair[m] * kI)[c4];
      const int e0 = 4 * c4;
      *reinterpret_cast<float4*>(hp + (size_t)m * kHpStride + e0 + 4 * (e0 / 96)) = h;
    }
    __syncthreads();
    for (int v = threadIdx.x; v < n * kHGroups; v += blockDim.x) {
      const int m = v / kHGroups, G = v - m * kHGroups;
      const float* src = hp + (size_t)m * kHpStride + 32 * G + 4 * (G / 3);
      float s = 0.f;
      for (int i = 0; i < 32; ++i) s += src[i];
      chp[m * kHGroups + G] = kBiasCoef * s;
    }
    __syncthreads();
    const float* hq = hp + 100 * q;
    const float* cq = chp + q * kDnChunks;
    for (int vb = warp; vb < kDnUnits; vb += kGWarps) {
      const uint8_t* base = p.dn + ((size_t)e * kDnUnits + vb) * kDnUnitBytes;
      uint4 wq[kDnChunks];
      float sc[kDnChunks];
#pragma unroll
      for (int j = 0; j < kDnChunks; ++j) {
        wq[j] = ldg_stream(base + j * 512 + 16 * lane);
        sc[j] = bf16_to_f32(ldg_stream16(base + kDnScaleOff + j * 64 + 2 * lane));
      }
      float acc[kTile];
#pragma unroll
      for (int m = 0; m < kTile; ++m) acc[m] = 0.f;
#pragma unroll
      for (int j = 0; j < kDnChunks; ++j) {
        float part[kTile];
#pragma unroll
        for (int m = 0; m < kTile; ++m) part[m] = (m < n) ? cq[m * kHGroups + j] : 0.f;
        const uint32_t wj[4] = {wq[j].x, wq[j].y, wq[j].z, wq[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float f[8];
          dequant8(wj[i], f);
#pragma unroll
          for (int m = 0; m < kTile; ++m) {
            if (m < n) {
              const float* h = hq + m * kHpStride + 32 * j + 8 * i;
              part[m] = dot8_f(f, *reinterpret_cast<const float4*>(h),
                               *reinterpret_cast<const float4*>(h + 4), part[m]);
            }
          }
        }
#pragma unroll
        for (int m = 0; m < kTile; ++m) acc[m] = fmaf(sc[j], part[m], acc[m]);
      }
#pragma unroll
      for (int m = 0; m < kTile; ++m) {
        if (m < n) {
          float v = acc[m];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          if (q == (m & 7)) ws.y[(size_t)s_pair[m] * kH + 4 * vb + r] = kCodeScale * v;
        }
      }
    }
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
          for (int sl = 0; sl < p.k; ++sl) {
            const int pr = tok * p.k + sl;
            s += ws.topk_w[pr] * ws.y[(size_t)pr * kH + nrow];
          }
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
  if ((e = cudaFuncSetAttribute(grp_gateup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kGuSmem)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(grp_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kDnSmem)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(grp_shared_gu_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(kTile * kXTok * sizeof(float)))) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(grp_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kOutSmem)) != cudaSuccess) return e;
  return cudaSuccess;
}

cudaError_t launch_grouped(const GroupedParams& p, const GroupedWorkspace& ws, cudaStream_t s,
                           int* nlaunch) {
  int nl = 0;
  cudaError_t e;
  const int P = p.T * p.k;
  grp_router_kernel<<<(p.T + 7) / 8, 256, kRouterSmem, s>>>(p, ws.logits);
  ++nl;
  grp_topk_kernel<<<(p.T + 7) / 8, 256, 0, s>>>(p, ws.logits, ws.topk_idx, ws.topk_w);
  ++nl;
  grp_sort_kernel<<<(p.E + 7) / 8, 256, 0, s>>>(ws.topk_idx, P, p.E, 0, ws.cnt, ws.off, ws.perm);
  ++nl;
  grp_scan_kernel<<<1, 32, 0, s>>>(ws.cnt, p.E, ws.off, ws.tile_off);
  ++nl;
  grp_sort_kernel<<<(p.E + 7) / 8, 256, 0, s>>>(ws.topk_idx, P, p.E, 1, ws.cnt, ws.off, ws.perm);
  ++nl;
  grp_gateup_kernel<<<p.num_sms, kGThreads, kGuSmem, s>>>(p, ws);
  ++nl;
  grp_down_kernel<<<p.num_sms, kGThreads, kDnSmem, s>>>(p, ws);
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
