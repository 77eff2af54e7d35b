// Routing (router logits + top-k + renormalised weights) for callers that
// cannot allocate device memory.
//
// This is a variant of the decode kernel's routing front-end: every SM
// computes a slice of the router logits, the slices meet in scratch memory,
// and one CTA selects the top-k.  Its scratch does not come from cudaMalloc
// or a library handle: it lives in a file-scope static __device__ array that
// every GPU loading the library holds until the process exits.  Callers that
// cannot allocate -- code running inside a CUDA-graph capture, a framework
// whose memory is owned by its own pool, or a plugin that must not touch the
// device allocator -- can still route tokens with it.
#include <mutex>

#include <cuda_runtime.h>

#include "common.cuh"
#include "ling_moe.h"

namespace lingmoe {

// Scratch: logits of up to kRouteMaxT tokens x kMaxExperts experts, then two
// counters (router rows published, CTAs finished).  The counters start at
// zero (static storage) and the last CTA of every call puts them back to
// zero.  Calls that overlap on the GPU share the scratch and race.
constexpr int kRouteMaxT = 4;
constexpr size_t kRouteLogitsBytes = (size_t)kRouteMaxT * kMaxExperts * sizeof(float);  // 8192
constexpr size_t kRouteScratchBytes = kRouteLogitsBytes + 256;
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

constexpr int kRouteWarps = 8;
constexpr int kRouteThreads = kRouteWarps * 32;
constexpr unsigned long long kRouteWaitNs = 2000000000ull;  // 2 s

// scratch: logits [T][E] fp32 at offset 0; counters at kRouteLogitsBytes
__global__ void __launch_bounds__(kRouteThreads)
route_noalloc_kernel(const __nv_bfloat16* __restrict__ x, int T, const __nv_bfloat16* __restrict__ wr,
                     const float* __restrict__ bias, int E, int K, int32_t* topk_idx, float* topk_w,
                     unsigned char* scratch) {
  __shared__ __align__(16) unsigned char xs[kRouteMaxT * kH * 2];
  __shared__ __align__(16) float lg[kRouteMaxT][kMaxExperts];
  __shared__ int si[kRouteMaxT][kMaxTopK];
  __shared__ float sw[kRouteMaxT][kMaxTopK];
  __shared__ int ok_s;
  float* logits = reinterpret_cast<float*>(scratch);
  unsigned int* rows_done = reinterpret_cast<unsigned int*>(scratch + kRouteLogitsBytes);
  unsigned int* ctas_done = rows_done + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cta = blockIdx.x, ncta = gridDim.x;

  for (int v = tid; v < T * kH / 8; v += kRouteThreads)
    reinterpret_cast<uint4*>(xs)[v] = reinterpret_cast<const uint4*>(x)[v];
  __syncthreads();

  // this CTA's router rows, one warp per row; the same accumulation order as
  // the decode kernel's router rows, so both entry points agree bit for bit
  const int r0 = (int)((long long)cta * E / ncta), r1 = (int)((long long)(cta + 1) * E / ncta);
  for (int e = r0 + warp; e < r1; e += kRouteWarps) {
    const __nv_bfloat16* row = wr + (size_t)e * kH;
    float g0[kRouteMaxT], g1[kRouteMaxT], g2[kRouteMaxT], g3[kRouteMaxT];
#pragma unroll
    for (int t = 0; t < kRouteMaxT; ++t) g0[t] = g1[t] = g2[t] = g3[t] = 0.f;
#pragma unroll
    for (int m = 0; m < kH / 256; m += 2) {
      const int c0 = lane + 32 * m, c1 = c0 + 32;
      const uint4 w0 = ldg_stream(row + 8 * c0), w1 = ldg_stream(row + 8 * c1);
#pragma unroll
      for (int t = 0; t < kRouteMaxT; ++t) {
        if (t < T) {
          dot8_bf16_bf16_2(w0, lds128(xs + t * kH * 2 + 16 * c0), g0[t], g1[t]);
          dot8_bf16_bf16_2(w1, lds128(xs + t * kH * 2 + 16 * c1), g2[t], g3[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kRouteMaxT; ++t) {
      if (t < T) {
        const float v = warp_sum((g0[t] + g1[t]) + (g2[t] + g3[t]));
        if (lane == 0) logits[t * E + e] = v + (bias ? bias[e] : 0.f);
      }
    }
    if (lane == 0) {
      __threadfence();
      atomicAdd(rows_done, 1u);
    }
  }

  if (cta == 0) {
    // wait (bounded) for every row, then select
    if (tid == 0) {
      int ok = 1;
      const unsigned long long t0 = globaltimer_ns();
      while (ld_acquire_u32(rows_done) < (unsigned)E) {
        if (globaltimer_ns() - t0 > kRouteWaitNs) { ok = 0; break; }
      }
      ok_s = ok;
    }
    __syncthreads();
    const bool ok = ok_s != 0;
    if (ok) {
      for (int v = tid; v < T * E; v += kRouteThreads) lg[v / E][v % E] = ldcg_f32(logits + v);
    }
    __syncthreads();
    if (warp < T) {
      if (ok) {
        warp_topk_fast(lg[warp], E, K, si[warp], sw[warp]);
        if (lane < K) {
          topk_idx[warp * K + lane] = si[warp][lane];
          topk_w[warp * K + lane] = sw[warp][lane];
        }
      } else if (lane < K) {
        topk_idx[warp * K + lane] = -1;  // a wait ran out: no routing
        topk_w[warp * K + lane] = 0.f;
      }
    }
  }
  // every CTA counts itself out; the last one zeroes the counters for the next call
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(ctas_done, 1u) == (unsigned)ncta - 1u) {
      atomicExch(rows_done, 0u);
      atomicExch(ctas_done, 0u);
    }
  }
}

void set_last_error(const char* msg);  // the library's thread-local message (api.cpp)

namespace {
std::mutex g_mu;
unsigned char* g_scratch_ptr[64] = {};  // device address of the scratch, per device ordinal
int reject(int code, const char* msg) {
  set_last_error(msg);
  return code;
}
}  // namespace

}  // namespace lingmoe

using namespace lingmoe;

extern "C" int ling_moe_route_noalloc(const void* x, int T, const void* router_w, const float* router_bias,
                                      int num_experts, int top_k, int32_t* topk_idx, float* topk_w,
                                      void* stream) {
  if (T == 0) return LING_MOE_OK;
  if (!x || !router_w || !topk_idx || !topk_w)
    return reject(LING_MOE_ERR_INVALID_ARG, "route_noalloc: NULL pointer");
  if (T < 0 || T > kRouteMaxT)
    return reject(LING_MOE_ERR_INVALID_ARG, "route_noalloc: T must be in [0, 4] (scratch holds 4 tokens)");
  if (num_experts <= 0 || num_experts > kMaxExperts)
    return reject(LING_MOE_ERR_INVALID_ARG, "route_noalloc: num_experts must be in [1, 512]");
  if (top_k <= 0 || top_k > kMaxTopK || top_k > num_experts)
    return reject(LING_MOE_ERR_INVALID_ARG, "route_noalloc: top_k must be in [1, min(8, num_experts)]");
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(router_w) & 15) ||
      (reinterpret_cast<uintptr_t>(topk_idx) & 3) || (reinterpret_cast<uintptr_t>(topk_w) & 3) ||
      (router_bias && (reinterpret_cast<uintptr_t>(router_bias) & 3)))
    return reject(LING_MOE_ERR_INVALID_ARG, "route_noalloc: misaligned pointer");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return reject(LING_MOE_ERR_CUDA, "route_noalloc: cudaGetDevice failed");
  unsigned char* scratch;
  int nsm = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
      // first call on this device: the device address of the static scratch
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
      if (e != cudaSuccess || !p) return reject(LING_MOE_ERR_CUDA, "route_noalloc: cudaGetSymbolAddress failed");
      g_scratch_ptr[dev] = static_cast<unsigned char*>(p);
    }
    scratch = g_scratch_ptr[dev];
  }
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
    return reject(LING_MOE_ERR_CUDA, "route_noalloc: SM count query failed");
  const int nctas = nsm < num_experts ? nsm : num_experts;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, route_noalloc_kernel, static_cast<const __nv_bfloat16*>(x), T,
                                           static_cast<const __nv_bfloat16*>(router_w), router_bias, num_experts,
                                           top_k, topk_idx, topk_w, scratch);
  if (e != cudaSuccess) return reject(LING_MOE_ERR_CUDA, cudaGetErrorString(e));
  return LING_MOE_OK;
}
