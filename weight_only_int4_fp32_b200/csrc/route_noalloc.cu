// Routing (router logits + top-k + renormalised weights) for callers that
// cannot allocate device memory.
//
// This is a variant of the decode kernel's routing front-end: every SM
// computes a slice of the router logits, the slices meet in scratch memory,
// and one CTA selects the top-k.  Its scratch does not come from cudaMalloc
// or a library handle: it lives in a file-scope static __device__ array that
// every GPU loading the library holds until the process exits.  Callers that
// cannot allocate -- a framework whose device memory is owned by its own
// pool, or a latency-critical path that must not call cudaMalloc (which can
// synchronise the device) -- can still route tokens with it.
//
// Every call finds the scratch as the last call left it, so nothing in it has
// to start at zero: each logit slot is one 64-bit word holding a call tag in
// its upper half and the fp32 logit in its lower half, written in one store.
// All CTAs read the generation word when they start; the call's tag is the
// generation + 1 (never 0, the value of untouched static storage).  CTA 0
// waits until every slot it needs carries the tag, selects, and writes the
// tag back as the new generation.  A call therefore never reads a value from
// an earlier call, and a call that ran out of time, or two calls that
// overlapped on the GPU (a race the caller must avoid), leave nothing behind
// that a later call could misread: the next call uses a fresh tag.
#include <mutex>

#include <cuda_runtime.h>

#include "common.cuh"
#include "ling_moe.h"

namespace lingmoe {

// Scratch: tagged logit slots of up to kRouteMaxT tokens x kMaxExperts
// experts, then the generation word and the sticky error word.
constexpr int kRouteMaxT = 4;
constexpr size_t kRouteSlotBytes = (size_t)kRouteMaxT * kMaxExperts * sizeof(unsigned long long);  // 16384
constexpr size_t kRouteGenOff = kRouteSlotBytes;
constexpr size_t kRouteErrOff = kRouteSlotBytes + 4;
constexpr size_t kRouteScratchBytes = kRouteSlotBytes + 256;  // 16,640
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

constexpr int kRouteWarps = 8;
constexpr int kRouteThreads = kRouteWarps * 32;
constexpr unsigned long long kRouteWaitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" :: "l"(p), "l"(v) : "memory");
}

// scratch: slots [T][E] at offset 0, generation and error words after them
__global__ void __launch_bounds__(kRouteThreads)
route_noalloc_kernel(const __nv_bfloat16* __restrict__ x, int T, const __nv_bfloat16* __restrict__ wr,
                     const float* __restrict__ bias, int E, int K, int32_t* topk_idx, float* topk_w,
                     unsigned char* scratch, int skip_cta, unsigned long long wait_ns) {
  __shared__ __align__(16) unsigned char xs[kRouteMaxT * kH * 2];
  __shared__ __align__(16) float lg[kRouteMaxT][kMaxExperts];
  __shared__ int si[kRouteMaxT][kMaxTopK];
  __shared__ float sw[kRouteMaxT][kMaxTopK];
  __shared__ int late;
  __shared__ unsigned long long tk_scratch[kRouteMaxT][40];
  __shared__ unsigned int xmag[kRouteMaxT];
  unsigned long long* slots = reinterpret_cast<unsigned long long*>(scratch);
  unsigned int* gen = reinterpret_cast<unsigned int*>(scratch + kRouteGenOff);
  unsigned int* err = reinterpret_cast<unsigned int*>(scratch + kRouteErrOff);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cta = blockIdx.x, ncta = gridDim.x;

  // this call's tag: read before this CTA publishes anything, so CTA 0 (which
  // moves the generation on only after every slot carries the tag) cannot
  // have moved it yet
  const unsigned int g0 = *reinterpret_cast<volatile unsigned int*>(gen);
  const unsigned int tag = g0 + 1u == 0u ? 1u : g0 + 1u;
  if (tid == 0) late = 0;
  if (tid < kRouteMaxT) xmag[tid] = 0u;
  __syncthreads();
  // x and each token's largest |x| (bf16 magnitude bits; a warp's 32 chunks
  // never straddle two tokens: 320 chunks per token)
  for (int v = tid; v < T * kH / 8; v += kRouteThreads) {
    const uint4 w = reinterpret_cast<const uint4*>(x)[v];
    reinterpret_cast<uint4*>(xs)[v] = w;
    const uint32_t m2 = __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu),
                                 __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu));
    const uint32_t wm = __reduce_max_sync(0xffffffffu, max(m2 & 0xFFFFu, m2 >> 16));
    if (lane == 0) atomicMax(&xmag[v / (kH / 8)], wm);
  }
  __syncthreads();
  // tokens outside the direct range are divided by their power-of-two scale
  // s_t, exactly as the decode kernel does: the bias then enters as b / s_t
  // and the weights as exp(s_t (l - l_0))
  bool any = false;
  for (int t = 0; t < T; ++t) any |= token_sigma(xmag[t]) != 0;
  if (any) {
    for (int v = tid; v < T * kH / 8; v += kRouteThreads) {
      const int st = token_sigma(xmag[v / (kH / 8)]);
      if (st == 0) continue;
      const float inv = pow2_int(-st);
      uint4 w = reinterpret_cast<const uint4*>(xs)[v];
      uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
      for (int o = 0; o < 4; ++o) {
        const __nv_bfloat162 r2 = __floats2bfloat162_rn(bf16lo(wv[o]) * inv, bf16hi(wv[o]) * inv);
        wv[o] = *reinterpret_cast<const uint32_t*>(&r2);
      }
      reinterpret_cast<uint4*>(xs)[v] = w;
    }
    __syncthreads();
  }

  // this CTA's router rows, one warp per row; the same accumulation order as
  // the decode kernel's router rows, so both entry points agree bit for bit
  const int r0 = (int)((long long)cta * E / ncta), r1 = (int)((long long)(cta + 1) * E / ncta);
  for (int e = r0 + warp; e < r1 && cta != skip_cta; e += kRouteWarps) {
    const __nv_bfloat16* row = wr + (size_t)e * kH;
    float g0a[kRouteMaxT], g1[kRouteMaxT], g2[kRouteMaxT], g3[kRouteMaxT];
#pragma unroll
    for (int t = 0; t < kRouteMaxT; ++t) g0a[t] = g1[t] = g2[t] = g3[t] = 0.f;
#pragma unroll
    for (int m = 0; m < kH / 256; m += 2) {
      const int c0 = lane + 32 * m, c1 = c0 + 32;
      const uint4 w0 = ldg_stream(row + 8 * c0), w1 = ldg_stream(row + 8 * c1);
#pragma unroll
      for (int t = 0; t < kRouteMaxT; ++t) {
        if (t < T) {
          dot8_bf16_bf16_2(w0, lds128(xs + t * kH * 2 + 16 * c0), g0a[t], g1[t]);
          dot8_bf16_bf16_2(w1, lds128(xs + t * kH * 2 + 16 * c1), g2[t], g3[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kRouteMaxT; ++t) {
      if (t < T) {
        const float v = warp_sum((g0a[t] + g1[t]) + (g2[t] + g3[t])) +
                        (bias ? bias[e] * pow2_int(-token_sigma(xmag[t])) : 0.f);
        if (lane == 0)
          st_relaxed_u64(slots + (size_t)t * E + e, ((unsigned long long)tag << 32) | __float_as_uint(v));
      }
    }
  }

  if (cta != 0) return;
  // CTA 0: wait (bounded) until every slot carries this call's tag, then select
  const unsigned long long t0 = globaltimer_ns();
  for (int v = tid; v < T * E; v += kRouteThreads) {
    unsigned long long s = ld_relaxed_u64(slots + v);
    while ((unsigned int)(s >> 32) != tag) {
      if (*reinterpret_cast<volatile int*>(&late) || globaltimer_ns() - t0 > wait_ns) {
        late = 1;
        break;
      }
      s = ld_relaxed_u64(slots + v);
    }
    lg[v / E][v % E] = __uint_as_float((unsigned int)s);
  }
  __syncthreads();
  const bool ok = late == 0;
  if (warp < T) {
    if (ok) {
      warp_topk_thresh(lg[warp], E, K, tk_scratch[warp], si[warp], sw[warp], pow2_int(token_sigma(xmag[warp])));
      if (lane < K) {
        topk_idx[warp * K + lane] = si[warp][lane];
        topk_w[warp * K + lane] = sw[warp][lane];
      }
    } else if (lane < K) {
      topk_idx[warp * K + lane] = -1;  // a wait ran out: no routing
      topk_w[warp * K + lane] = 0.f;
    }
  }
  if (tid == 0) {
    if (!ok) atomicOr(err, 1u);  // sticky until ling_moe_route_noalloc_status reads it
    *reinterpret_cast<volatile unsigned int*>(gen) = tag;
  }
}

void set_last_error(const char* msg);  // the library's thread-local message (api.cpp)

namespace {
std::mutex g_mu;
unsigned char* g_scratch_ptr[64] = {};  // device address of the scratch, per device ordinal
int g_skip_cta = -1;                    // test hook: next call only
unsigned long long g_wait_ns = kRouteWaitNs;
int reject(int code, const char* msg) {
  set_last_error(msg);
  return code;
}
// The scratch's device address on the current device (looked up once per device).
int scratch_address(int* dev_out, unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return reject(LING_MOE_ERR_CUDA, "route_noalloc: cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || !p) return reject(LING_MOE_ERR_CUDA, "route_noalloc: cudaGetSymbolAddress failed");
    g_scratch_ptr[dev] = static_cast<unsigned char*>(p);
  }
  *dev_out = dev;
  *out = g_scratch_ptr[dev];
  return LING_MOE_OK;
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
  unsigned char* scratch = nullptr;
  int rc = scratch_address(&dev, &scratch);
  if (rc) return rc;
  int nsm = 0;
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
    return reject(LING_MOE_ERR_CUDA, "route_noalloc: SM count query failed");
  const int nctas = nsm < num_experts ? nsm : num_experts;
  int skip;
  unsigned long long wait_ns;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    skip = g_skip_cta;
    g_skip_cta = -1;  // one call only
    wait_ns = g_wait_ns;
  }
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
                                           top_k, topk_idx, topk_w, scratch, skip, wait_ns);
  if (e != cudaSuccess) return reject(LING_MOE_ERR_CUDA, cudaGetErrorString(e));
  return LING_MOE_OK;
}

extern "C" int ling_moe_route_noalloc_status(void* stream) {
  int dev = 0;
  unsigned char* scratch = nullptr;
  int rc = scratch_address(&dev, &scratch);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int err = 0;
  cudaError_t e = cudaMemcpyAsync(&err, scratch + kRouteErrOff, sizeof(err), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return reject(LING_MOE_ERR_CUDA, "route_noalloc: reading the error word failed");
  if (err) {
    const unsigned int zero = 0;
    e = cudaMemcpyAsync(scratch + kRouteErrOff, &zero, sizeof(zero), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return reject(LING_MOE_ERR_CUDA, "route_noalloc: clearing the error word failed");
    return reject(LING_MOE_ERR_DEVICE_TIMEOUT, "route_noalloc: a device-side wait gave up (indices -1)");
  }
  return LING_MOE_OK;
}

extern "C" int ling_moe_route_noalloc_test_set_wait(int skip_cta, uint64_t wait_limit_ns) {
  if (skip_cta >= kMaxExperts) return reject(LING_MOE_ERR_INVALID_ARG, "route_noalloc: skip_cta out of range");
  std::lock_guard<std::mutex> lk(g_mu);
  g_skip_cta = skip_cta < 0 ? -1 : skip_cta;
  g_wait_ns = wait_limit_ns ? wait_limit_ns : kRouteWaitNs;
  return LING_MOE_OK;
}
