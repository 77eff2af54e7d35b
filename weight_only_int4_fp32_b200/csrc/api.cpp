// C ABI of the W4 g32 MoE-layer library: validation, ownership, dispatch.
// The layer it computes is documented in include/ling_moe.h.
#include "ling_moe.h"

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "layout.h"
#include "decode.h"
#include "grouped.h"
#include "lmhead.h"
#include "repack.h"
#include "ep.h"

using namespace lingmoe;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(e == cudaErrorMemoryAllocation ? LING_MOE_ERR_OOM : LING_MOE_ERR_CUDA, "%s: %s (%s)",
              what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s

}  // namespace

namespace lingmoe {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace lingmoe

struct ling_moe {
  ling_moe_config_t cfg{};
  int codec = kCodecInt4;  // routed-weight format
  // expert parallel: routed weights of experts [e0, e0 + e_local) of the
  // num_experts the router scores; the shared expert is computed iff shared_on
  int e0 = 0, e_local = 0;
  int shared_on = 1;
  bool partial_only = false;  // an expert-parallel handle: forward_partial only
  int device = 0;
  int num_sms = 0;
  int decode_ctas = 0;
  int decode_T = 0;  // tokens the decode workspace holds
  std::vector<void*> allocs;
  // owned weights
  __nv_bfloat16* router_w = nullptr;
  float* router_bias = nullptr;
  uint8_t* gu = nullptr;
  uint8_t* dn = nullptr;
  __nv_bfloat16* sh_gate = nullptr;
  __nv_bfloat16* sh_up = nullptr;
  __nv_bfloat16* sh_down = nullptr;
  // decode workspace: exchange buffers and the arrival counters
  float* logits = nullptr;
  float* h_s = nullptr;
  float* h_pair = nullptr;
  unsigned long long* sync = nullptr;  // monotonic arrival counters of the decode kernel
  unsigned int* err = nullptr;
  // grouped-path workspace
  GroupedWorkspace gws{};
  // host entry point staging
  __nv_bfloat16* x_stage = nullptr;
  __nv_bfloat16* out_stage = nullptr;
  std::string desc;
  std::atomic<int64_t> launches{0};
  int skip_arrive_cta = -1;
  unsigned long long wait_limit_ns = kDefaultWaitNs;
  // optional per-kernel timing: events around the launches of the last call
  bool timing = false;
  cudaEvent_t tev[kGroupedKernels + 1] = {};
  int tev_kernels = 0;   // kernels timed in the last call
  bool tev_grouped = false;

  cudaError_t alloc(void** p, size_t bytes) {
    *p = nullptr;
    if (bytes == 0) return cudaSuccess;
    cudaError_t e = cudaMalloc(p, bytes);
    if (e == cudaSuccess) allocs.push_back(*p);
    return e;
  }
  void release() {
    for (void* p : allocs) cudaFree(p);
    allocs.clear();
  }
};

namespace {

int validate_cfg(const ling_moe_config_t* c) {
  if (c->hidden <= 0 || c->inter <= 0 || c->num_experts <= 0 || c->top_k <= 0 ||
      c->group_size <= 0 || c->max_tokens <= 0)
    return fail(LING_MOE_ERR_INVALID_ARG, "config fields must be positive");
  if (c->top_k > c->num_experts)
    return fail(LING_MOE_ERR_INVALID_ARG, "top_k (%d) exceeds num_experts (%d)", c->top_k,
                c->num_experts);
  if (c->hidden % c->group_size || c->inter % c->group_size)
    return fail(LING_MOE_ERR_INVALID_ARG, "hidden and inter must be multiples of group_size");
  if (c->hidden != kH || c->inter != kI)
    return fail(LING_MOE_ERR_UNSUPPORTED, "kernels are built for hidden=%d inter=%d (got %d, %d)",
                kH, kI, c->hidden, c->inter);
  if (c->group_size != kGroup)
    return fail(LING_MOE_ERR_UNSUPPORTED, "group_size must be %d", kGroup);
  if (c->top_k > kMaxTopK) return fail(LING_MOE_ERR_UNSUPPORTED, "top_k must be <= %d", kMaxTopK);
  if (c->num_experts > kMaxExperts)
    return fail(LING_MOE_ERR_UNSUPPORTED, "num_experts must be <= %d", kMaxExperts);
  return LING_MOE_OK;
}

int validate_weights(const ling_moe_weights_t* w, bool shared) {
  const void* req[] = {w->router_w, w->gate_q, w->gate_s, w->up_q, w->up_s, w->down_q, w->down_s,
                       shared ? w->sh_gate : w->router_w, shared ? w->sh_up : w->router_w,
                       shared ? w->sh_down : w->router_w};
  for (const void* p : req)
    if (!p) return fail(LING_MOE_ERR_INVALID_ARG, "a required weight pointer is NULL");
  for (const void* p : req)
    if (!aligned16(p)) return fail(LING_MOE_ERR_INVALID_ARG, "weight pointers must be 16-byte aligned");
  if (w->router_bias && !aligned16(w->router_bias))
    return fail(LING_MOE_ERR_INVALID_ARG, "router_bias must be 16-byte aligned");
  return LING_MOE_OK;
}

}  // namespace

extern "C" {

const char* ling_moe_last_error(void) { return g_last_error.c_str(); }

static int create_impl(const ling_moe_config_t* cfg, const ling_moe_weights_t* w, int codec,
                       const ling_moe_ep_t* ep, ling_moe_t** out) {
  if (!out) return fail(LING_MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!cfg || !w) return fail(LING_MOE_ERR_INVALID_ARG, "cfg or weights is NULL");
  int rc = validate_cfg(cfg);
  if (rc) return rc;
  if (ep && (ep->expert_begin < 0 || ep->expert_count < 1 ||
             ep->expert_begin > cfg->num_experts - ep->expert_count || (ep->with_shared & ~1)))
    return fail(LING_MOE_ERR_INVALID_ARG, "expert range [%d, %d + %d) outside [0, %d) or with_shared not 0/1",
                ep ? ep->expert_begin : 0, ep ? ep->expert_begin : 0, ep ? ep->expert_count : 0,
                cfg->num_experts);
  const bool shared = !ep || ep->with_shared;
  rc = validate_weights(w, shared);
  if (rc) return rc;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10)
    return fail(LING_MOE_ERR_UNSUPPORTED, "needs an sm_100 GPU (got sm_%d%d)", prop.major, prop.minor);
  if (!prop.cooperativeLaunch) return fail(LING_MOE_ERR_UNSUPPORTED, "cooperative launch unsupported");
  if (prop.multiProcessorCount < 80)
    return fail(LING_MOE_ERR_UNSUPPORTED, "needs at least 80 SMs (got %d)", prop.multiProcessorCount);

  e = setup_decode();
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel attributes");
  if (decode_max_ctas_per_sm() < 1)
    return fail(LING_MOE_ERR_UNSUPPORTED, "decode kernel does not fit on an SM");
  e = setup_grouped();
  if (e != cudaSuccess) return cuda_fail(e, "grouped kernel attributes");

  ling_moe* h = new ling_moe();
  h->cfg = *cfg;
  h->codec = codec;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  h->decode_ctas = prop.multiProcessorCount;
  h->decode_T = cfg->max_tokens < kMaxDecodeT ? cfg->max_tokens : kMaxDecodeT;
  h->e0 = ep ? ep->expert_begin : 0;
  h->e_local = ep ? ep->expert_count : cfg->num_experts;
  h->shared_on = shared ? 1 : 0;
  h->partial_only = ep != nullptr;

  const int E = cfg->num_experts, K = cfg->top_k, EL = h->e_local;
  const size_t shb = shared ? 1 : 0;
  const size_t bf = sizeof(__nv_bfloat16);
  struct A { void** p; size_t n; } plan[] = {
      {(void**)&h->router_w, (size_t)E * kH * bf},
      {(void**)&h->router_bias, w->router_bias ? (size_t)E * sizeof(float) : 0},
      {(void**)&h->gu, (size_t)EL * kGuExpertBytes},
      {(void**)&h->dn, (size_t)EL * kDnExpertBytes},
      {(void**)&h->sh_gate, shb * kI * kH * bf},
      {(void**)&h->sh_up, shb * kI * kH * bf},
      {(void**)&h->sh_down, shb * kH * kI * bf},
      {(void**)&h->logits, (size_t)h->decode_T * E * sizeof(float)},
      {(void**)&h->h_s, (size_t)h->decode_T * kI * sizeof(float)},
      {(void**)&h->h_pair, (size_t)h->decode_T * K * kI * sizeof(float)},
      {(void**)&h->sync, 4 * sizeof(unsigned long long)},
      {(void**)&h->err, 4 * sizeof(unsigned int)},
      {(void**)&h->x_stage, (size_t)cfg->max_tokens * kH * bf},
      {(void**)&h->out_stage, (size_t)cfg->max_tokens * kH * bf},
  };
  for (auto& a : plan) {
    e = h->alloc(a.p, a.n);
    if (e != cudaSuccess) {
      rc = cuda_fail(e, "cudaMalloc");
      h->release();
      delete h;
      return rc;
    }
  }
  const bool grouped = cfg->max_tokens > kMaxDecodeT;
  if (grouped) {
    h->gws.err = h->err;
    e = grouped_alloc(&h->gws, E, K, cfg->max_tokens,
                      [h](void** p, size_t n) { return h->alloc(p, n); });
    if (e != cudaSuccess) {
      rc = cuda_fail(e, "cudaMalloc (grouped workspace)");
      h->release();
      delete h;
      return rc;
    }
  }

  cudaStream_t s = nullptr;
  e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaMemcpyAsync(h->router_w, w->router_w, (size_t)E * kH * bf, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && w->router_bias)
    e = cudaMemcpyAsync(h->router_bias, w->router_bias, (size_t)E * sizeof(float), cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && shared)
    e = cudaMemcpyAsync(h->sh_gate, w->sh_gate, (size_t)kI * kH * bf, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && shared)
    e = cudaMemcpyAsync(h->sh_up, w->sh_up, (size_t)kI * kH * bf, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess && shared)
    e = cudaMemcpyAsync(h->sh_down, w->sh_down, (size_t)kH * kI * bf, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->sync, 0, 4 * sizeof(unsigned long long), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->err, 0, 4 * sizeof(unsigned int), s);
  if (e == cudaSuccess)
    e = launch_repack(w->gate_q, w->up_q, w->gate_s, w->up_s, w->down_q, w->down_s, h->gu, h->dn, EL, codec, s);
  if (e == cudaSuccess && grouped)
    e = grouped_prepare(&h->gws, E, shared ? h->sh_gate : nullptr, h->sh_up, h->sh_down, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (s) cudaStreamDestroy(s);
  if (e != cudaSuccess) {
    rc = cuda_fail(e, "create: copy/repack");
    h->release();
    delete h;
    return rc;
  }

  std::string ep_desc;
  if (ep) {
    char eb[160];
    snprintf(eb, sizeof(eb), " | expert parallel: experts [%d, %d) of %d, shared expert %s, fp32 partial output",
             h->e0, h->e0 + h->e_local, E, shared ? "here" : "elsewhere");
    ep_desc = eb;
  }
  char buf[1200];
  snprintf(buf, sizeof(buf),
           "ling_moe sm_%d%d %d SMs | H=%d I=%d E=%d k=%d g=%d max_tokens=%d bias=%s%s | "
           "decode path (1<=T<=%d): 1 cooperative launch grid=%dx%d smem=%zuB, %s GEMV "
           "dequant-in-register, fp32 accumulate, expert union deduplicated over the call's tokens | "
           "grouped path (T>%d): %s",
           prop.major, prop.minor, h->num_sms, kH, kI, E, K, kGroup, cfg->max_tokens,
           w->router_bias ? "yes" : "no", ep_desc.c_str(), kMaxDecodeT, h->decode_ctas, kDecodeThreads,
           decode_smem_bytes(1), codec == kCodecMxfp4 ? "MXFP4 (E2M1, E8M0 per 32)" : "W4 g32", kMaxDecodeT,
           grouped_describe());
  h->desc = buf;
  *out = h;
  return LING_MOE_OK;
}

int ling_moe_create(const ling_moe_config_t* cfg, const ling_moe_weights_t* w, ling_moe_t** out) {
  return create_impl(cfg, w, kCodecInt4, nullptr, out);
}

int ling_moe_create_mxfp4(const ling_moe_config_t* cfg, const ling_moe_weights_t* w, ling_moe_t** out) {
  return create_impl(cfg, w, kCodecMxfp4, nullptr, out);
}

int ling_moe_create_ep(const ling_moe_config_t* cfg, const ling_moe_weights_t* w, const ling_moe_ep_t* ep,
                       ling_moe_t** out) {
  if (!ep) return fail(LING_MOE_ERR_INVALID_ARG, "ep is NULL");
  if (ep->format != LING_MOE_FORMAT_INT4 && ep->format != LING_MOE_FORMAT_MXFP4)
    return fail(LING_MOE_ERR_INVALID_ARG, "ep->format must be LING_MOE_FORMAT_INT4 or LING_MOE_FORMAT_MXFP4");
  return create_impl(cfg, w, ep->format == LING_MOE_FORMAT_MXFP4 ? kCodecMxfp4 : kCodecInt4, ep, out);
}

// out: bf16 [T, H], or (partial) fp32 [T, H]
static int forward_impl(ling_moe_t* h, const void* x, int T, void* out, int32_t* topk_idx,
                        float* topk_w, void* stream_v, bool partial = false) {
  if (!h) return fail(LING_MOE_ERR_INVALID_ARG, "handle is NULL");
  if (h->partial_only && !partial)
    return fail(LING_MOE_ERR_INVALID_ARG, "an expert-parallel handle computes partial sums: use ling_moe_forward_partial");
  if (T < 0 || T > h->cfg.max_tokens)
    return fail(LING_MOE_ERR_INVALID_ARG, "T=%d outside [0, max_tokens=%d]", T, h->cfg.max_tokens);
  if (T == 0) return LING_MOE_OK;
  if (!x || !out) return fail(LING_MOE_ERR_INVALID_ARG, "x or out is NULL");
  if (!aligned16(x) || !aligned16(out))
    return fail(LING_MOE_ERR_INVALID_ARG, "x and out must be 16-byte aligned");
  const size_t nbytes = (size_t)T * kH * sizeof(__nv_bfloat16);
  if (overlaps(x, nbytes, out, partial ? 2 * nbytes : nbytes)) return fail(LING_MOE_ERR_INVALID_ARG, "out overlaps x");
  float* out_f32 = partial ? static_cast<float*>(out) : nullptr;
  if ((topk_idx && (reinterpret_cast<uintptr_t>(topk_idx) & 3)) ||
      (topk_w && (reinterpret_cast<uintptr_t>(topk_w) & 3)))
    return fail(LING_MOE_ERR_INVALID_ARG, "topk outputs must be 4-byte aligned");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  cudaError_t e;
  // Up to kMaxDecodeT (8) tokens: one decode launch, each distinct expert of
  // the tokens' union read once.  Beyond: the token-grouped path.
  if (T <= kMaxDecodeT) {
    const int nchunk = 1;
    if (h->timing) cudaEventRecord(h->tev[0], stream);
    for (int c = 0; c < nchunk; ++c) {
      const int t0 = c * kMaxDecodeT, Tc = c == 0 ? (T < kMaxDecodeT ? T : kMaxDecodeT) : T - kMaxDecodeT;
      DecodeParams p{};
      p.x = static_cast<const __nv_bfloat16*>(x) + (size_t)t0 * kH;
      p.out = partial ? nullptr : static_cast<__nv_bfloat16*>(out) + (size_t)t0 * kH;
      p.out_f32 = partial ? out_f32 + (size_t)t0 * kH : nullptr;
      p.e0 = h->e0;
      p.e_local = h->e_local;
      p.shared_on = h->shared_on;
      p.T = Tc;
      p.E = h->cfg.num_experts;
      p.k = h->cfg.top_k;
      p.router_w = h->router_w;
      p.router_bias = h->router_bias;
      p.gu = h->gu;
      p.dn = h->dn;
      p.sh_gate = h->sh_gate;
      p.sh_up = h->sh_up;
      p.sh_down = h->sh_down;
      p.logits = h->logits;
      p.h_s = h->h_s;
      p.h_pair = h->h_pair;
      p.topk_idx_out = topk_idx ? topk_idx + (size_t)t0 * h->cfg.top_k : nullptr;
      p.topk_w_out = topk_w ? topk_w + (size_t)t0 * h->cfg.top_k : nullptr;
      p.sync = h->sync;
      p.err = h->err;
      p.skip_arrive_cta = h->skip_arrive_cta;
      p.wait_limit_ns = h->wait_limit_ns;
      p.codec = h->codec;
      h->skip_arrive_cta = -1;  // one launch only
      e = launch_decode(p, h->decode_ctas, stream);
      if (e != cudaSuccess) return cuda_fail(e, "decode launch");
      h->launches.fetch_add(1);
      if (h->timing) cudaEventRecord(h->tev[c + 1], stream);
    }
    if (h->timing) {
      h->tev_kernels = nchunk;
      h->tev_grouped = false;
    }
    return LING_MOE_OK;
  }
  GroupedParams gp{};
  gp.x = static_cast<const __nv_bfloat16*>(x);
  gp.out = partial ? nullptr : static_cast<__nv_bfloat16*>(out);
  gp.out_f32 = out_f32;
  gp.e0 = h->e0;
  gp.e_local = h->e_local;
  gp.shared_on = h->shared_on;
  gp.T = T;
  gp.E = h->cfg.num_experts;
  gp.k = h->cfg.top_k;
  gp.router_w = h->router_w;
  gp.router_bias = h->router_bias;
  gp.gu = h->gu;
  gp.dn = h->dn;
  gp.topk_idx_out = topk_idx;
  gp.topk_w_out = topk_w;
  gp.num_sms = h->num_sms;
  gp.codec = h->codec;
  int nl = 0;
  e = launch_grouped(gp, h->gws, stream, &nl, h->timing ? h->tev : nullptr);
  h->launches.fetch_add(nl);
  if (e != cudaSuccess) return cuda_fail(e, "grouped launch");
  if (h->timing) {
    h->tev_kernels = kGroupedKernels;
    h->tev_grouped = true;
  }
  return LING_MOE_OK;
}

int ling_moe_forward(ling_moe_t* h, const void* x, int T, void* out, void* stream) {
  return forward_impl(h, x, T, out, nullptr, nullptr, stream);
}

int ling_moe_forward_ex(ling_moe_t* h, const void* x, int T, void* out, int32_t* topk_idx,
                        float* topk_w, void* stream) {
  return forward_impl(h, x, T, out, topk_idx, topk_w, stream);
}

int ling_moe_forward_partial(ling_moe_t* h, const void* x, int T, float* partial, int32_t* topk_idx,
                             float* topk_w, void* stream) {
  return forward_impl(h, x, T, partial, topk_idx, topk_w, stream, true);
}

int ling_moe_round_bf16(const float* in, void* out, size_t n, void* stream) {
  if (n == 0) return LING_MOE_OK;
  if (!in || !out) return fail(LING_MOE_ERR_INVALID_ARG, "in or out is NULL");
  if (!aligned16(in) || !aligned16(out) || (n & 7))
    return fail(LING_MOE_ERR_INVALID_ARG, "in and out must be 16-byte aligned and n a multiple of 8");
  if (overlaps(in, n * sizeof(float), out, n * sizeof(__nv_bfloat16)))
    return fail(LING_MOE_ERR_INVALID_ARG, "out overlaps in");
  const cudaError_t e = launch_round_bf16(in, static_cast<__nv_bfloat16*>(out), n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LING_MOE_OK : cuda_fail(e, "round launch");
}

int ling_moe_forward_host(ling_moe_t* h, const void* x_host, int T, void* out_host, void* stream_v) {
  if (!h) return fail(LING_MOE_ERR_INVALID_ARG, "handle is NULL");
  if (h->partial_only)
    return fail(LING_MOE_ERR_INVALID_ARG, "an expert-parallel handle computes partial sums: use ling_moe_forward_partial");
  if (T < 0 || T > h->cfg.max_tokens)
    return fail(LING_MOE_ERR_INVALID_ARG, "T=%d outside [0, max_tokens=%d]", T, h->cfg.max_tokens);
  if (T == 0) return LING_MOE_OK;
  if (!x_host || !out_host) return fail(LING_MOE_ERR_INVALID_ARG, "x_host or out_host is NULL");
  const size_t nbytes = (size_t)T * kH * sizeof(__nv_bfloat16);
  if (overlaps(x_host, nbytes, out_host, nbytes))
    return fail(LING_MOE_ERR_INVALID_ARG, "out_host overlaps x_host");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  cudaError_t e = cudaMemcpyAsync(h->x_stage, x_host, nbytes, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return cuda_fail(e, "host->device copy");
  int rc = forward_impl(h, h->x_stage, T, h->out_stage, nullptr, nullptr, stream_v);
  if (rc) return rc;
  e = cudaMemcpyAsync(out_host, h->out_stage, nbytes, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return cuda_fail(e, "device->host copy");
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  return LING_MOE_OK;
}

int ling_moe_status(ling_moe_t* h, void* stream_v) {
  if (!h) return fail(LING_MOE_ERR_INVALID_ARG, "handle is NULL");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned int err = 0;
  e = cudaMemcpy(&err, h->err, sizeof(err), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (err) {
    // A wait gave up, so some arrivals of that launch never happened and the
    // monotonic counters no longer match the launch index: clear them (no
    // launch is in flight after the synchronize) and the error word.
    cudaMemset(h->err, 0, 4 * sizeof(unsigned int));
    cudaMemset(h->sync, 0, 4 * sizeof(unsigned long long));
    if (h->gws.cnt) {  // grouped-path counters that a cut-short call may have left behind
      cudaMemset(h->gws.cnt, 0, (size_t)h->cfg.num_experts * sizeof(int32_t));
      cudaMemset(h->gws.fill, 0, (size_t)h->cfg.num_experts * sizeof(int32_t));
    }
    cudaDeviceSynchronize();
    return fail(LING_MOE_ERR_DEVICE_TIMEOUT, "a bounded device-side wait gave up (error word %u)", err);
  }
  return LING_MOE_OK;
}

const char* ling_moe_describe(const ling_moe_t* h) { return h ? h->desc.c_str() : ""; }

int64_t ling_moe_launch_count(const ling_moe_t* h) { return h ? h->launches.load() : 0; }

static void timing_events(ling_moe_t* h, bool on) {
  for (auto& ev : h->tev) {
    if (ev) cudaEventDestroy(ev);
    ev = nullptr;
  }
  h->timing = false;
  h->tev_kernels = 0;
  if (!on) return;
  for (auto& ev : h->tev)
    if (cudaEventCreate(&ev) != cudaSuccess) {
      timing_events(h, false);
      return;
    }
  h->timing = true;
}

int ling_moe_set_kernel_timing(ling_moe_t* h, int on) {
  if (!h) return fail(LING_MOE_ERR_INVALID_ARG, "handle is NULL");
  cudaError_t e = cudaSetDevice(h->device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  timing_events(h, on != 0);
  if (on && !h->timing) return fail(LING_MOE_ERR_CUDA, "could not create the timing events");
  return LING_MOE_OK;
}

int ling_moe_kernel_times(ling_moe_t* h, float* ms, int capacity, int* count) {
  if (!h || !count) return fail(LING_MOE_ERR_INVALID_ARG, "handle or count is NULL");
  if (!h->timing) return fail(LING_MOE_ERR_INVALID_ARG, "kernel timing is off");
  const int n = h->tev_kernels;
  *count = n;
  if (n == 0) return LING_MOE_OK;
  if (!ms || capacity < n) return fail(LING_MOE_ERR_INVALID_ARG, "need room for %d times", n);
  cudaError_t e = cudaEventSynchronize(h->tev[n]);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
  for (int i = 0; i < n; ++i)
    if ((e = cudaEventElapsedTime(&ms[i], h->tev[i], h->tev[i + 1])) != cudaSuccess)
      return cuda_fail(e, "cudaEventElapsedTime");
  return LING_MOE_OK;
}

const char* ling_moe_kernel_name(const ling_moe_t* h, int i) {
  static const char* const grouped[kGroupedKernels] = {"route", "topk", "plan", "scatter", "gemv_gu",
                                                       "tc_gu", "gemv_dn", "tc_dn", "combine"};
  if (!h || i < 0 || i >= h->tev_kernels) return "";
  return h->tev_grouped ? grouped[i] : "decode";
}

void ling_moe_destroy(ling_moe_t* h) {
  if (!h) return;
  timing_events(h, false);
  h->release();
  delete h;
}

#ifdef LING_MOE_TRACE
// Trace builds only: copy a grouped-path workspace buffer to the host.
int ling_moe_debug_ws(ling_moe_t* h, int which, void* dst, size_t bytes) {
  const void* src = nullptr;
  switch (which) {
    case 0: src = h->gws.h16; break;
    case 1: src = h->gws.y; break;
    case 2: src = h->gws.perm; break;
    case 3: src = h->gws.xg; break;
    case 4: src = h->gws.ntiles; break;
    case 5: src = h->gws.gu_tiles; break;
    case 6: src = h->gws.topk_w; break;
    case 7: src = h->gws.inv; break;
    default: return LING_MOE_ERR_INVALID_ARG;
  }
  return cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost) == cudaSuccess ? 0 : LING_MOE_ERR_CUDA;
}
#endif

int ling_moe_test_set_wait(ling_moe_t* h, int skip_arrive_cta, uint64_t wait_limit_ns) {
  if (!h) return fail(LING_MOE_ERR_INVALID_ARG, "handle is NULL");
  if (skip_arrive_cta >= h->decode_ctas)
    return fail(LING_MOE_ERR_INVALID_ARG, "skip_arrive_cta out of range");
  h->skip_arrive_cta = skip_arrive_cta < 0 ? -1 : skip_arrive_cta;
  h->wait_limit_ns = wait_limit_ns ? wait_limit_ns : kDefaultWaitNs;
  return LING_MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Online-FP8 LM head

struct ling_moe_lmhead {
  int device = 0;
  int vocab = 0;
  int hidden = 0;
  int nctas = 0;
  uint8_t* codes = nullptr;      // e4m3, tiled (lmh_codes_bytes)
  float* scales = nullptr;       // fp32 [vocab]
  __nv_bfloat16* x_stage = nullptr;
  float* logits_stage = nullptr;
  unsigned int* err = nullptr;   // sticky device error word
  std::atomic<int64_t> launches{0};
  int skip_cta = -1;             // test hook
  unsigned long long wait_limit_ns = kDefaultWaitNs;
  void release() {
    for (void* p : {(void*)codes, (void*)scales, (void*)x_stage, (void*)logits_stage, (void*)err})
      if (p) cudaFree(p);
    err = nullptr;
    codes = nullptr;
    scales = nullptr;
    x_stage = nullptr;
    logits_stage = nullptr;
  }
};

extern "C" {

int ling_moe_lmhead_create(const void* w, int vocab, int hidden, ling_moe_lmhead_t** out) {
  if (!out) return fail(LING_MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!w) return fail(LING_MOE_ERR_INVALID_ARG, "w is NULL");
  if (!aligned16(w)) return fail(LING_MOE_ERR_INVALID_ARG, "w must be 16-byte aligned");
  if (vocab <= 0 || hidden <= 0) return fail(LING_MOE_ERR_INVALID_ARG, "vocab and hidden must be positive");
  if (hidden % 512 || hidden > kLmhMaxHidden)
    return fail(LING_MOE_ERR_UNSUPPORTED, "hidden must be a multiple of 512 and at most %d (got %d)",
                kLmhMaxHidden, hidden);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10)
    return fail(LING_MOE_ERR_UNSUPPORTED, "needs an sm_100 GPU (got sm_%d%d)", prop.major, prop.minor);
  e = setup_lmhead();
  if (e != cudaSuccess) return cuda_fail(e, "LM-head kernel attributes");

  ling_moe_lmhead* h = new ling_moe_lmhead();
  h->device = dev;
  h->vocab = vocab;
  h->hidden = hidden;
  h->nctas = prop.multiProcessorCount;
  struct A { void** p; size_t n; } plan[] = {
      {(void**)&h->codes, lmh_codes_bytes(vocab, hidden)},
      {(void**)&h->scales, (size_t)vocab * sizeof(float)},
      {(void**)&h->x_stage, (size_t)kLmhMaxT * hidden * sizeof(__nv_bfloat16)},
      {(void**)&h->logits_stage, (size_t)kLmhMaxT * vocab * sizeof(float)},
      {(void**)&h->err, sizeof(unsigned int)},
  };
  for (auto& a : plan) {
    e = cudaMalloc(a.p, a.n);
    if (e != cudaSuccess) {
      *a.p = nullptr;
      const int rc = cuda_fail(e, "cudaMalloc");
      h->release();
      delete h;
      return rc;
    }
  }
  e = cudaMemset(h->err, 0, sizeof(unsigned int));
  if (e == cudaSuccess)
    e = launch_lmh_quantize(static_cast<const __nv_bfloat16*>(w), vocab, hidden, h->codes, h->scales, nullptr);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    const int rc = cuda_fail(e, "LM-head quantisation");
    h->release();
    delete h;
    return rc;
  }
  *out = h;
  return LING_MOE_OK;
}

static int lmhead_forward_impl(ling_moe_lmhead_t* h, const void* x, int T, float* logits, uint8_t* x_codes,
                               float* x_scales, void* stream) {
  if (!h) return fail(LING_MOE_ERR_INVALID_ARG, "handle is NULL");
  if (T < 0 || T > kLmhMaxT) return fail(LING_MOE_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, kLmhMaxT);
  if (T == 0) return LING_MOE_OK;
  if (!x || !logits) return fail(LING_MOE_ERR_INVALID_ARG, "x or logits is NULL");
  if (!aligned16(x)) return fail(LING_MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(logits) & 3u) return fail(LING_MOE_ERR_INVALID_ARG, "logits must be 4-byte aligned");
  if (x_codes && !aligned16(x_codes)) return fail(LING_MOE_ERR_INVALID_ARG, "x_codes must be 16-byte aligned");
  if (x_scales && (reinterpret_cast<uintptr_t>(x_scales) & 3u))
    return fail(LING_MOE_ERR_INVALID_ARG, "x_scales must be 4-byte aligned");
  const size_t xb = (size_t)T * h->hidden * sizeof(__nv_bfloat16), lb = (size_t)T * h->vocab * sizeof(float);
  if (overlaps(x, xb, logits, lb)) return fail(LING_MOE_ERR_INVALID_ARG, "logits overlaps x");
  if (x_codes && (overlaps(x_codes, (size_t)T * h->hidden, logits, lb) || overlaps(x_codes, (size_t)T * h->hidden, x, xb)))
    return fail(LING_MOE_ERR_INVALID_ARG, "x_codes overlaps x or logits");
  if (x_scales && (overlaps(x_scales, (size_t)T * 4, logits, lb) || overlaps(x_scales, (size_t)T * 4, x, xb)))
    return fail(LING_MOE_ERR_INVALID_ARG, "x_scales overlaps x or logits");
  cudaError_t e = launch_lmh_forward(h->codes, h->scales, h->vocab, h->hidden, static_cast<const __nv_bfloat16*>(x),
                                     T, logits, x_codes, x_scales, h->err, h->wait_limit_ns, h->skip_cta, h->nctas,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "LM-head launch");
  h->launches.fetch_add(1);
  return LING_MOE_OK;
}

int ling_moe_lmhead_forward(ling_moe_lmhead_t* h, const void* x, int T, float* logits, void* stream) {
  return lmhead_forward_impl(h, x, T, logits, nullptr, nullptr, stream);
}

int ling_moe_lmhead_forward_ex(ling_moe_lmhead_t* h, const void* x, int T, float* logits, uint8_t* x_codes,
                               float* x_scales, void* stream) {
  return lmhead_forward_impl(h, x, T, logits, x_codes, x_scales, stream);
}

int ling_moe_lmhead_forward_host(ling_moe_lmhead_t* h, const void* x_host, int T, float* logits_host,
                                 void* stream_v) {
  if (!h) return fail(LING_MOE_ERR_INVALID_ARG, "handle is NULL");
  if (T < 0 || T > kLmhMaxT) return fail(LING_MOE_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, kLmhMaxT);
  if (T == 0) return LING_MOE_OK;
  if (!x_host || !logits_host) return fail(LING_MOE_ERR_INVALID_ARG, "x_host or logits_host is NULL");
  const size_t xb = (size_t)T * h->hidden * sizeof(__nv_bfloat16), lb = (size_t)T * h->vocab * sizeof(float);
  if (overlaps(x_host, xb, logits_host, lb)) return fail(LING_MOE_ERR_INVALID_ARG, "logits_host overlaps x_host");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  cudaError_t e = cudaMemcpyAsync(h->x_stage, x_host, xb, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return cuda_fail(e, "host->device copy");
  int rc = lmhead_forward_impl(h, h->x_stage, T, h->logits_stage, nullptr, nullptr, stream_v);
  if (rc) return rc;
  e = cudaMemcpyAsync(logits_host, h->logits_stage, lb, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return cuda_fail(e, "device->host copy");
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  return LING_MOE_OK;
}

int ling_moe_lmhead_weights(const ling_moe_lmhead_t* h, uint8_t* codes, float* scales, void* stream_v) {
  if (!h || !codes || !scales) return fail(LING_MOE_ERR_INVALID_ARG, "handle, codes or scales is NULL");
  if (!aligned16(codes)) return fail(LING_MOE_ERR_INVALID_ARG, "codes must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(scales) & 3u) return fail(LING_MOE_ERR_INVALID_ARG, "scales must be 4-byte aligned");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  cudaError_t e = launch_lmh_untile(h->codes, h->vocab, h->hidden, codes, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(scales, h->scales, (size_t)h->vocab * sizeof(float), cudaMemcpyDeviceToDevice, stream);
  if (e != cudaSuccess) return cuda_fail(e, "LM-head weights copy");
  return LING_MOE_OK;
}

int ling_moe_lmhead_status(ling_moe_lmhead_t* h, void* stream_v) {
  if (!h) return fail(LING_MOE_ERR_INVALID_ARG, "handle is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream_v));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned int err = 0;
  e = cudaMemcpy(&err, h->err, sizeof(err), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (err) {
    cudaMemset(h->err, 0, sizeof(unsigned int));
    cudaDeviceSynchronize();
    return fail(LING_MOE_ERR_DEVICE_TIMEOUT, "a bounded device-side wait of the LM head gave up (error word %u)", err);
  }
  return LING_MOE_OK;
}

int64_t ling_moe_lmhead_launch_count(const ling_moe_lmhead_t* h) { return h ? h->launches.load() : 0; }

int ling_moe_lmhead_test_set_wait(ling_moe_lmhead_t* h, int skip_cta, uint64_t wait_limit_ns) {
  if (!h) return fail(LING_MOE_ERR_INVALID_ARG, "handle is NULL");
  if (skip_cta >= h->nctas) return fail(LING_MOE_ERR_INVALID_ARG, "skip_cta out of range");
  h->skip_cta = skip_cta < 0 ? -1 : skip_cta;
  h->wait_limit_ns = wait_limit_ns ? wait_limit_ns : kDefaultWaitNs;
  return LING_MOE_OK;
}

void ling_moe_lmhead_destroy(ling_moe_lmhead_t* h) {
  if (!h) return;
  h->release();
  delete h;
}

}  // extern "C"
