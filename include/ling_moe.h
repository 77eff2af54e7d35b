/*
 * ling_moe.h -- C ABI of a B200 (sm_100a) library for the routed-expert
 * mixture-of-experts layer of a Ling-3.0-flash-shaped model with W4 g32
 * routed-expert weights.
 *
 * What one call computes (for each of T tokens x[t], hidden H):
 *
 *   logits[e] = sum_h x[h] * Wr[e,h] (+ b[e])                    fp32
 *   S         = the k experts with the largest logits, ties to the lower index
 *   w_e       = exp(logits[e]) / sum_{j in S} exp(logits[j]),  e in S
 *               (softmax over all experts renormalised over S; sums to 1)
 *   out       = sum_{e in S} w_e * Wd_e (SiLU(Wg_e x) * (Wu_e x))
 *             + Wd_s (SiLU(Wg_s x) * (Wu_s x))                   -> bf16
 *
 * Sources for the structure: the vLLM recipe page "inclusionAI/Ling-3.0-flash"
 * (section Overview: 512 routed experts, 8 active per token, one shared
 * expert; section "Single-GPU int4": symmetric W4, group_size 32, routed
 * experts only, shared expert in bf16) and the bpdata article "Harom
 * optimalizacio a Ling-3.0-flash MoE inferenciajanak" (section "Modell es
 * kiindulo konfiguracio": 8 of 512 routed experts plus one shared expert,
 * hidden 2,560; section "Optimalizacio 1": moe_intermediate_size 768).  The
 * pages do not state the gate function or the FFN form; this library fixes
 * softmax -> top-k (ties to the lower index) -> renormalise, and the SwiGLU
 * FFN above.  Routed weights are w = q * s with q a signed 4-bit code in
 * [-8, 7] and s one bf16 scale per 32 consecutive elements along K.
 *
 * Canonical int4 packing at this boundary: two's-complement nibbles, two per
 * byte, the LOW nibble holds the EVEN index along K, bytes run along K,
 * rows are row-major [rows, K/2].  The library copies and repacks weights
 * into its own layout inside ling_moe_create.
 *
 * Threading / streams: a handle owns a workspace, so one handle must not be
 * used by two streams (or two host threads) at the same time.  Different
 * handles are independent.
 */
#ifndef LING_MOE_H
#define LING_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes of every entry point. */
typedef enum {
  LING_MOE_OK = 0,
  LING_MOE_ERR_INVALID_ARG = -1,   /* bad pointer, size, alignment or aliasing; nothing enqueued */
  LING_MOE_ERR_CUDA = -2,          /* a CUDA runtime call failed; see ling_moe_last_error() */
  LING_MOE_ERR_OOM = -3,           /* device allocation failed in ling_moe_create */
  LING_MOE_ERR_UNSUPPORTED = -4,   /* shape outside what the kernels are built for */
  LING_MOE_ERR_DEVICE_TIMEOUT = -5 /* a bounded device-side wait gave up (sticky) */
} ling_moe_status_t;

/* Layer shape.  Supported: hidden == 2560, inter == 768 (the Ling-3.0-flash
 * MoE shape; the kernels are specialised for it), group_size == 32,
 * 1 <= top_k <= 8, top_k <= num_experts <= 512, max_tokens >= 1. */
typedef struct {
  int hidden;       /* H */
  int inter;        /* I, per expert (moe_intermediate_size) */
  int num_experts;  /* E, routed experts */
  int top_k;        /* k */
  int group_size;   /* g, int4 scale group along K */
  int max_tokens;   /* largest T any forward call on this handle will pass */
} ling_moe_config_t;

/* Weights in the canonical layout, all DEVICE pointers on the current device.
 * Read only during ling_moe_create (copied and repacked); the caller may free
 * them as soon as it returns.  bf16 tensors are raw 16-bit patterns. */
typedef struct {
  const void *router_w;     /* bf16 [E, H] row-major */
  const float *router_bias; /* fp32 [E], added to the logits before selection, or NULL */
  const uint8_t *gate_q;    /* int4 [E, I, H/2] packed as described above */
  const void *gate_s;       /* bf16 [E, I, H/g] */
  const uint8_t *up_q;      /* int4 [E, I, H/2] */
  const void *up_s;         /* bf16 [E, I, H/g] */
  const uint8_t *down_q;    /* int4 [E, H, I/2] */
  const void *down_s;       /* bf16 [E, H, I/g] */
  const void *sh_gate;      /* bf16 [I, H] shared expert */
  const void *sh_up;        /* bf16 [I, H] */
  const void *sh_down;      /* bf16 [H, I] */
} ling_moe_weights_t;

typedef struct ling_moe ling_moe_t; /* opaque handle */

/* Validate cfg and weights, allocate library-owned device memory (repacked
 * weights + workspace sized for cfg->max_tokens), repack, synchronise.
 * The only entry point that allocates or synchronises the device.
 * On success *out is a new handle; on failure *out is NULL and nothing leaks.
 * Errors: INVALID_ARG (NULL pointers, nonsensical sizes), UNSUPPORTED (a shape
 * the kernels are not built for), OOM, CUDA. */
int ling_moe_create(const ling_moe_config_t *cfg, const ling_moe_weights_t *w,
                    ling_moe_t **out);

/* The same layer with MXFP4 routed experts (OCP Microscaling MXFP4: FP4
 * E2M1 elements -- bit 3 sign, bits 2..1 exponent with bias 1, bit 0
 * mantissa, values +-{0, 0.5, 1, 1.5, 2, 3, 4, 6} -- and one E8M0 scale
 * 2^(e - 127) per 32 consecutive K elements).  The pages profile an MXFP4
 * checkpoint of the model (bpdata article, sections "Modell es kiindulo
 * konfiguracio" and "Optimalizacio 1: Humming MXFP4 MoE backend") without
 * defining the format; this is the OCP definition.
 * Weights: as ling_moe_create, except that gate_q / up_q / down_q hold E2M1
 * codes (two per byte, low nibble = even K index) and gate_s / up_s / down_s
 * hold E8M0 scale bytes, uint8 [E, rows, K/32].  Scale exponents above 240
 * (scales of 2^114 and more) are not supported: they give NaN outputs.  The
 * token-grouped path (T > 8) feeds the tensor cores exact fp16 weights
 * value * scale * 2^8, which holds for exponents e in [96, 132] (scales 2^-31
 * to 2^5); outside that range its weights lose bits or overflow.
 * Limits: as ling_moe_create.  Every other entry point works on the handle as
 * documented; both paths (T <= 8 decode launches, T > 8 token-grouped) run
 * for MXFP4 weights. */
int ling_moe_create_mxfp4(const ling_moe_config_t *cfg, const ling_moe_weights_t *w,
                          ling_moe_t **out);

/* out[T, H] (bf16) = layer(x[T, H] bf16) on `stream` (a cudaStream_t, NULL =
 * legacy default stream).  x and out are DEVICE pointers owned by the caller,
 * contiguous row-major, 16-byte aligned; out must not overlap x.
 * 0 <= T <= max_tokens; T == 0 returns OK and enqueues nothing.
 * Range: every finite bf16 x (subnormals and values up to bf16's largest
 * included) is computed with the same relative precision, through a
 * power-of-two scale per token; out is the exact result rounded once to bf16,
 * so +-inf where that result overflows bf16.  Non-finite x is outside the
 * contract (no trap, no check; the outputs are then undefined).
 * Asynchronous: no host synchronisation and no allocation, so the call can be
 * captured into a CUDA graph.  Device-detected failures (a bounded wait that
 * gave up) are reported later by ling_moe_status.
 * Kernels: T <= 4 one persistent decode launch; 5 <= T <= 8 two of them (the
 * first 4 tokens, then the rest); larger T the token-grouped path (9 launches).
 * Errors: INVALID_ARG (checked on the host before anything is enqueued), CUDA. */
int ling_moe_forward(ling_moe_t *h, const void *x, int T, void *out, void *stream);

/* As ling_moe_forward, and also writes the routing: topk_idx int32 [T, k]
 * (expert indices ordered by logit descending, ties to the lower index) and
 * topk_w fp32 [T, k] (renormalised weights, same order).  Either may be NULL.
 * Both are DEVICE pointers. */
int ling_moe_forward_ex(ling_moe_t *h, const void *x, int T, void *out,
                        int32_t *topk_idx, float *topk_w, void *stream);

/* End-to-end call on HOST buffers: copies x_host [T, H] bf16 to the device,
 * runs the layer, copies the result to out_host [T, H] bf16 and waits for the
 * stream.  Pinned (page-locked) host buffers give asynchronous copies.
 * Errors: as ling_moe_forward, plus DEVICE_TIMEOUT if the call's own device
 * wait gave up. */
int ling_moe_forward_host(ling_moe_t *h, const void *x_host, int T, void *out_host,
                          void *stream);

/* ---- Expert parallel: the layer's experts partitioned over several GPUs.
 * The pages run the model as TP4 + EP4 on four H200s with vLLM's
 * --enable-expert-parallel (vLLM recipe page "inclusionAI/Ling-3.0-flash",
 * section "Launching the Server"); they give no kernel-level definition.
 * Here each GPU (rank) holds the full router and a contiguous range of the
 * routed experts, and one rank also holds the shared expert.  Every rank
 * scores all experts and selects the same top-k with the same weights; it
 * computes only the terms of the selected experts it holds (plus the shared
 * expert where it lives) and returns their sum in fp32.  The sum of all ranks'
 * partial outputs (an all-reduce) rounded once to bf16 (ling_moe_round_bf16)
 * is the layer's output. */
typedef enum { LING_MOE_FORMAT_INT4 = 0, LING_MOE_FORMAT_MXFP4 = 1 } ling_moe_format_t;

typedef struct {
  int expert_begin; /* first expert held here, 0 <= expert_begin */
  int expert_count; /* experts held here, >= 1, expert_begin + expert_count <= num_experts */
  int with_shared;  /* 1: this handle also computes the shared expert; 0: it does not */
  int format;       /* ling_moe_format_t of the routed weights */
} ling_moe_ep_t;

/* An expert-parallel handle.  cfg->num_experts is the number of experts the
 * router scores (all ranks together).  w->router_w [num_experts, H] and
 * w->router_bias [num_experts] are the full router; gate_q / gate_s / up_q /
 * up_s / down_q / down_s hold only the expert_count experts held here, in
 * the layouts of ling_moe_create (int4) or ling_moe_create_mxfp4 (MXFP4)
 * with E = expert_count; sh_gate / sh_up / sh_down are read only when
 * with_shared = 1 (they may be NULL otherwise).  Copies what it needs, as
 * ling_moe_create does.  Such a handle serves ling_moe_forward_partial;
 * ling_moe_forward / _forward_ex / _forward_host return INVALID_ARG on it.
 * Errors: as ling_moe_create; INVALID_ARG for a range outside
 * [0, num_experts), with_shared not 0/1 or an unknown format. */
int ling_moe_create_ep(const ling_moe_config_t *cfg, const ling_moe_weights_t *w,
                       const ling_moe_ep_t *ep, ling_moe_t **out);

/* partial[T, H] (fp32, DEVICE, 16-byte aligned, not overlapping x) = the sum,
 * in fp32, of the routed terms w_e * Wd_e(...) of the selected experts this
 * handle holds (slot order) plus its shared-expert term, before any bf16
 * rounding.  On a handle from ling_moe_create it is the whole layer in fp32.
 * topk_idx / topk_w as in ling_moe_forward_ex: every selected expert, held
 * here or not (global indices).  Same kernels, asynchrony and errors as
 * ling_moe_forward. */
int ling_moe_forward_partial(ling_moe_t *h, const void *x, int T, float *partial,
                             int32_t *topk_idx, float *topk_w, void *stream);

/* out[i] (bf16) = in[i] (fp32) rounded to nearest even, i < n, on `stream`:
 * the one rounding of the layer's output once the ranks' partial sums are
 * added.  DEVICE pointers, 16-byte aligned, not overlapping; n a multiple of
 * 8.  One launch; asynchronous.  Errors: INVALID_ARG, CUDA. */
int ling_moe_round_bf16(const float *in, void *out, size_t n, void *stream);

/* Synchronise `stream` and return the handle's sticky device error
 * (OK or DEVICE_TIMEOUT), or CUDA if the synchronisation itself failed. */
int ling_moe_status(ling_moe_t *h, void *stream);

/* Human-readable description of the active configuration and kernel path
 * (shape, per-path kernels, grid size).  Owned by the handle. */
const char *ling_moe_describe(const ling_moe_t *h);

/* Number of kernel launches this handle has enqueued since creation. */
int64_t ling_moe_launch_count(const ling_moe_t *h);

/* Message of the last error on the calling host thread ("" if none). */
const char *ling_moe_last_error(void);

/* ---- per-kernel timing (measurement; off by default) ----
 * With on != 0, every later forward call also records CUDA events on its
 * stream around each kernel it launches (one for T <= 4, two for 5 <= T <= 8,
 * nine for larger T:
 * route, topk, plan, scatter, gemv_gu, tc_gu, gemv_dn, tc_dn, combine).  The
 * events add a little time of their own; do not leave timing on while
 * capturing a stream into a graph.  on == 0 frees the events.  Returns OK,
 * INVALID_ARG (NULL handle) or CUDA. */
int ling_moe_set_kernel_timing(ling_moe_t *h, int on);
/* Durations in milliseconds of the kernels of the last forward call issued
 * while timing was on, in launch order: waits for that call's last event,
 * writes *count (0 if no call was timed) and ms[0 .. *count).  capacity is
 * the length of ms (at least *count, 9 is always enough).  Returns OK,
 * INVALID_ARG (NULL handle or count, timing off, ms too short) or CUDA. */
int ling_moe_kernel_times(ling_moe_t *h, float *ms, int capacity, int *count);
/* Name of kernel i of the last timed call ("" if there is none).  The
 * string is static. */
const char *ling_moe_kernel_name(const ling_moe_t *h, int i);

/* Free everything the handle owns.  NULL is a no-op.  The caller must make
 * sure no enqueued work still uses the handle. */
void ling_moe_destroy(ling_moe_t *h);

/* ---- test hooks (not needed in normal use) ----
 * skip_arrive_cta >= 0 makes that CTA of the next decode launch withhold the
 * router logits it computes, so that every CTA's bounded wait for them runs
 * out; wait_limit_ns bounds every device-side wait (0 keeps the default, 2 s).
 * Used to test that a wait that runs out ends the launch with an error status
 * (reported by ling_moe_status) instead of hanging, and that the next launch
 * runs normally. */
int ling_moe_test_set_wait(ling_moe_t *h, int skip_arrive_cta, uint64_t wait_limit_ns);

/* ---- routing that allocates nothing ----
 * The pages have no counterpart of this call.  It is for callers that cannot
 * allocate device memory at the point where they route tokens: code running
 * under a framework that owns all device memory through its own pool, or a
 * latency-critical path that must not call cudaMalloc (which can synchronise
 * the device).  It needs no handle.
 *
 * For T tokens x[T, H] (bf16, H = 2560) it computes the router logits
 * x . router_w[E, H]^T (+ router_bias[E]) in fp32, the top_k experts (ties
 * to the lower index) and their renormalised softmax weights, into
 * topk_idx int32 [T, top_k] and topk_w fp32 [T, top_k]: the same values that
 * ling_moe_forward_ex reports for the same router.  All pointers are DEVICE
 * pointers; x and router_w 16-byte aligned, the others 4-byte aligned;
 * router_bias may be NULL.
 * Limits: 0 <= T <= 4, 1 <= num_experts <= 512, 1 <= top_k <= min(8, num_experts);
 * anything else returns LING_MOE_ERR_INVALID_ARG (message in
 * ling_moe_last_error) before anything is launched.
 * Scratch: a static array of 16,640 bytes in device memory (tagged logit
 * slots of 4 x 512 experts, a generation word and an error word) that every
 * GPU which loads the library holds until the process exits.  Nothing is
 * allocated, by this call or on its behalf.  The first call on a device looks
 * up that array's device address (cudaGetSymbolAddress) and keeps it for the
 * life of the process, so make the first call on each device before any
 * stream capture on it, and do not use this call across a device reset
 * (cudaDeviceReset), after which the kept address may be stale.
 * Every call shares the array.  Nothing in it needs to start at zero: each
 * call tags the logits it writes with a fresh tag and reads only slots that
 * carry it, so a call never sees an earlier call's values.  Calls that
 * overlap on the GPU (two streams, or two host threads) race on the array and
 * must not be issued; if they are, their own results are undefined, but the
 * next call on its own is correct again.
 * A device-side wait that runs out (2 s) writes -1 indices and 0 weights and
 * sets a sticky error word, which ling_moe_route_noalloc_status reports. */
int ling_moe_route_noalloc(const void *x, int T, const void *router_w, const float *router_bias,
                           int num_experts, int top_k, int32_t *topk_idx, float *topk_w, void *stream);

/* Synchronises `stream`, then reports whether a ling_moe_route_noalloc call
 * on the current device had a device-side wait run out since the last status
 * call: LING_MOE_ERR_DEVICE_TIMEOUT (and clears the error word) or
 * LING_MOE_OK.  Allocates nothing.  Errors: CUDA. */
int ling_moe_route_noalloc_status(void *stream);

/* Test hook: the next ling_moe_route_noalloc call has CTA skip_cta (-1:
 * none) withhold its logits, so that CTA 0's wait runs out; wait_limit_ns
 * bounds that wait for this and later calls (0 restores 2 s).  Errors:
 * INVALID_ARG (skip_cta >= 512). */
int ling_moe_route_noalloc_test_set_wait(int skip_cta, uint64_t wait_limit_ns);

/* ---- online-FP8 LM head ----
 * Source: bpdata article "Harom optimalizacio a Ling-3.0-flash MoE
 * inferenciajanak", section "Optimalizacio 2: Online FP8 LM head kvantalas":
 * the bf16 LM head (157,184 x 2,560 in Ling-3.0-flash) is quantised to FP8
 * once, when the head is built, so that each decoded token reads about half
 * as many bytes.  The pages do not fix the FP8 format or the scaling; this
 * library takes:
 *   FP8 = e4m3 (no infinities, largest finite 448), round to nearest even,
 *         saturating;
 *   weights: one fp32 scale per vocabulary row, s_w[v] = max_k |W[v,k]| / 448
 *         (1 for an all-zero row), codes e4m3(W[v,k] / s_w[v]);
 *   tokens: the same per token at every call, s_x[t], codes e4m3(x[t,k] / s_x[t]);
 *   both divisions correctly rounded in fp32;
 *   logits[t, v] = (sum_k e4m3(x)[t,k] * e4m3(W)[v,k]) * s_x[t] * s_w[v],
 *         every product exact; tensor cores sum 256 products at a time
 *         (16 per instruction, chained), those sums are accumulated in fp32.
 */
typedef struct ling_moe_lmhead ling_moe_lmhead_t; /* opaque handle */

/* Quantise the head w [vocab, hidden] (bf16, DEVICE, row-major, 16-byte
 * aligned; read only during this call) into library-owned device memory:
 * the codes (vocab rounded up to a multiple of 32, times hidden bytes, in a
 * tiled layout that the GEMV streams in order), vocab fp32 scales, and
 * staging buffers for ling_moe_lmhead_forward_host (8 tokens).
 * Synchronises the device.
 * Limits: vocab >= 1; hidden a multiple of 512, at most 4096.
 * Errors: INVALID_ARG (NULL, misaligned, non-positive sizes), UNSUPPORTED
 * (hidden outside the limits, not an sm_100 GPU), OOM, CUDA.  On failure
 * *out is NULL and nothing leaks. */
int ling_moe_lmhead_create(const void *w, int vocab, int hidden, ling_moe_lmhead_t **out);

/* logits[T, vocab] (fp32, DEVICE, 4-byte aligned, row-major) of the tokens
 * x[T, hidden] (bf16, DEVICE, 16-byte aligned) on `stream`; 0 <= T <= 8
 * (T == 0 enqueues nothing).  logits must not overlap x.  One kernel launch;
 * asynchronous, no allocation, capturable into a CUDA graph.  Device-side
 * failures (a bounded wait that gave up) are reported by
 * ling_moe_lmhead_status.
 * Errors: INVALID_ARG (checked before anything is enqueued), CUDA. */
int ling_moe_lmhead_forward(ling_moe_lmhead_t *h, const void *x, int T, float *logits, void *stream);

/* As ling_moe_lmhead_forward, and also writes the tokens' quantisation:
 * x_codes [T, hidden] e4m3 bytes (16-byte aligned) and x_scales fp32 [T]
 * (DEVICE; either may be NULL; neither may overlap x or logits). */
int ling_moe_lmhead_forward_ex(ling_moe_lmhead_t *h, const void *x, int T, float *logits,
                               uint8_t *x_codes, float *x_scales, void *stream);

/* End-to-end call on HOST buffers: copies x_host [T, hidden] bf16 to the
 * device, runs the head, copies logits [T, vocab] fp32 to logits_host and
 * waits for the stream.  Pinned host buffers give asynchronous copies. */
int ling_moe_lmhead_forward_host(ling_moe_lmhead_t *h, const void *x_host, int T, float *logits_host,
                                 void *stream);

/* The handle's quantised head in row-major order: writes codes [vocab,
 * hidden] (e4m3 bytes, 16-byte aligned) and scales [vocab] (fp32) to the
 * caller's DEVICE buffers on `stream` (asynchronous; one kernel launch,
 * which ling_moe_lmhead_launch_count does not count).  The handle keeps
 * the codes in its own tiled layout; this call is for inspection and tests. */
int ling_moe_lmhead_weights(const ling_moe_lmhead_t *h, uint8_t *codes, float *scales, void *stream);

/* Synchronise `stream` and return the handle's sticky device error: OK, or
 * DEVICE_TIMEOUT if a bounded wait inside the kernel (2 s) gave up (the word
 * is cleared), or CUDA if the synchronisation itself failed. */
int ling_moe_lmhead_status(ling_moe_lmhead_t *h, void *stream);

/* Number of kernel launches the handle's forward calls have enqueued. */
int64_t ling_moe_lmhead_launch_count(const ling_moe_lmhead_t *h);

/* Free everything the handle owns.  NULL is a no-op.  The caller must make
 * sure no enqueued work still uses the handle. */
void ling_moe_lmhead_destroy(ling_moe_lmhead_t *h);

/* Test hook: skip_cta >= 0 makes that CTA of the next forward calls issue
 * none of its weight copies, so that its waits for them run out and the
 * launch ends with an error status (reported by ling_moe_lmhead_status)
 * instead of hanging; -1 turns it off.  wait_limit_ns bounds every
 * device-side wait (0 keeps the default, 2 s). */
int ling_moe_lmhead_test_set_wait(ling_moe_lmhead_t *h, int skip_cta, uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* LING_MOE_H */
