// Host-visible interface of the decode / verify kernel (1 <= T <= kMaxDecodeT),
// one launch per call for up to 8 tokens (a verify window of 8).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lingmoe {

constexpr int kMaxDecodeT = 8;     // tokens per call handled by the decode kernel
constexpr int kDecodeWarps = 12;
constexpr int kDecodeThreads = kDecodeWarps * 32;

// Values exchanged between CTAs inside one launch are published through
// arrival counters: a producer stores its values, fences, and adds 1 to the
// counter of its kind; a consumer polls the counter (bounded) until all
// producers of the launch have arrived, then reads the values once.  The last
// CTA to finish resets the counters for the next launch.
struct DecodeParams {
  const __nv_bfloat16* x;        // [T, H]
  __nv_bfloat16* out;            // [T, H]
  int T, E, k;
  const __nv_bfloat16* router_w; // [E, H]
  const float* router_bias;      // [E] or nullptr
  const uint8_t* gu;             // repacked routed gate/up
  const uint8_t* dn;             // repacked routed down
  const __nv_bfloat16* sh_gate;  // [I, H]
  const __nv_bfloat16* sh_up;    // [I, H]
  const __nv_bfloat16* sh_down;  // [H, I]
  float* logits;                 // workspace [T, E]
  float* h_s;                    // workspace [T, I]
  float* h_pair;                 // workspace [T*k, I]
  int32_t* topk_idx_out;         // optional caller output [T, k]
  float* topk_w_out;             // optional caller output [T, k]
  unsigned long long* sync;      // monotonic: [0] router rows, [1] shared rows, [2] CTAs past the
                                 // routed gate/up, [3] CTAs done (launch index x CTAs)
  unsigned int* err;             // sticky device error word
  int skip_arrive_cta;           // test hook: this CTA withholds its router rows (-1: none)
  unsigned long long wait_limit_ns;
  int codec;                     // kCodecInt4 or kCodecMxfp4 (common.cuh): how gu / dn codes decode
  // Expert parallel: gu / dn hold experts [e0, e0 + e_local) of the E the
  // router scores; the selection and its weights still run over all E, only
  // the local experts' terms are computed.  shared_on = 0 leaves the shared
  // expert out (its weights are not read).  out_f32 != nullptr: the sum of the
  // computed terms goes there in fp32 (times s_t^2) instead of a bf16 out.
  int e0, e_local;
  int shared_on;
  float* out_f32;                // [T, H] or nullptr
};

size_t decode_smem_bytes(int T);
cudaError_t setup_decode();
int decode_max_ctas_per_sm();
cudaError_t launch_decode(const DecodeParams& p, int nctas, cudaStream_t stream);

}  // namespace lingmoe
