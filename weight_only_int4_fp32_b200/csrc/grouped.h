// Host-visible interface of the token-grouped path (T > kMaxDecodeT).
#pragma once

#include <cstddef>
#include <cstdint>
#include <functional>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "grouped_tc.h"

namespace lingmoe {

struct GroupedParams {
  const __nv_bfloat16* x;        // [T, H]
  __nv_bfloat16* out;            // [T, H]
  int T, E, k;
  const __nv_bfloat16* router_w; // [E, H]
  const float* router_bias;      // [E] or nullptr
  const uint8_t* gu;             // repacked routed gate/up
  const uint8_t* dn;             // repacked routed down
  int32_t* topk_idx_out;         // optional [T, k]
  float* topk_w_out;             // optional [T, k]
  int num_sms;
  int codec;                     // kCodecInt4 or kCodecMxfp4 (layout.h)
  // Expert parallel (as DecodeParams): gu / dn hold experts [e0, e0 + e_local)
  // of the E the router scores; shared_on = 0 leaves the shared expert out;
  // out_f32 != nullptr takes the fp32 sum instead of the bf16 out.
  int e0, e_local;
  int shared_on;
  float* out_f32;
};

// Positions: the T*k token-expert pairs sorted by expert occupy positions
// [0, T*k); the shared expert's rows are positions T*k + t.
struct GroupedWorkspace {
  int max_T = 0;
  size_t rows = 0;              // max_T * (k + 1) positions
  float* logits = nullptr;      // [T, E] router logits
  int32_t* topk_idx = nullptr;  // [T*k]
  float* topk_w = nullptr;      // [T*k]
  int32_t* cnt = nullptr;       // [E] pairs per expert (left at zero after each call)
  int32_t* fill = nullptr;      // [E] scatter cursors (left at zero after each call)
  int32_t* off = nullptr;       // [E+1] first position of each expert
  int32_t* perm = nullptr;      // [T*k] position -> pair id t*k + slot
  int32_t* inv = nullptr;       // [T*k] pair id -> position
  float* xscale = nullptr;      // [T] 2^sigma_t
  __half* xg = nullptr;         // [rows, H]  x * 2^-sigma_t in fp16 by position (tensor-core B operand)
  __half* h16 = nullptr;        // [rows, 2, I] SiLU(gate)*up * 2^-8 by position, fp16 hi + lo
  float* y = nullptr;           // [rows, H] expert output by position (routed ones weighted)
  __half* shgu16 = nullptr;     // [2I, H] shared gate/up in fp16, rows interleaved, scaled
  __half* shdn16 = nullptr;     // [H, I]  shared down in fp16, scaled
  float* sh_scale = nullptr;    // [3] undo factors of those scales
  unsigned int* amax = nullptr; // [3] scratch of the shared-expert preparation
  int4* gu_tiles = nullptr;     // tcgen05 tile lists
  int4* dn_tiles = nullptr;
  int32_t* ntiles = nullptr;    // [2]
  int4* small = nullptr;        // [E] experts for the GEMV kernels: (expert, first position, tokens, 0)
  int32_t* nsmall = nullptr;    // [1] entries in small
  TcMaps maps{};
  unsigned int* err = nullptr;  // the handle's sticky device error word
};

using AllocFn = std::function<cudaError_t(void**, size_t)>;
cudaError_t grouped_alloc(GroupedWorkspace* ws, int E, int k, int max_T, const AllocFn& alloc);
// One-time preparation at create: fp16 shared-expert copies, tensor maps and
// zeroed counters.  Enqueued on `stream`.
cudaError_t grouped_prepare(GroupedWorkspace* ws, int E, const __nv_bfloat16* sh_gate, const __nv_bfloat16* sh_up,
                            const __nv_bfloat16* sh_down, cudaStream_t stream);
cudaError_t setup_grouped();
const char* grouped_describe();
// Enqueues the grouped path; *nlaunch receives the number of kernels launched.
// marks: optional, kGroupedKernels + 1 events; marks[i] is recorded just
// before kernel i of the sequence below and marks[kGroupedKernels] after the
// last one (per-kernel timing; nullptr records nothing).
constexpr int kGroupedKernels = 9;  // route, topk, plan, scatter, gemv_gu, tc_gu, gemv_dn, tc_dn, combine
cudaError_t launch_grouped(const GroupedParams& p, const GroupedWorkspace& ws, cudaStream_t stream,
                           int* nlaunch, cudaEvent_t* marks = nullptr);

}  // namespace lingmoe
