// Host-visible interface of the token-grouped path (T > kMaxDecodeT).
#pragma once

#include <cstddef>
#include <cstdint>
#include <functional>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace lingmoe {

struct GroupedParams {
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
  int32_t* topk_idx_out;         // optional [T, k]
  float* topk_w_out;             // optional [T, k]
  int num_sms;
};

struct GroupedWorkspace {
  int max_T = 0;
  float* logits = nullptr;   // [T, E]
  int32_t* topk_idx = nullptr;  // [T*k]
  float* topk_w = nullptr;      // [T*k]
  int32_t* cnt = nullptr;       // [E]   tokens per expert
  int32_t* off = nullptr;       // [E+1] start of each expert's run in perm
  int32_t* tile_off = nullptr;  // [E+1] first token tile of each expert
  int32_t* perm = nullptr;      // [T*k] pair ids (t*k+slot) sorted by (expert, pair id)
  int32_t* inv = nullptr;       // [T*k] pair id -> position in perm
  float* y = nullptr;           // [T*k, H] routed expert output per position, weighted
  float* hs = nullptr;          // [T, I]   shared SiLU(gate)*up
  __half* x16 = nullptr;        // [T, H]   x in fp16 (tensor-core B operand)
  float* xscale = nullptr;      // [T]
  __half* h16 = nullptr;        // [T*k, 2, I] SiLU(gate)*up per position, fp16 hi + lo
  int4* gu_tiles = nullptr;     // tcgen05 tile lists
  int4* dn_tiles = nullptr;
  int32_t* ntiles = nullptr;    // [2]
  unsigned int* err = nullptr;  // the handle's sticky device error word
};

using AllocFn = std::function<cudaError_t(void**, size_t)>;
cudaError_t grouped_alloc(GroupedWorkspace* ws, int E, int k, int max_T, const AllocFn& alloc);
cudaError_t setup_grouped();
const char* grouped_describe();
// Enqueues the grouped path; *nlaunch receives the number of kernels launched.
cudaError_t launch_grouped(const GroupedParams& p, const GroupedWorkspace& ws, cudaStream_t stream,
                           int* nlaunch);

}  // namespace lingmoe
