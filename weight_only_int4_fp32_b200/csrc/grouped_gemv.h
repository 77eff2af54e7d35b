// Host-visible interface of the grouped path's GEMV kernels: routed experts
// that hold at most kGvMaxTok tokens of the call (too few for a dense tile).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "layout.h"

namespace lingmoe {

constexpr int kGvMaxTok = 8;   // experts with 1..8 tokens take the GEMV kernels (one MMA column group)

struct GvParams {
  const uint8_t* gu;            // repacked routed gate/up (MMA-fragment units)
  const uint8_t* dn;            // repacked routed down
  const __half* xg;             // [rows, H] x * 2^-sigma_t in fp16 by position, natural K order
  const float* xscale;          // [T] 2^sigma_t
  const int32_t* perm;          // position -> pair id t*k + slot
  const float* topk_w;          // [P] routing weight per pair id
  int k;
  __half* h16;                  // [rows, 2, I] (h / c_t^2) * 2^-8 as fp16 hi + lo, natural K order (written here)
  float* y;                     // [rows, H] routed output per position / c_t^2, times the routing weight
  const int4* small;            // [E] (expert, first position, tokens, 0)
  const int32_t* nsmall;        // number of entries in small
  unsigned int* err;            // sticky device error word
  unsigned long long wait_limit_ns;
  int codec;                    // kCodecInt4 or kCodecMxfp4 (layout.h)
};

cudaError_t setup_grouped_gemv();
// gate/up + SiLU*up (writes h16 for the small experts' positions), then down
// (writes y for those positions); both loop over tasks with `nctas` CTAs
cudaError_t launch_gemv_gu(const GvParams& p, int nctas, cudaStream_t s);
cudaError_t launch_gemv_dn(const GvParams& p, int nctas, cudaStream_t s);

}  // namespace lingmoe
