// Host-visible interface of the tensor-core (tcgen05) grouped GEMMs.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace lingmoe {

struct TcParams {
  const uint8_t* gu;        // repacked routed gate/up
  const uint8_t* dn;        // repacked routed down
  const __half* x16;        // [T, H] fp16, permuted K order, scaled by 1/xscale
  const float* xscale;      // [T]
  __half* h16;              // [positions, 2, I] fp16 hi and lo terms, permuted K order
  float* y;                 // [positions, H] fp32, weighted by the routing weight
  const int32_t* perm;      // position -> pair id (t*k + slot)
  const float* topk_w;      // [pairs]
  int k;
  const int4* gu_tiles;     // (expert, m-tile, first position, tokens)
  const int4* dn_tiles;
  const int32_t* ntiles;    // [0] gate/up tiles, [1] down tiles
  unsigned int* err;        // sticky device error word
};

size_t tc_smem_bytes();
cudaError_t setup_grouped_tc();
cudaError_t launch_x16(const __nv_bfloat16* x, int T, __half* x16, float* xscale, cudaStream_t s);
cudaError_t launch_tc_tiles(const int32_t* cnt, const int32_t* off, int E, int4* gu_tiles, int4* dn_tiles,
                            int32_t* ntiles, cudaStream_t s);
cudaError_t launch_tc_gemm(int mode, const TcParams& p, int nctas, cudaStream_t s);
// upper bounds on the tile counts for P token-expert pairs over E experts
inline size_t tc_max_tiles_gu(int P, int E) { return ((size_t)P / 128 + (size_t)E + 1) * 12; }
inline size_t tc_max_tiles_dn(int P, int E) { return ((size_t)P / 128 + (size_t)E + 1) * 20; }

}  // namespace lingmoe
