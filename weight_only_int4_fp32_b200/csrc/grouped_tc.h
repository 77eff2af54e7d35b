// Host-visible interface of the tensor-core (tcgen05) grouped GEMMs.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>  // CUtensorMap (types only; the encoder is fetched at run time)
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "layout.h"

namespace lingmoe {

constexpr int kTcTileM = 256;                  // weight rows per CTA tile
constexpr int kTcTileN = 128;                  // positions per CTA tile (max)
constexpr int kTcMTilesGu = 2 * kI / kTcTileM;  // 6: gate/up rows interleaved
constexpr int kTcMTilesDn = kH / kTcTileM;      // 10
// Routed weights enter the MMA as q * s * 2^kTcScaleShift and h as h *
// 2^-kTcScaleShift, which keeps both inside fp16's normal range for scales in
// [2^-22, 32] and |h| < 2^23.
constexpr int kTcScaleShift = 8;
// A token's x enters as x * 2^-sigma_t with its largest |x| in [2^14, 2^15);
// h and y are kept relative to c_t = 2^(sigma_t + kGrpUnitShift), h as
// h / c_t^2 and y as y / c_t^2, and the combine multiplies by c_t twice.  A
// token whose largest |x| lies in [2, 4) has c_t = 1.  So no intermediate
// grows or shrinks with the token's magnitude: every finite bf16 token keeps
// the same relative precision, and only the final product can overflow
// (to the infinity bf16 rounds the exact result to) or underflow.
constexpr int kGrpUnitShift = 13;

// Tile record: (expert or E for the shared expert, m-tile, first position, positions).
struct TcParams {
  const uint8_t* gu;        // repacked routed gate/up
  const uint8_t* dn;        // repacked routed down
  const float* xscale;      // [T] 2^sigma_t: x16 rows hold x * 2^-sigma_t
  __half* h16;              // [rows, 2, I] (h / c_t^2) * 2^-8 as fp16 hi + lo, natural K order
  float* y;                 // [rows, H] expert output per position / c_t^2, times the routing weight
  const int32_t* perm;      // position (< P) -> pair id t*k + slot
  const float* topk_w;      // [P] routing weight per pair id
  const float* sh_scale;    // [3] 2^-c of the fp16 shared-expert copies (gate, up, down)
  int k, E, P;              // shared-expert tiles carry expert E and positions P + t
  const int4* gu_tiles;
  const int4* dn_tiles;
  const int32_t* ntiles;    // [0] gate/up tiles, [1] down tiles
  unsigned int* err;        // sticky device error word
  const __half* xg;         // the buffers behind the tensor maps (for L2 prefetch)
  int codec;                // kCodecInt4 or kCodecMxfp4 (layout.h)
  const __half* shgu16;
  const __half* shdn16;
};

// TMA descriptors: the B operands (x rows by position, h rows by position)
// and the fp16 copies of the shared expert, all 128-byte swizzled.
struct TcMaps {
  CUtensorMap b_x;     // xg  [rows, H]     box 64 x 32
  CUtensorMap b_h;     // h16 [rows, 2I]    box 64 x 32
  CUtensorMap a_shgu;  // shgu16 [2I, H]    box 64 x 128
  CUtensorMap a_shdn;  // shdn16 [H, I]     box 64 x 128
};

cudaError_t setup_grouped_tc();
cudaError_t tc_encode_maps(TcMaps* m, const __half* xg, const __half* h16, int rows, const __half* shgu16,
                           const __half* shdn16);
// fp16 copies of the shared expert (gate/up in natural K order, 128 gate rows
// then the 128 up rows of the same intermediate rows per block; down in
// natural K order too), each matrix scaled by a power of two 2^c so that max |w| * 2^c
// lies in [2^14, 2^15); sh_scale receives 2^-c.  amax_scratch: 3 words.
cudaError_t launch_tc_prep_shared(const __nv_bfloat16* g, const __nv_bfloat16* u, const __nv_bfloat16* d,
                                  __half* shgu16, __half* shdn16, float* sh_scale, unsigned int* amax_scratch,
                                  cudaStream_t s);
cudaError_t launch_tc_gemm(int mode, const TcMaps& m, const TcParams& p, int nctas, cudaStream_t s);
// upper bound on the number of N-tiles (each expands into kTcMTiles* tiles)
inline size_t tc_max_ntiles(int P, int T, int E) {
  return (size_t)P / kTcTileN + (size_t)E + (size_t)T / kTcTileN + 2;
}

}  // namespace lingmoe
