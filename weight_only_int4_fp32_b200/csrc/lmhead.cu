// Online-FP8 LM head (hidden -> vocabulary): bf16 weights quantised once, at
// build time, to e4m3 with one fp32 scale per vocabulary row; per call the
// tokens are quantised the same way and every logit is the scaled sum of
// exact e4m3 x e4m3 products, accumulated in fp32.
//
// Quantisation of a row (or token): scale = max|v| / 448 (1 for an all-zero
// row), code = e4m3(v / scale), both divisions correctly rounded in fp32,
// the conversion round-to-nearest-even and saturating (cvt.rn.satfinite).
//
// The GEMV streams the 157,184 x 2,560 codes (402 MB per call) once: a warp
// takes two rows at a time, each lane 16 consecutive codes per 512-byte
// column block with 128-bit non-caching loads, so that ~10 loads per lane
// are in flight.  The codes become fp16 pairs (exact), multiply the tokens'
// fp16 codes with mixed-precision FMAs (exact products, fp32 sums) and a
// warp-shuffle reduction ends each row.
//
// Source: bpdata article "Harom optimalizacio a Ling-3.0-flash MoE
// inferenciajanak", section "Optimalizacio 2: Online FP8 LM head kvantalas"
// (157,184 x 2,560 head quantised dynamically to FP8 when the head is built;
// roughly half the bytes of the bf16 head).
#include "common.cuh"
#include "lmhead.h"

namespace lingmoe {

constexpr int kLmhWarps = 16;
constexpr int kLmhThreads = kLmhWarps * 32;
constexpr int kLmhMaxChunks = kLmhMaxHidden / 512;

// two floats -> two e4m3 codes; v0 in the low byte (the lower K index)
__device__ __forceinline__ uint32_t e4m3x2(float v0, float v1) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(v1), "f"(v0));
  return r;
}
// two e4m3 codes (a 16-bit pair) -> the same two values as fp16 (exact)
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t pair) {
  uint32_t r;
  const unsigned short p = (unsigned short)pair;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(p));
  return r;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float fma_f16h_lo(uint32_t a, uint32_t b, float c) {
  float d;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fma_f16h_hi(uint32_t a, uint32_t b, float c) {
  float d;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, ah, bh, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
  return d;
}

// One warp quantises one row of n values (n % 256 == 0): codes and scale.
// Every lane takes 8 consecutive values per step of 256.
__device__ __forceinline__ void quantize_row_warp(const __nv_bfloat16* src, int n, uint8_t* codes, float* scale) {
  const int lane = threadIdx.x & 31;
  float amax = 0.f;
  for (int c = lane; c < n / 8; c += 32) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + 8 * c);
    amax = fmaxf(amax, fmaxf(fmaxf(fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x))),
                                   fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y)))),
                             fmaxf(fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))),
                                   fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w))))));
  }
  amax = warp_max(amax);
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  for (int c = lane; c < n / 8; c += 32) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + 8 * c);
    const uint32_t lo = e4m3x2(__fdiv_rn(bf16lo(v.x), s), __fdiv_rn(bf16hi(v.x), s)) |
                        e4m3x2(__fdiv_rn(bf16lo(v.y), s), __fdiv_rn(bf16hi(v.y), s)) << 16;
    const uint32_t hi = e4m3x2(__fdiv_rn(bf16lo(v.z), s), __fdiv_rn(bf16hi(v.z), s)) |
                        e4m3x2(__fdiv_rn(bf16lo(v.w), s), __fdiv_rn(bf16hi(v.w), s)) << 16;
    *reinterpret_cast<uint2*>(codes + 8 * c) = make_uint2(lo, hi);
  }
  if (lane == 0) *scale = s;
}

__global__ void __launch_bounds__(256) lmh_quantize_kernel(const __nv_bfloat16* __restrict__ w, int vocab,
                                                           int hidden, uint8_t* __restrict__ codes,
                                                           float* __restrict__ scales) {
  const int warps = blockDim.x / 32;
  for (long long r = (long long)blockIdx.x * warps + (threadIdx.x >> 5); r < vocab; r += (long long)gridDim.x * warps)
    quantize_row_warp(w + r * hidden, hidden, codes + r * hidden, scales + r);
}

// Persistent GEMV: every CTA quantises the T tokens into shared memory
// (fp16 copies of their codes, and their scales), then its warps stream
// rows r = warp id + k * (all warps), R at a time (R = 2 up to 4 tokens, 1
// above, which keeps the loads and the accumulators within 128 registers).
template <int T, int R>
__global__ void __launch_bounds__(kLmhThreads, 1)
lmh_gemv_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ scales, int vocab, int hidden,
                const __nv_bfloat16* __restrict__ x, float* __restrict__ logits, uint8_t* x_codes, float* x_scales) {
  extern __shared__ __align__(16) unsigned char lsm[];
  __half* xh = reinterpret_cast<__half*>(lsm);                       // [T][hidden]
  float* xs = reinterpret_cast<float*>(lsm + (size_t)T * hidden * 2);  // [T]
  uint8_t* xq = lsm + (size_t)T * hidden * 2 + 64;                    // [T][hidden] codes
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (warp < T) quantize_row_warp(x + (size_t)warp * hidden, hidden, xq + (size_t)warp * hidden, &xs[warp]);
  __syncthreads();
  for (int i = tid; i < T * hidden / 2; i += kLmhThreads) {
    const uint32_t pair = *reinterpret_cast<const unsigned short*>(xq + 2 * i);
    *reinterpret_cast<uint32_t*>(xh + 2 * i) = e4m3x2_to_f16x2(pair);
  }
  if (blockIdx.x == 0 && x_codes != nullptr)
    for (int i = tid; i < T * hidden / 16; i += kLmhThreads)
      reinterpret_cast<uint4*>(x_codes)[i] = reinterpret_cast<const uint4*>(xq)[i];
  if (blockIdx.x == 0 && x_scales != nullptr && tid < T) x_scales[tid] = xs[tid];
  __syncthreads();

  const int nc = hidden / 512;
  const long long nw = (long long)gridDim.x * kLmhWarps;
#pragma unroll 1
  for (long long rb = (long long)blockIdx.x * kLmhWarps + warp; rb < vocab; rb += R * nw) {
    long long row[R];
    bool has[R];
#pragma unroll
    for (int j = 0; j < R; ++j) {
      row[j] = rb + j * nw;
      has[j] = row[j] < vocab;
    }
    uint4 w[R][kLmhMaxChunks];
#pragma unroll
    for (int c = 0; c < kLmhMaxChunks; ++c)
      if (c < nc)
#pragma unroll
        for (int j = 0; j < R; ++j)
          w[j][c] = has[j] ? ldg_stream(codes + row[j] * hidden + 512 * c + 16 * lane) : make_uint4(0, 0, 0, 0);
    float a[R][T], b[R][T];
#pragma unroll
    for (int j = 0; j < R; ++j)
#pragma unroll
      for (int t = 0; t < T; ++t) a[j][t] = b[j][t] = 0.f;
#pragma unroll
    for (int c = 0; c < kLmhMaxChunks; ++c) {
      if (c < nc) {
        // the 16 codes of each row as 8 fp16 pairs (element order kept)
        uint32_t f[R][8];
#pragma unroll
        for (int j = 0; j < R; ++j) {
          const uint32_t p[4] = {w[j][c].x, w[j][c].y, w[j][c].z, w[j][c].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            f[j][2 * q] = e4m3x2_to_f16x2(p[q]);
            f[j][2 * q + 1] = e4m3x2_to_f16x2(p[q] >> 16);
          }
        }
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const uint4* xv = reinterpret_cast<const uint4*>(xh + (size_t)t * hidden + 512 * c + 16 * lane);
          const uint4 xa = xv[0], xb = xv[1];
          const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
          for (int q = 0; q < 8; ++q)
#pragma unroll
            for (int j = 0; j < R; ++j) {
              a[j][t] = fma_f16h_lo(f[j][q], xw[q], a[j][t]);
              b[j][t] = fma_f16h_hi(f[j][q], xw[q], b[j][t]);
            }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const float sw = has[j] ? scales[row[j]] : 0.f;
#pragma unroll
      for (int t = 0; t < T; ++t) {
        const float v = warp_sum(a[j][t] + b[j][t]);
        if (lane == 0 && has[j]) logits[(size_t)t * vocab + row[j]] = v * xs[t] * sw;
      }
    }
  }
}

template <int T>
constexpr int lmh_rows() { return T <= 4 ? 2 : 1; }

static size_t lmh_smem(int T, int hidden) { return (size_t)T * hidden * 3 + 64; }

cudaError_t setup_lmhead() {
  cudaError_t e = cudaSuccess;
  const int smax = (int)lmh_smem(kLmhMaxT, kLmhMaxHidden);
#define LMH_SETUP(TT) \
  if ((e = cudaFuncSetAttribute(lmh_gemv_kernel<TT, lmh_rows<TT>()>, cudaFuncAttributeMaxDynamicSharedMemorySize, smax)) != cudaSuccess) \
    return e;
  LMH_SETUP(1) LMH_SETUP(2) LMH_SETUP(3) LMH_SETUP(4) LMH_SETUP(5) LMH_SETUP(6) LMH_SETUP(7) LMH_SETUP(8)
#undef LMH_SETUP
  return e;
}

cudaError_t launch_lmh_quantize(const __nv_bfloat16* w, int vocab, int hidden, uint8_t* codes, float* scales,
                                cudaStream_t s) {
  lmh_quantize_kernel<<<4 * 148, 256, 0, s>>>(w, vocab, hidden, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_lmh_forward(const uint8_t* codes, const float* scales, int vocab, int hidden,
                               const __nv_bfloat16* x, int T, float* logits, uint8_t* x_codes, float* x_scales,
                               int nctas, cudaStream_t s) {
  const size_t smem = lmh_smem(T, hidden);
  switch (T) {
#define LMH_CASE(TT) \
  case TT: lmh_gemv_kernel<TT, lmh_rows<TT>()><<<nctas, kLmhThreads, smem, s>>>(codes, scales, vocab, hidden, x, logits, x_codes, x_scales); break;
    LMH_CASE(1) LMH_CASE(2) LMH_CASE(3) LMH_CASE(4) LMH_CASE(5) LMH_CASE(6) LMH_CASE(7) LMH_CASE(8)
#undef LMH_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace lingmoe
