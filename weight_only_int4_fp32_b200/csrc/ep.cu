// Expert parallel: each rank computes the fp32 sum of the routed terms of the
// experts it holds (and, on one rank, the shared expert) with the ordinary
// kernels (DecodeParams / GroupedParams e0, e_local, shared_on, out_f32); the
// ranks' partial sums are added by an all-reduce, and this kernel rounds the
// total once to bf16.  Partitioning and the exchange: the vLLM recipe page
// "inclusionAI/Ling-3.0-flash", section "Launching the Server" (TP4 + EP4 with
// --enable-expert-parallel).
#include "ep.h"

namespace lingmoe {

// 8 values per thread: two 16-byte loads, one 16-byte store; a grid of 148 x
// 4 CTAs strides over the array (the launch size does not depend on n).
__global__ void __launch_bounds__(256) round_bf16_kernel(const float4* __restrict__ in, uint4* __restrict__ out,
                                                         size_t n8) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const float4 a = __ldcs(in + 2 * i), b = __ldcs(in + 2 * i + 1);
    __nv_bfloat162 r[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                           __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
    out[i] = *reinterpret_cast<const uint4*>(r);
  }
}

cudaError_t launch_round_bf16(const float* in, __nv_bfloat16* out, size_t n, cudaStream_t stream) {
  const size_t n8 = n / 8;
  const size_t blocks = (n8 + 255) / 256;
  round_bf16_kernel<<<(unsigned)(blocks < 592 ? blocks : 592), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(in), reinterpret_cast<uint4*>(out), n8);
  return cudaGetLastError();
}

}  // namespace lingmoe
