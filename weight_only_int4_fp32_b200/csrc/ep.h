// Expert parallel: the last step of the combine (host-visible interface).
#pragma once

#include <cstddef>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace lingmoe {

// out[i] = bf16 round-to-nearest-even of in[i], i < n (n a multiple of 8,
// both pointers 16-byte aligned): the one rounding of the layer's output
// after the ranks' fp32 partial sums have been added.
cudaError_t launch_round_bf16(const float* in, __nv_bfloat16* out, size_t n, cudaStream_t stream);

}  // namespace lingmoe
