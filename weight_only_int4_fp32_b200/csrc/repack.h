// Create-time repack of the routed weights (int4 or MXFP4) into the kernels'
// unit layouts.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace lingmoe {

// gu must hold E * kGuExpertBytes bytes, dn E * kDnExpertBytes bytes.  All
// source pointers are canonical-layout device pointers, 16-byte aligned;
// the scales are bf16 (kCodecInt4) or E8M0 bytes (kCodecMxfp4).
cudaError_t launch_repack(const uint8_t* gate_q, const uint8_t* up_q, const void* gate_s,
                          const void* up_s, const uint8_t* down_q, const void* down_s, uint8_t* gu,
                          uint8_t* dn, int E, int codec, cudaStream_t stream);

}  // namespace lingmoe
