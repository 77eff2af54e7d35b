// Online-FP8 LM head: the bf16 head [vocab, hidden] quantised at build time
// to e4m3 with one fp32 scale per vocabulary row (codes stored in a tiled
// layout, see lmhead.cu); each call quantises the tokens the same way and
// returns fp32 logits.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace lingmoe {

constexpr int kLmhMaxT = 8;          // tokens per call
constexpr int kLmhMaxHidden = 4096;  // hidden % 512 == 0

// Bytes of the tiled codes (the vocabulary rounded up to whole 32-row tiles).
size_t lmh_codes_bytes(int vocab, int hidden);
// w [vocab, hidden] bf16 -> tiled codes (lmh_codes_bytes), scales [vocab] fp32
cudaError_t launch_lmh_quantize(const __nv_bfloat16* w, int vocab, int hidden, uint8_t* codes, float* scales,
                                cudaStream_t s);
// tiled codes -> row-major codes [vocab, hidden]
cudaError_t launch_lmh_untile(const uint8_t* codes, int vocab, int hidden, uint8_t* out, cudaStream_t s);
// logits [T, vocab] fp32; x_codes / x_scales: optional copies of the tokens'
// codes [T, hidden] and scales [T].  Bounded waits: one that runs out sets
// bit 2 of *err.  skip_cta >= 0 (a test hook) makes that CTA issue no copies.
cudaError_t launch_lmh_forward(const uint8_t* codes, const float* scales, int vocab, int hidden,
                               const __nv_bfloat16* x, int T, float* logits, uint8_t* x_codes, float* x_scales,
                               unsigned int* err, unsigned long long wait_limit_ns, int skip_cta, int nctas,
                               cudaStream_t s);
cudaError_t setup_lmhead();

}  // namespace lingmoe
