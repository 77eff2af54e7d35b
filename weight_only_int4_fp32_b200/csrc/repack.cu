// Create-time repack of the routed weights from the canonical boundary
// layout (4-bit codes, low nibble = even K, row-major [rows, K/2], one scale
// per 32 K [rows, K/32]) into the unit layouts the kernels stream, regrouped
// into the MMA-fragment words of layout.h.
//   int4: two's-complement codes become offset-binary (q + 8) by flipping the
//         top bit of every nibble; the bf16 scales are copied.
//   MXFP4: the E2M1 codes are kept; each E8M0 scale byte e becomes the bf16
//         2^(e - 113) = 2^(e - 127) * 2^14 (exponents above 240, whose
//         scales would not fit, become NaN).
#include "common.cuh"
#include "repack.h"

namespace lingmoe {

// gate/up: one thread per 32-bit fragment word and per (group, row pair)
// scale slot.  A word gathers two bytes of the gate row and two of the up row
// (each byte: K even in the low nibble, K odd in the high one).
__device__ __forceinline__ uint32_t nib(uint32_t byte, int hi) { return (byte >> (4 * hi)) & 0xFu; }
// the stored bf16 scale of element `i` of a scale array in the codec's format
__device__ __forceinline__ uint32_t scale_bits(const void* s, long long i, int codec) {
  if (codec == kCodecInt4) return static_cast<const uint16_t*>(s)[i];
  const uint32_t e = static_cast<const uint8_t*>(s)[i];
  return e <= 240 ? (e + 14) << 7 : 0x7FC0u;  // bf16: exponent field e - 113 + 127, mantissa 0
}
__global__ void repack_gu_kernel(const uint8_t* __restrict__ gate_q, const uint8_t* __restrict__ up_q,
                                 const void* __restrict__ gate_s, const void* __restrict__ up_s,
                                 uint8_t* __restrict__ gu, int E, int codec) {
  const uint32_t flip = codec == kCodecInt4 ? 0x88888888u : 0u;
  constexpr int kBlocks = kH / 16;                    // K blocks per row
  const long long nword = (long long)E * kGuUnits * kBlocks * 32;
  const long long nscale = (long long)E * kGuUnits * (kH / kGroup) * 8;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < nword + nscale;
       g += (long long)gridDim.x * blockDim.x) {
    if (g < nword) {
      const int t = (int)(g & 31);
      const long long rest = g >> 5;
      const int kb = (int)(rest % kBlocks);
      const long long eu = rest / kBlocks;            // e * kGuUnits + b
      const int b = (int)(eu % kGuUnits);
      const long long e = eu / kGuUnits;
      const int i = 8 * b + (t >> 2);
      const int c = 16 * kb + 2 * (t & 3);
      const uint8_t* gr = gate_q + (e * kI + i) * (kH / 2);
      const uint8_t* ur = up_q + (e * kI + i) * (kH / 2);
      const uint32_t g0 = gr[c / 2], g1 = gr[(c + 8) / 2], u0 = ur[c / 2], u1 = ur[(c + 8) / 2];
      uint32_t w = nib(g0, 0) | nib(g1, 0) << 4 | nib(u0, 0) << 8 | nib(u1, 0) << 12 |
                   nib(g0, 1) << 16 | nib(g1, 1) << 20 | nib(u0, 1) << 24 | nib(u1, 1) << 28;
      w ^= flip;  // int4: two's complement -> offset binary
      const int j = kb >> 2, wi = kb & 3;
      *reinterpret_cast<uint32_t*>(gu + eu * kGuUnitBytes + j * 512 + 16 * t + 4 * wi) = w;
    } else {
      const long long g2 = g - nword;
      const int r8 = (int)(g2 & 7);
      const long long rest = g2 >> 3;
      const int grp = (int)(rest % (kH / kGroup));
      const long long eu = rest / (kH / kGroup);
      const int b = (int)(eu % kGuUnits);
      const long long e = eu / kGuUnits;
      const int i = 8 * b + r8;
      const uint32_t sg = scale_bits(gate_s, (e * kI + i) * (kH / kGroup) + grp, codec);
      const uint32_t su = scale_bits(up_s, (e * kI + i) * (kH / kGroup) + grp, codec);
      *reinterpret_cast<uint32_t*>(gu + eu * kGuUnitBytes + kGuScaleOff + grp * 32 + 4 * r8) = sg | (su << 16);
    }
  }
}

// down: one thread per 32-bit fragment word and per (group, row pair) scale
// word.  A word gathers four bytes of one row: K = 32G + c (+1), c + 8 (+9),
// c + 16 (+17), c + 24 (+25).
__global__ void repack_dn_kernel(const uint8_t* __restrict__ down_q, const void* __restrict__ down_s,
                                 uint8_t* __restrict__ dn, int E, int codec) {
  const uint32_t flip = codec == kCodecInt4 ? 0x88888888u : 0u;
  constexpr int kGroups = kI / kGroup;                // 24
  const long long nword = (long long)E * kDnUnits * kGroups * 32;
  const long long nscale = (long long)E * kDnUnits * kGroups * 4;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < nword + nscale;
       g += (long long)gridDim.x * blockDim.x) {
    if (g < nword) {
      const int t = (int)(g & 31);
      const long long rest = g >> 5;
      const int G = (int)(rest % kGroups);
      const long long ev = rest / kGroups;            // e * kDnUnits + v
      const int v = (int)(ev % kDnUnits);
      const long long e = ev / kDnUnits;
      const int n = kDnUnitRows * v + (t >> 2);
      const int c = kGroup * G + 2 * (t & 3);
      const uint8_t* row = down_q + (e * kH + n) * (kI / 2);
      const uint32_t b0 = row[c / 2], b1 = row[(c + 8) / 2], b2 = row[(c + 16) / 2], b3 = row[(c + 24) / 2];
      uint32_t w = nib(b0, 0) | nib(b1, 0) << 4 | nib(b2, 0) << 8 | nib(b3, 0) << 12 |
                   nib(b0, 1) << 16 | nib(b1, 1) << 20 | nib(b2, 1) << 24 | nib(b3, 1) << 28;
      w ^= flip;  // int4: two's complement -> offset binary
      *reinterpret_cast<uint32_t*>(dn + ev * kDnUnitBytes + (G >> 2) * 512 + 16 * t + 4 * (G & 3)) = w;
    } else {
      const long long g2 = g - nword;
      const int cp = (int)(g2 & 3);
      const long long rest = g2 >> 2;
      const int G = (int)(rest % kGroups);
      const long long ev = rest / kGroups;
      const int v = (int)(ev % kDnUnits);
      const long long e = ev / kDnUnits;
      const int n = kDnUnitRows * v + 2 * cp;
      const uint32_t s0 = scale_bits(down_s, (e * kH + n) * kGroups + G, codec);
      const uint32_t s1 = scale_bits(down_s, (e * kH + n + 1) * kGroups + G, codec);
      *reinterpret_cast<uint32_t*>(dn + ev * kDnUnitBytes + kDnScaleOff + (G >> 2) * 64 + 16 * cp + 4 * (G & 3)) =
          s0 | (s1 << 16);
    }
  }
}

cudaError_t launch_repack(const uint8_t* gate_q, const uint8_t* up_q, const void* gate_s,
                          const void* up_s, const uint8_t* down_q, const void* down_s, uint8_t* gu,
                          uint8_t* dn, int E, int codec, cudaStream_t stream) {
  const int threads = 256, blocks = 4096;
  repack_gu_kernel<<<blocks, threads, 0, stream>>>(gate_q, up_q, gate_s, up_s, gu, E, codec);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  repack_dn_kernel<<<blocks, threads, 0, stream>>>(down_q, down_s, dn, E, codec);
  return cudaGetLastError();
}

}  // namespace lingmoe
