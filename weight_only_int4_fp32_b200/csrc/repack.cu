// Create-time repack of the routed int4 weights from the canonical boundary
// layout (two's-complement nibbles, low nibble = even K, row-major [rows, K/2],
// bf16 scales [rows, K/32]) into the unit layouts the kernels stream.
// The codes become offset-binary (q + 8) by flipping the top bit of every
// nibble; nothing else about a 16-byte group changes.
#include "common.cuh"
#include "repack.h"

namespace lingmoe {

__device__ __forceinline__ uint4 flip_sign_nibbles(uint4 v) {
  v.x ^= 0x88888888u;
  v.y ^= 0x88888888u;
  v.z ^= 0x88888888u;
  v.w ^= 0x88888888u;
  return v;
}

// gate/up: one thread per 16-byte chunk slot and per 8-byte scale slot.
__global__ void repack_gu_kernel(const uint8_t* __restrict__ gate_q, const uint8_t* __restrict__ up_q,
                                 const uint16_t* __restrict__ gate_s, const uint16_t* __restrict__ up_s,
                                 uint8_t* __restrict__ gu, int E) {
  const long long nchunk = (long long)E * kGuUnits * kGuChunks * 32;
  const long long nscale = (long long)E * kGuUnits * (kGuChunks / 4) * 32;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < nchunk + nscale;
       g += (long long)gridDim.x * blockDim.x) {
    if (g < nchunk) {
      const int lane = (int)(g & 31);
      const long long rest = g >> 5;
      const int j = (int)(rest % kGuChunks);
      const long long eu = rest / kGuChunks;  // e * kGuUnits + b
      const int b = (int)(eu % kGuUnits);
      const long long e = eu / kGuUnits;
      const int r = lane & 7, q = lane >> 3;
      const int row = 4 * b + (r & 3);
      const int G = q * kGuChunks + j;
      const uint8_t* src = (r < 4 ? gate_q : up_q) + ((e * kI + row) * (kH / 2) + 16 * G);
      const uint4 v = *reinterpret_cast<const uint4*>(src);
      *reinterpret_cast<uint4*>(gu + eu * kGuUnitBytes + j * 512 + 16 * lane) = flip_sign_nibbles(v);
    } else {
      const long long g2 = g - nchunk;
      const int lane = (int)(g2 & 31);
      const long long rest = g2 >> 5;
      const int bb = (int)(rest % (kGuChunks / 4));
      const long long eu = rest / (kGuChunks / 4);
      const int b = (int)(eu % kGuUnits);
      const long long e = eu / kGuUnits;
      const int r = lane & 7, q = lane >> 3;
      const int row = 4 * b + (r & 3);
      const int G = q * kGuChunks + 4 * bb;
      const uint16_t* src = (r < 4 ? gate_s : up_s) + ((e * kI + row) * (kH / kGroup) + G);
      const uint2 v = *reinterpret_cast<const uint2*>(src);
      *reinterpret_cast<uint2*>(gu + eu * kGuUnitBytes + kGuScaleOff + bb * 256 + 8 * lane) = v;
    }
  }
}

// down: one thread per 16-byte chunk slot and per 2-byte scale slot.
__global__ void repack_dn_kernel(const uint8_t* __restrict__ down_q, const uint16_t* __restrict__ down_s,
                                 uint8_t* __restrict__ dn, int E) {
  const long long nslot = (long long)E * kDnUnits * kDnChunks * 32;
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < 2 * nslot;
       g += (long long)gridDim.x * blockDim.x) {
    const bool is_scale = g >= nslot;
    const long long g1 = is_scale ? g - nslot : g;
    const int lane = (int)(g1 & 31);
    const long long rest = g1 >> 5;
    const int j = (int)(rest % kDnChunks);
    const long long ev = rest / kDnChunks;  // e * kDnUnits + v
    const int v = (int)(ev % kDnUnits);
    const long long e = ev / kDnUnits;
    const int r = lane & 3, q = lane >> 2;
    const int n = 4 * v + r;
    const int G = q * kDnChunks + j;
    if (!is_scale) {
      const uint4 w = *reinterpret_cast<const uint4*>(down_q + ((e * kH + n) * (kI / 2) + 16 * G));
      *reinterpret_cast<uint4*>(dn + ev * kDnUnitBytes + j * 512 + 16 * lane) = flip_sign_nibbles(w);
    } else {
      const uint16_t s = down_s[(e * kH + n) * (kI / kGroup) + G];
      *reinterpret_cast<uint16_t*>(dn + ev * kDnUnitBytes + kDnScaleOff + j * 64 + 2 * lane) = s;
    }
  }
}

cudaError_t launch_repack(const uint8_t* gate_q, const uint8_t* up_q, const void* gate_s,
                          const void* up_s, const uint8_t* down_q, const void* down_s, uint8_t* gu,
                          uint8_t* dn, int E, cudaStream_t stream) {
  const int threads = 256, blocks = 4096;
  repack_gu_kernel<<<blocks, threads, 0, stream>>>(gate_q, up_q, (const uint16_t*)gate_s,
                                                   (const uint16_t*)up_s, gu, E);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  repack_dn_kernel<<<blocks, threads, 0, stream>>>(down_q, (const uint16_t*)down_s, dn, E);
  return cudaGetLastError();
}

}  // namespace lingmoe
