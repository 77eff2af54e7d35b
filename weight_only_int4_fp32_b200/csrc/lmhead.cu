// Online-FP8 LM head (hidden -> vocabulary): bf16 weights quantised once, at
// build time, to e4m3 with one fp32 scale per vocabulary row; per call the
// tokens are quantised the same way and every logit is the scaled sum of
// exact e4m3 x e4m3 products.
//
// Quantisation of a row (or token): scale = max|v| / 448 (1 for an all-zero
// row), code = e4m3(v / scale), both divisions correctly rounded in fp32,
// the conversion round-to-nearest-even and saturating (cvt.rn.satfinite).
//
// Layout of the codes in HBM (written by the build-time kernel): tiles of 32
// vocabulary rows, each cut along K into chunks of 256 codes; a chunk is 8 KB
// of contiguous bytes, already in the order the GEMV's fragment loads want:
// for 64-code block b, 16-row half h and row group p (rows g or g + 8 of the
// half), 512 bytes = 32 lanes x 16 codes, lane 4 g + t holding codes
// 64 b + 16 t .. + 15 of row 16 h + 8 p + g.  Tiles follow one another, and
// the chunks of a tile, so each CTA streams one contiguous byte range.
// Rows past the vocabulary (the last tile's padding) hold zero codes.
//
// Source: bpdata article "Harom optimalizacio a Ling-3.0-flash MoE
// inferenciajanak", section "Optimalizacio 2: Online FP8 LM head kvantalas"
// (157,184 x 2,560 head quantised dynamically to FP8 when the head is built;
// roughly half the bytes of the bf16 head).
#include "common.cuh"
#include "lmhead.h"

namespace lingmoe {

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

constexpr int kLmhTile = 32;                          // vocabulary rows per tile (two m16 halves)
constexpr int kLmhKc = 256;                           // codes per row per chunk
constexpr int kLmhChunkBytes = kLmhTile * kLmhKc;     // 8 KB

// Byte offset of code k of row r in the tiled layout (k % 16 == 0 or 8).
__host__ __device__ __forceinline__ size_t lmh_tiled_off(long long r, int k, int nq) {
  const long long j = r / kLmhTile;
  const int rr = (int)(r % kLmhTile), q = k / kLmhKc, kk = k % kLmhKc;
  const int b = kk / 64, t = (kk % 64) / 16, e = kk % 16;
  const int h = rr / 16, p = (rr % 16) / 8, g = rr % 8;
  return (size_t)(j * nq + q) * kLmhChunkBytes + (size_t)((b * 2 + h) * 2 + p) * 512 + (4 * g + t) * 16 + e;
}

// One warp quantises one row of n values (n % 256 == 0): its scale, and its
// codes, 8 consecutive ones at a time to dst(k) for k = 0, 8, 16, ...
template <class Dst>
__device__ __forceinline__ void quantize_row_warp(const __nv_bfloat16* src, int n, Dst dst, float* scale) {
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
    *reinterpret_cast<uint2*>(dst(8 * c)) = make_uint2(lo, hi);
  }
  if (lane == 0) *scale = s;
}

// Build time: one warp per vocabulary row, codes to the tiled layout.
__global__ void __launch_bounds__(256) lmh_quantize_kernel(const __nv_bfloat16* __restrict__ w, int vocab,
                                                           int hidden, uint8_t* __restrict__ codes,
                                                           float* __restrict__ scales) {
  const int warps = blockDim.x / 32, nq = hidden / kLmhKc;
  for (long long r = (long long)blockIdx.x * warps + (threadIdx.x >> 5); r < vocab; r += (long long)gridDim.x * warps)
    quantize_row_warp(w + r * hidden, hidden, [=](int k) { return codes + lmh_tiled_off(r, k, nq); }, scales + r);
}

// The tiled codes back in row-major order [vocab, hidden] (16 codes a thread).
__global__ void __launch_bounds__(256) lmh_untile_kernel(const uint8_t* __restrict__ tiled, int vocab, int hidden,
                                                         uint8_t* __restrict__ out) {
  const int nq = hidden / kLmhKc, per_row = hidden / 16;
  const long long n = (long long)vocab * per_row;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / per_row;
    const int k = (int)(i % per_row) * 16;
    *reinterpret_cast<uint4*>(out + r * hidden + k) = *reinterpret_cast<const uint4*>(tiled + lmh_tiled_off(r, k, nq));
  }
}

// ---------------------------------------------------------------- pipelined tensor-core GEMV
// Every CTA owns a contiguous range of tiles, i.e. one contiguous byte range
// of the tiled codes, n = tiles x (hidden / 256) chunks.  Consumer warp w
// takes the contiguous chunks [n w / C, n (w + 1) / C) of it, so all warps
// stream to the end together; a tile cut by such a boundary is summed from
// the warps' partial sums after all of them are done, in warp order.  One
// producer thread sweeps the consumers and, for each one whose next ring
// slot is free, issues that chunk with one non-multicast 8 KB bulk copy.
// Each consumer owns kLmhDepth slots with a full and an empty mbarrier
// each; because a slot only ever serves one warp, that warp sees every
// phase of its barriers in order.  The tokens' codes sit in shared memory
// in the same fragment order as the head (lane 4 t + u holds codes
// 16 u .. + 15 of token t in each 64-code block; zero for tokens beyond T).
// For each 64-code block a lane loads its 16 codes of the tokens and of rows
// g and g + 8 of each 16-row half (lane-contiguous, so free of bank
// conflicts), turns them into fp16 pairs (exact) and issues four m16n8k16
// MMAs per half (columns = tokens).  The K order inside an MMA is a
// permutation of the block's 64 codes, the same for A and B.  The MMAs of
// one chunk (256 codes) are chained on one accumulator per half, which is
// then added to the fp32 sum of the row.  Every wait is bounded
// (globaltimer); a wait that runs out sets bit 2 of the error word and the
// CTA stops, after its copies in flight have landed.
constexpr int kLmhConsumers = 8;
constexpr int kLmhDepth = 2;  // ring slots per consumer warp
constexpr int kLmhMmaThreads = (kLmhConsumers + 1) * 32;
constexpr int kLmhSlots = kLmhDepth * kLmhConsumers;
constexpr int kLmhRecBytes = 32 * 8 * 4;  // one warp's partial sums of a tile (8 per lane)

struct LmhParams {
  const uint8_t* codes;  // tiled
  const float* scales;
  const __nv_bfloat16* x;
  float* logits;
  uint8_t* x_codes;
  float* x_scales;
  unsigned int* err;
  unsigned long long wait_limit_ns;
  int vocab, hidden, T;
  int skip_cta;  // test hook: this CTA's producer issues no copies (-1: none)
};

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Wait for phase `parity`; false once *stop is set or the limit has passed
// (the latter also sets the error word).
__device__ __forceinline__ bool lmh_wait(uint64_t* bar, uint32_t parity, volatile int* stop,
                                         unsigned long long limit_ns, unsigned int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*stop) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(err, 2u);
      *stop = 1;
      return false;
    }
  }
  return true;
}

size_t lmh_mma_smem(int hidden) {
  return (size_t)kLmhSlots * kLmhChunkBytes + (size_t)hidden * 8 + 32 + 16 * kLmhSlots + 16;
}

// logits of the 32 rows of tile row0 from one lane's sums a[half][4]
__device__ __forceinline__ void lmh_store(const LmhParams& p, const float* xs, long long row0, int lane,
                                          const float (&a)[2][4]) {
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
      const long long row = row0 + 16 * h + 8 * hi + g;
      if (row >= p.vocab) continue;
      const float sw = __ldg(p.scales + row);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int tok = 2 * t4 + k;
        if (tok < p.T) p.logits[(size_t)tok * p.vocab + row] = a[h][2 * hi + k] * xs[tok] * sw;
      }
    }
}

__global__ void __launch_bounds__(kLmhMmaThreads, 1) lmh_mma_kernel(const LmhParams p) {
  extern __shared__ __align__(128) unsigned char lsm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.hidden, nq = H / kLmhKc;
  unsigned char* ring = lsm;                                 // [slots][8 KB]
  uint8_t* xf = ring + (size_t)kLmhSlots * kLmhChunkBytes;   // [H/64][32 lanes][16 codes]
  float* xs = reinterpret_cast<float*>(xf + (size_t)H * 8);   // [8]
  uint64_t* full = reinterpret_cast<uint64_t*>(xs + 8);
  uint64_t* empty = full + kLmhSlots;
  volatile int* stop = reinterpret_cast<volatile int*>(empty + kLmhSlots);

  const int tiles = (p.vocab + kLmhTile - 1) / kLmhTile;
  const int j0 = (int)((long long)tiles * blockIdx.x / gridDim.x);
  const int j1 = (int)((long long)tiles * (blockIdx.x + 1) / gridDim.x);
  const int nchunks = (j1 - j0) * nq;

  if (tid == 0) {
    for (int s = 0; s < kLmhSlots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    *stop = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kLmhConsumers) {
    // ---- producer: issue warp w's r-th chunk (slot D w + r % D) once that slot is free
    if (lane == 0) {
      const uint8_t* base = p.codes + (size_t)j0 * nq * kLmhChunkBytes;
      int next[kLmhConsumers];
      int left = nchunks;
#pragma unroll
      for (int w = 0; w < kLmhConsumers; ++w) next[w] = 0;
      unsigned long long t0 = globaltimer_ns();
      const bool withhold = (int)blockIdx.x == p.skip_cta;
      while (left > 0 && !*stop) {
        bool moved = false;
#pragma unroll
        for (int w = 0; w < kLmhConsumers; ++w) {
          const int cb = nchunks * w / kLmhConsumers, n_w = nchunks * (w + 1) / kLmhConsumers - cb;
          const int r = next[w];
          if (r >= n_w) continue;
          const int s = kLmhDepth * w + r % kLmhDepth;
          if (withhold || (r >= kLmhDepth && !mbar_test(&empty[s], (r / kLmhDepth - 1) & 1))) continue;
          mbar_arrive_expect_tx(&full[s], kLmhChunkBytes);
          bulk_g2s(ring + (size_t)s * kLmhChunkBytes, base + (size_t)(cb + r) * kLmhChunkBytes, kLmhChunkBytes,
                   &full[s]);
          next[w] = r + 1;
          --left;
          moved = true;
        }
        if (moved) {
          t0 = globaltimer_ns();
        } else if (globaltimer_ns() - t0 > p.wait_limit_ns) {
          atomicOr(p.err, 2u);
          *stop = 1;
        } else {
          __nanosleep(32);  // leave the issue slots to the consumers of this sub-partition
        }
      }
      // every issued copy lands before the CTA may end
      volatile int never = 0;
#pragma unroll
      for (int w = 0; w < kLmhConsumers; ++w)
        for (int b = 0; b < kLmhDepth; ++b) {
          const int uses = (next[w] - b + kLmhDepth - 1) / kLmhDepth;  // rounds below next[w] with r % D == b
          if (uses > 0) lmh_wait(&full[kLmhDepth * w + b], (uses - 1) & 1, &never, p.wait_limit_ns, p.err);
        }
    }
    return;
  }

  // ---- consumers: the tokens' codes (fragment order) and scales
  for (int e = tid; e < (H / 64) * 32; e += kLmhConsumers * 32)
    if ((e & 31) >> 2 >= p.T) *reinterpret_cast<uint4*>(xf + 16 * (size_t)e) = make_uint4(0, 0, 0, 0);
  for (int t = warp; t < p.T; t += kLmhConsumers)
    quantize_row_warp(p.x + (size_t)t * H, H,
                      [=](int k) { return xf + (k >> 6) * 512 + (4 * t + ((k & 63) >> 4)) * 16 + (k & 15); }, &xs[t]);
  asm volatile("bar.sync 1, %0;" :: "n"(kLmhConsumers * 32) : "memory");
  if (blockIdx.x == 0 && p.x_codes != nullptr)
    for (int e = tid; e < p.T * H / 16; e += kLmhConsumers * 32) {
      const int t = e / (H / 16), k = (e % (H / 16)) * 16;
      reinterpret_cast<uint4*>(p.x_codes)[e] =
          *reinterpret_cast<const uint4*>(xf + (k >> 6) * 512 + (4 * t + ((k & 63) >> 4)) * 16);
    }
  if (blockIdx.x == 0 && p.x_scales != nullptr && tid < p.T) p.x_scales[tid] = xs[tid];

  // partial sums of the (at most two) tiles this warp has only a piece of;
  // they go to the first of its own ring slots once its chunks are done
  // (record 0: the piece its range starts inside, record 1: the one it ends inside)
  const int cb = nchunks * warp / kLmhConsumers, ce = nchunks * (warp + 1) / kLmhConsumers;
  bool ok = true;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  float part[2][8];
  for (int c = cb, r = 0; c < ce; ++c, ++r) {
    const int q = c % nq, s = kLmhDepth * warp + r % kLmhDepth;
    if (!__all_sync(0xffffffffu, lmh_wait(&full[s], (r / kLmhDepth) & 1, stop, p.wait_limit_ns, p.err))) {
      ok = false;
      break;
    }
    const unsigned char* st = ring + (size_t)s * kLmhChunkBytes + 16 * lane;
    const unsigned char* xb = xf + (size_t)q * (kLmhKc / 64) * 512 + 16 * lane;
    float cs[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int b = 0; b < kLmhKc / 64; ++b) {
      const uint4 xc = lds128(xb + 512 * b);
      const uint32_t xp[4] = {xc.x, xc.y, xc.z, xc.w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 wa = lds128(st + ((b * 2 + h) * 2 + 0) * 512);
        const uint4 wb = lds128(st + ((b * 2 + h) * 2 + 1) * 512);
        const uint32_t pa[4] = {wa.x, wa.y, wa.z, wa.w}, pb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int m = 0; m < 4; ++m)
          mma_16816(cs[h][0], cs[h][1], cs[h][2], cs[h][3], e4m3x2_to_f16x2(pa[m]), e4m3x2_to_f16x2(pb[m]),
                    e4m3x2_to_f16x2(pa[m] >> 16), e4m3x2_to_f16x2(pb[m] >> 16), e4m3x2_to_f16x2(xp[m]),
                    e4m3x2_to_f16x2(xp[m] >> 16), cs[h][0], cs[h][1], cs[h][2], cs[h][3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[h][i] += cs[h][i];
    if (q == nq - 1 || c == ce - 1) {
      // end of this warp's piece of tile c / nq: whole tile -> logits; else a partial record
      const int tile_first = c - q;
      if (tile_first >= cb && q == nq - 1) {
        lmh_store(p, xs, (long long)(j0 + c / nq) * kLmhTile, lane, acc);
      } else if (tile_first < cb) {
#pragma unroll
        for (int i = 0; i < 8; ++i) part[0][i] = acc[i >> 2][i & 3];
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) part[1][i] = acc[i >> 2][i & 3];
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][i] = 0.f;
    }
  }
  // (no copy is in flight into this warp's slots once it has consumed its
  // last chunk; after a failed wait the records are not used)
  if (ok && cb < ce) {
    float* own = reinterpret_cast<float*>(ring + (size_t)kLmhDepth * warp * kLmhChunkBytes);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      own[32 * i + lane] = part[0][i];
      own[kLmhRecBytes / 4 + 32 * i + lane] = part[1][i];
    }
  }
  // tiles cut between warps: the warp holding a tile's last chunk sums the
  // records of every warp that has a piece of it, in warp order
  asm volatile("bar.sync 1, %0;" :: "n"(kLmhConsumers * 32) : "memory");
  if (!__all_sync(0xffffffffu, ok) || *stop || cb >= ce || cb % nq == 0) return;
  const int f = cb / nq;                       // the tile this warp's range starts inside
  if ((f + 1) * nq - 1 >= ce) return;          // its last chunk belongs to a later warp
  float sum[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  for (int w = 0; w <= warp; ++w) {
    const int wb = nchunks * w / kLmhConsumers, we = nchunks * (w + 1) / kLmhConsumers;
    if (we <= f * nq || wb >= (f + 1) * nq || wb >= we) continue;  // no piece of tile f
    // its piece is its first one (record 0) if its range starts inside tile f
    const float* src = reinterpret_cast<const float*>(ring + (size_t)kLmhDepth * w * kLmhChunkBytes) +
                       (f * nq < wb ? 0 : kLmhRecBytes / 4);
#pragma unroll
    for (int i = 0; i < 8; ++i) sum[i >> 2][i & 3] += src[32 * i + lane];
  }
  lmh_store(p, xs, (long long)(j0 + f) * kLmhTile, lane, sum);
}

size_t lmh_codes_bytes(int vocab, int hidden) {
  return (size_t)((vocab + kLmhTile - 1) / kLmhTile) * kLmhTile * hidden;
}

cudaError_t setup_lmhead() {
  return cudaFuncSetAttribute(lmh_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)lmh_mma_smem(kLmhMaxHidden));
}

cudaError_t launch_lmh_quantize(const __nv_bfloat16* w, int vocab, int hidden, uint8_t* codes, float* scales,
                                cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(codes, 0, lmh_codes_bytes(vocab, hidden), s);  // the last tile's padding rows
  if (e != cudaSuccess) return e;
  lmh_quantize_kernel<<<4 * 148, 256, 0, s>>>(w, vocab, hidden, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_lmh_untile(const uint8_t* codes, int vocab, int hidden, uint8_t* out, cudaStream_t s) {
  lmh_untile_kernel<<<4 * 148, 256, 0, s>>>(codes, vocab, hidden, out);
  return cudaGetLastError();
}

cudaError_t launch_lmh_forward(const uint8_t* codes, const float* scales, int vocab, int hidden,
                               const __nv_bfloat16* x, int T, float* logits, uint8_t* x_codes, float* x_scales,
                               unsigned int* err, unsigned long long wait_limit_ns, int skip_cta, int nctas,
                               cudaStream_t s) {
  if (hidden % 512 || hidden > kLmhMaxHidden || T < 1 || T > kLmhMaxT) return cudaErrorInvalidValue;
  LmhParams p{codes, scales, x, logits, x_codes, x_scales, err, wait_limit_ns, vocab, hidden, T, skip_cta};
  lmh_mma_kernel<<<nctas, kLmhMmaThreads, lmh_mma_smem(hidden), s>>>(p);
  return cudaGetLastError();
}

}  // namespace lingmoe
