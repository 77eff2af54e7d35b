// Tensor-core grouped GEMMs of the token-grouped path (tcgen05, sm_100a).
//
// For every routed expert e with m_e positions (token-expert pairs after the
// sort by expert), and for the shared expert over all T tokens:
//   gate/up:  H_e[m_e, 768]  = SiLU(X_e Wg_e^T) * (X_e Wu_e^T)     K = 2560
//   down:     Y_e[m_e, 2560] = w * (H_e Wd_e^T)                    K = 768
// as tiles of M = 256 weight rows (two M=128 MMAs) x N <= 128 positions.
//
// The weights are the A operand.  Routed weights are dequantised by
// producer warps into exact fp16 values q * s * 2^8 (q has at most 4
// significant bits and s is a bf16, so the product fits fp16's 11 bits) and
// written into 128-byte-swizzled K-major shared-memory tiles.  Their int4
// codes and scales arrive ahead of use: gate/up loads them into registers one
// stage ahead (two producer groups, 4 stages), down through a per-thread
// cp.async ring (one group, 3 stages).
// The shared expert's weights are pre-converted fp16 copies that TMA loads
// directly.  The activations are the B operand, fetched by TMA from buffers
// in position order: x (fp16, exact after a per-token power-of-two scale) for
// gate/up and h as two fp16 terms hi + lo (~22 significant bits) for down.
// All tiles are in natural K order: a producer gathers one row's K slice
// from the four MMA-fragment words of the repacked layouts that hold it.
//
// One thread issues tcgen05.mma into a double-buffered TMEM accumulator
// (2 x 256 columns); tcgen05.commit releases each pipeline stage, and 4
// epilogue warps drain a finished accumulator with tcgen05.ld while the next
// tile is already accumulating.
//
// Source of the layer: vLLM recipe page "inclusionAI/Ling-3.0-flash"
// ("Single-GPU int4": symmetric W4, group 32; "Launching the Server":
// chunked prefill) and the bpdata article "Harom optimalizacio a
// Ling-3.0-flash MoE inferenciajanak" ("Modell es kiindulo konfiguracio").
#include "common.cuh"
#include "grouped_tc.h"

namespace lingmoe {

// ---------------------------------------------------------------- roles and sizes
// A producer group is 8 warps, one A row per thread.  Gate/up runs two
// groups that take alternate pipeline stages (its dequantisation per stage is
// a dependent chain per warp, so a second group doubles the stages in work);
// down, whose shared memory holds two B parts per stage, runs one (two
// groups there need an even stage count, and its two stages measured slower).
constexpr int kProdWarps = 8;                  // warps per producer group
constexpr int kEpiWarps = 4;                   // TMEM lane quadrants 0..3
constexpr int kProd = kProdWarps * 32;            // 256 rows per group
static_assert(kProd == kTcTileM, "one producer thread per A row");
__host__ __device__ constexpr int tc_groups(int mode) { return mode == 0 ? 2 : 1; }
__host__ __device__ constexpr int tc_mma_warp(int mode) { return tc_groups(mode) * kProdWarps + kEpiWarps; }
__host__ __device__ constexpr int tc_threads(int mode) { return (tc_mma_warp(mode) + 2) * 32; }  // + MMA, TMA warps
static_assert(kProdWarps % 4 == 0, "epilogue warps must start at a multiple of 4");

constexpr int kTcK = 64;                        // K per stage: one 128-byte swizzle row of fp16
// pipeline stages: gate/up 4 (its B stage is half the size), down 3
// an even count for gate/up, so that every stage slot belongs to one group
__host__ __device__ constexpr int tc_stages(int mode) { return mode == 0 ? 4 : 3; }
constexpr int kStageA = kTcTileM * kTcK * 2;    // 32 KB
constexpr int kStageBPart = kTcTileN * kTcK * 2;  // 16 KB per B part
constexpr int kBoxRows = 32;                    // B rows per TMA box
constexpr int kBoxBytes = kBoxRows * kTcK * 2;  // 4 KB
constexpr int kShBoxRows = 128;                 // shared-expert A rows per TMA box
constexpr int kTmemCols = 512;                  // 2 buffers x (2 M-halves x 128 columns)
// raw ring, per stage: int4 codes [4 fragment lanes][256 threads] x 8 B, then
// per thread the scale words: gate/up one (gate, up) word of 4 B, down the
// two 4-byte (row pair) words of the stage's two groups.
constexpr int kRawCodes = 4 * kProd * 8;
constexpr int kRawStage = kRawCodes + kProd * 8;  // 10 KB
constexpr unsigned long long kTcWaitNs = 2000000000ull;

__host__ __device__ constexpr int tc_bparts(int mode) { return mode == 0 ? 1 : 2; }
// down's code ring depth; gate/up loads its codes straight into registers
__host__ __device__ constexpr int tc_raw_stages(int mode) { return mode == 0 ? 0 : 2; }
__host__ __device__ constexpr int tc_nk(int mode) { return (mode == 0 ? kH : kI) / kTcK; }
__host__ __device__ constexpr size_t tc_bar_off(int mode) {
  return (size_t)tc_stages(mode) * (kStageA + tc_bparts(mode) * kStageBPart) +
         (size_t)tc_groups(mode) * tc_raw_stages(mode) * kRawStage;
}
// after the barriers: per epilogue warp, per TMEM buffer, 128 column factors
constexpr int kFacOff = 256;
constexpr int kFacBytes = kEpiWarps * 2 * kTcTileN * 4;
__host__ __device__ constexpr size_t tc_smem(int mode) {
  return 1024 /*align slack*/ + tc_bar_off(mode) + kFacOff + kFacBytes;
}
static_assert(tc_smem(1) <= 232448, "down-projection pipeline exceeds 227 KB of shared memory");
static_assert(tc_smem(0) <= 232448, "gate/up pipeline exceeds 227 KB of shared memory");


// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  // K-major, 128B swizzle: 8-row atoms of 128 B, atoms 1024 B apart (SBO),
  // LBO unused (1), descriptor version 1, layout type 2.
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ uint32_t make_idesc(int n) {
  // D = f32, A = B = f16, both K-major, M = 128, N = n
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__device__ __forceinline__ void tc_mma(uint32_t tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      :: "r"(tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0));
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float v[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld16x2(uint32_t ta, uint32_t tb, float va[16], float vb[16]) {
  uint32_t r[16], q[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(ta));
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3]), "=r"(q[4]), "=r"(q[5]), "=r"(q[6]), "=r"(q[7]),
        "=r"(q[8]), "=r"(q[9]), "=r"(q[10]), "=r"(q[11]), "=r"(q[12]), "=r"(q[13]), "=r"(q[14]), "=r"(q[15])
      : "r"(tb));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    va[i] = __uint_as_float(r[i]);
    vb[i] = __uint_as_float(q[i]);
  }
}
// SiLU(s g) (s u) / s^2 = g u sigmoid(s g) with the fast exponential and
// division (relative error ~1e-6); g, u: the scaled gate and up values
__device__ __forceinline__ float tc_silu_mul_scaled(float g, float u, float s) {
  return __fdividef(g, 1.0f + __expf(-(g * s))) * u;
}
// 2-D tiled TMA load (no multicast) into this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}

// bounded wait used by every role; on time-out sets the error word and the
// CTA's abort flag and returns false
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, unsigned int* err, int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*reinterpret_cast<volatile int*>(abort) || globaltimer_ns() - t0 > kTcWaitNs) {
      atomicOr(err, 4u);
      *reinterpret_cast<volatile int*>(abort) = 1;
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------- dequantisation
// Two exact fp16 weights from a nibble pair (1024 + n in each half):
// v - 1032 = q is exact, and so is q * s' for s' = s * 2^8 (q has at most 4
// significant bits, s' at most 8).  Folding the bias into one fma would
// round -1032 * s'.
__device__ __forceinline__ uint32_t deq_pair(uint32_t v, __half2 s2, __half2 b2) {
  const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&v), b2);
  const __half2 r = __hmul2(q, s2);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// MXFP4: an E2M1 pair as fp16 (value * 2^-14, exact; deq_e2m1) times the
// group's scale factor f = s * 2^(14 + 8) (s = 2^(e - 127), the stored bf16
// being s * 2^14), applied as fa * fb with fa = f limited to [2^-14, 2^15] and
// fb = f / fa, so that both factors are fp16 powers of two and each product is
// exact: value * s * 2^8 is an fp16 multiple of 2^-24 below 65504 for
// E8M0 exponents e in [96, 132].
__device__ __forceinline__ void mx_factors(float f, __half2& fa, __half2& fb) {
  const float a = fminf(fmaxf(f, 0x1p-14f), 0x1p15f);
  fa = __float2half2_rn(a);
  fb = __float2half2_rn(f / a);
}
__device__ __forceinline__ uint32_t mx_pair(uint32_t e2m1_pair, __half2 fa, __half2 fb) {
  const __half2 r = __hmul2(__hmul2(*reinterpret_cast<const __half2*>(&e2m1_pair), fa), fb);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// ---------------------------------------------------------------- shared-expert fp16 copies
// Power-of-two exponent c with max|w| * 2^c in [2^14, 2^15) (0 for an all-zero
// matrix), clamped so that 2^c and 2^-c stay normal fp32 numbers.
__device__ __forceinline__ int sh_exp(unsigned int amax_bits) {
  if (amax_bits == 0) return 0;
  const int e = (int)(amax_bits >> 23) - 127;
  return max(-100, min(100, 14 - e));
}
__device__ __forceinline__ float pow2f(int c) { return __uint_as_float((uint32_t)(127 + c) << 23); }

__global__ void __launch_bounds__(256) sh_amax_kernel(const __nv_bfloat16* g, const __nv_bfloat16* u,
                                                      const __nv_bfloat16* d, unsigned int* amax) {
  const int m = blockIdx.y;  // 0 gate, 1 up, 2 down (all kI * kH elements)
  const __nv_bfloat16* w = m == 0 ? g : (m == 1 ? u : d);
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  float a = 0.f;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < kI * kH / 8; c += gridDim.x * blockDim.x) {
    const uint4 v = w4[c];
    a = fmaxf(a, fmaxf(fmaxf(fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x))), fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y)))),
                       fmaxf(fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))), fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w))))));
  }
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) atomicMax(&amax[m], __float_as_uint(fminf(a, 3.0e38f)));
}

// One thread per 8 consecutive K elements: scale by 2^c, convert to fp16.
// All keep the natural K order of the routed tiles.  Gate/up rows are laid out
// per block of 128 intermediate rows i: 128 gate rows, then the 128 up rows of
// the same i.
__global__ void __launch_bounds__(256) sh_convert_kernel(const __nv_bfloat16* g, const __nv_bfloat16* u,
                                                         const __nv_bfloat16* d, const unsigned int* amax,
                                                         __half* shgu16, __half* shdn16, float* sh_scale) {
  const int m = blockIdx.y;
  const int c = sh_exp(amax[m]);
  if (blockIdx.x == 0 && threadIdx.x == 0) sh_scale[m] = pow2f(-c);
  const float f = pow2f(c);
  const __nv_bfloat16* w = m == 0 ? g : (m == 1 ? u : d);
  const int K = m < 2 ? kH : kI;
  for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < kI * kH / 8; v += gridDim.x * blockDim.x) {
    const int row = (v * 8) / K, k0 = (v * 8) % K;
    const uint4 x = reinterpret_cast<const uint4*>(w)[v];
    const float e[8] = {bf16lo(x.x), bf16hi(x.x), bf16lo(x.y), bf16hi(x.y),
                        bf16lo(x.z), bf16hi(x.z), bf16lo(x.w), bf16hi(x.w)};
    __half h[8];
#pragma unroll
    for (int o = 0; o < 8; ++o) h[o] = __float2half_rn(e[o] * f);
    const int grow = 2 * (row & ~127) + 128 * m + (row & 127);
    __half* dst = m < 2 ? shgu16 + (size_t)grow * kH + k0 : shdn16 + (size_t)row * kI + k0;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(h);
  }
}

cudaError_t launch_tc_prep_shared(const __nv_bfloat16* g, const __nv_bfloat16* u, const __nv_bfloat16* d,
                                  __half* shgu16, __half* shdn16, float* sh_scale, unsigned int* amax_scratch,
                                  cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(amax_scratch, 0, 3 * sizeof(unsigned int), s);
  if (e != cudaSuccess) return e;
  sh_amax_kernel<<<dim3(148, 3), 256, 0, s>>>(g, u, d, amax_scratch);
  sh_convert_kernel<<<dim3(296, 3), 256, 0, s>>>(g, u, d, amax_scratch, shgu16, shdn16, sh_scale);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- L2 prefetch of a tile
// Everything one tile reads is contiguous: its 256 weight rows (routed units
// or fp16 shared rows) and its B rows (positions pos0 .. pos0 + n - 1).
// Issued for the next tile while the current one runs, so that the code
// and TMA loads of the main loop find their data in L2.
template <int MODE>
__device__ __forceinline__ void prefetch_tile(const TcParams& p, int4 tl, const __half* xg, const __half* h16,
                                              const __half* shgu16, const __half* shdn16) {
  const unsigned char* a;
  size_t abytes;
  if (tl.x < p.E) {
    if (MODE == 0) {
      a = p.gu + ((size_t)tl.x * kGuUnits + (size_t)tl.y * (kTcTileM / 16)) * kGuUnitBytes;
      abytes = (size_t)(kTcTileM / 16) * kGuUnitBytes;
    } else {
      a = p.dn + ((size_t)tl.x * kDnUnits + (size_t)tl.y * (kTcTileM / kDnUnitRows)) * kDnUnitBytes;
      abytes = (size_t)(kTcTileM / kDnUnitRows) * kDnUnitBytes;
    }
  } else {
    const int K = MODE == 0 ? kH : kI;
    a = reinterpret_cast<const unsigned char*>((MODE == 0 ? shgu16 : shdn16) + (size_t)tl.y * kTcTileM * K);
    abytes = (size_t)kTcTileM * K * sizeof(__half);
  }
  const size_t rowb = (MODE == 0 ? kH : 2 * kI) * sizeof(__half);
  const unsigned char* b = reinterpret_cast<const unsigned char*>(MODE == 0 ? xg : h16) + (size_t)tl.z * rowb;
  const size_t bbytes = (size_t)tl.w * rowb;
  constexpr size_t kPiece = 32768;
  for (size_t o = 0; o < abytes; o += kPiece) prefetch_l2_bulk(a + o, (uint32_t)min(kPiece, abytes - o));
  for (size_t o = 0; o < bbytes; o += kPiece) prefetch_l2_bulk(b + o, (uint32_t)min(kPiece, bbytes - o));
}

// ---------------------------------------------------------------- the GEMM
// MODE 0, gate/up: A row r of tile (e, mt) is the gate row (r < 128) or the
// up row (r >= 128) of intermediate row i = 128 mt + r % 128, so the two
// M-halves of the accumulator hold g and u for the same i in the same TMEM
// lane; B = x rows of the tile's positions; the epilogue writes
// h = SiLU(g) * u per position as fp16 hi + lo.
// MODE 1, down: A row r is output row 256 mt + r; B = the hi and lo halves of
// h, both accumulated into one TMEM tile; the epilogue writes y = w (Wd h).
//
// Roles: the producer warps dequantise A (gate/up: warps 0-15 in two groups
// of 8 taking alternate stages; down: warps 0-7), the next 4 warps drain
// TMEM, then one warp issues the MMAs (one thread) and one the TMA loads (one
// thread).  Every role walks the same sequence of tiles (blockIdx.x,
// + gridDim.x, ...) and stages.
template <int MODE, int C>
__global__ void __launch_bounds__(tc_threads(MODE), 1)
tc_grouped_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmA,
                  const TcParams p) {
  constexpr int NB = tc_bparts(MODE);
  constexpr int R = tc_raw_stages(MODE);
  constexpr int NK = tc_nk(MODE);
  constexpr int S = tc_stages(MODE);
  constexpr int NG = tc_groups(MODE);
  constexpr int kMmaWarp = tc_mma_warp(MODE);
  constexpr int kPW = NG * kProdWarps;  // producer warps
  extern __shared__ __align__(1024) unsigned char smem_raw_tc[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw_tc) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = smem;
  unsigned char* sB = smem + S * kStageA;
  unsigned char* sRaw = sB + S * NB * kStageBPart;
  uint64_t* full_a = reinterpret_cast<uint64_t*>(smem + tc_bar_off(MODE));
  uint64_t* full_b = full_a + S;
  uint64_t* empty = full_b + S;
  uint64_t* accf = empty + S;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* fac_s = reinterpret_cast<float*>(smem + tc_bar_off(MODE) + kFacOff);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int4* tiles = MODE == 0 ? p.gu_tiles : p.dn_tiles;
  const int ntiles = p.ntiles[MODE];
  const int ntl = ntiles > (int)blockIdx.x ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_a[s], kProdWarps);
      mbar_init(&full_b[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < kPW) {
    // ------------------------------------------------ producers: A row r
    // group pg takes the stages g = NG q + pg, q = 0, 1, ...
    const int r = tid & (kProd - 1), pg = tid / kProd;
    const int total = ntl * NK;
    constexpr int RR = R > 0 ? R : 1;
    const uint32_t raw0 = smem_u32(sRaw) + pg * R * kRawStage;
    // the codes and the scale word of groups 2kk, 2kk+1 of row r for the
    // group's q-th stage: gate/up loads them into registers (nc, nsw) one own
    // stage ahead; down cp.asyncs them into its raw slot q % R (one commit
    // group per stage, empty or not)
    int jn = -1;
    int4 tln = make_int4(0, 0, 0, 0);
    uint2 nc[4] = {};
    uint32_t nsw = 0;
    auto issue = [&](int q) {
      const int gq = NG * q + pg;
      if (gq < total) {
        const int j = gq / NK, kk = gq - j * NK;
        if (j != jn) {
          tln = tiles[blockIdx.x + j * gridDim.x];
          jn = j;
        }
        const int4 tl = tln;
        if (tl.x < p.E) {
          const uint32_t slot = raw0 + (q % RR) * kRawStage;
          if (MODE == 0) {
            // row i (gate and up), K blocks 2 kh, 2 kh + 1 of chunk kk: 8 bytes
            // from each of the four fragment lanes 4 (i % 8) + m, and the
            // (gate, up) scale word of group 2 kk + kh
            const int il = r & 127, kh = r >> 7;
            const int i = (kTcTileM / 2) * tl.y + il;
            const uint8_t* ub = p.gu + ((size_t)tl.x * kGuUnits + (i >> 3)) * kGuUnitBytes;
#pragma unroll
            for (int m = 0; m < 4; ++m)
              nc[m] = __ldg(reinterpret_cast<const uint2*>(ub + kk * 512 + 16 * (4 * (i & 7) + m) + 8 * kh));
            nsw = __ldg(reinterpret_cast<const unsigned int*>(ub + kGuScaleOff + (2 * kk + kh) * 32 + 4 * (i & 7)));
          } else {
            // output row n, groups G = 2 kk and G + 1: 8 bytes from each of the
            // four fragment lanes 4 (n % 8) + m, and the two scale words of
            // the row pair that holds n
            const int n = kTcTileM * tl.y + r, G = 2 * kk;
            const uint8_t* ub = p.dn + ((size_t)tl.x * kDnUnits + (n >> 3)) * kDnUnitBytes;
#pragma unroll
            for (int m = 0; m < 4; ++m)
              cp_async8(slot + m * (kProd * 8) + r * 8, ub + (G >> 2) * 512 + 16 * (4 * (n & 7) + m) + 4 * (G & 3));
            cp_async8(slot + kRawCodes + r * 8, ub + kDnScaleOff + (G >> 2) * 64 + 16 * ((n & 7) >> 1) + 4 * (G & 3));
          }
        }
      }
      if (MODE == 1) cp_async_commit();
    };
    if constexpr (MODE == 0) {
      issue(0);
    } else {
#pragma unroll 1
      for (int q = 0; q < R - 1; ++q) issue(q);
    }
    int jc = -1;
    int4 tl = make_int4(0, 0, 0, 0);
#pragma unroll 1
    for (int q = 0; NG * q + pg < total; ++q) {
      const int g = NG * q + pg;
      uint2 cw[4];
      uint32_t sw0 = 0;
      if constexpr (MODE == 0) {
#pragma unroll
        for (int m = 0; m < 4; ++m) cw[m] = nc[m];
        sw0 = nsw;
        issue(q + 1);
      } else {
        issue(q + R - 1);
        cp_async_wait<R - 1>();
      }
      const int j = g / NK, kk = g - j * NK;
      if (j != jc) {
        tl = tiles[blockIdx.x + j * gridDim.x];
        jc = j;
      }
      const int s = g % S;
      bool ok = true;
      if (lane == 0) ok = tc_wait(&empty[s], ((g / S) & 1) ^ 1, p.err, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (tl.x < p.E) {
        const unsigned char* slot = sRaw + (pg * R + q % RR) * kRawStage;
        if (MODE == 0) {
          // exact fp16 q * s * 2^8 for gate row il and up row 128 + il, K blocks
          // 2 kh and 2 kh + 1 of this stage (natural K order)
          const int il = r & 127, kh = r >> 7;
          const uint32_t sw = sw0;
          const float sgf = __uint_as_float(sw << 16) * (float)(1 << kTcScaleShift);
          const float suf = __uint_as_float(sw & 0xFFFF0000u) * (float)(1 << kTcScaleShift);
          const __half2 sg = __float2half2_rn(sgf), sg16 = __float2half2_rn(sgf * 0.0625f);
          const __half2 su = __float2half2_rn(suf), su16 = __float2half2_rn(suf * 0.0625f);
          const __half2 be = __float2half2_rn(1032.0f), bo = __float2half2_rn(1152.0f);
          __half2 ga, gb, ua, ub;
          if constexpr (C == kCodecMxfp4) {
            mx_factors(sgf, ga, gb);
            mx_factors(suf, ua, ub);
          }
          unsigned char* ag = sA + s * kStageA + il * 128;
          unsigned char* au = sA + s * kStageA + (128 + il) * 128;
#pragma unroll
          for (int ww = 0; ww < 2; ++ww) {
            uint32_t glo[4], ghi[4], ulo[4], uhi[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const uint32_t w = ww ? cw[m].y : cw[m].x;
              if constexpr (C == kCodecMxfp4) {
                glo[m] = mx_pair(deq_e2m1<0>(w), ga, gb);   // gate c, c+1
                ghi[m] = mx_pair(deq_e2m1<4>(w), ga, gb);   // gate c+8, c+9
                ulo[m] = mx_pair(deq_e2m1<8>(w), ua, ub);   // up c, c+1
                uhi[m] = mx_pair(deq_e2m1<12>(w), ua, ub);  // up c+8, c+9
                continue;
              }
              uint32_t v0, v1, v2, v3;
              asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(v0) : "r"(w));
              asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xEA;" : "=r"(v1) : "r"(w));
              asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(v2) : "r"(w >> 8));
              asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xEA;" : "=r"(v3) : "r"(w >> 8));
              glo[m] = deq_pair(v0, sg, be);    // gate c, c+1:  (1024 + n - 1032) s
              ghi[m] = deq_pair(v1, sg16, bo);  // gate c+8, c+9: (1024 + 16 n - 1152) s / 16
              ulo[m] = deq_pair(v2, su, be);
              uhi[m] = deq_pair(v3, su16, bo);
            }
            const int cl = 4 * kh + 2 * ww, ch = cl + 1;
            *reinterpret_cast<uint4*>(ag + ((cl ^ (il & 7)) << 4)) = make_uint4(glo[0], glo[1], glo[2], glo[3]);
            *reinterpret_cast<uint4*>(ag + ((ch ^ (il & 7)) << 4)) = make_uint4(ghi[0], ghi[1], ghi[2], ghi[3]);
            *reinterpret_cast<uint4*>(au + ((cl ^ (il & 7)) << 4)) = make_uint4(ulo[0], ulo[1], ulo[2], ulo[3]);
            *reinterpret_cast<uint4*>(au + ((ch ^ (il & 7)) << 4)) = make_uint4(uhi[0], uhi[1], uhi[2], uhi[3]);
          }
        } else {
          // exact fp16 q * s * 2^8 for output row n, groups 2 kk and 2 kk + 1:
          // the fragment word of lane class m holds K = 2m, 2m+1 (even
          // extraction), 2m+8, 2m+9 (odd, as 16 q), and the same + 16 in w >> 8
          const int n = kTcTileM * tl.y + r;
          const uint2 sw = *reinterpret_cast<const uint2*>(slot + kRawCodes + r * 8);
          const __half2 be = __float2half2_rn(1032.0f), bo = __float2half2_rn(1152.0f);
#pragma unroll
          for (int m = 0; m < 4; ++m) cw[m] = *reinterpret_cast<const uint2*>(slot + m * (kProd * 8) + r * 8);
          unsigned char* a = sA + s * kStageA + r * 128;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t ws = h ? sw.y : sw.x;
            const float sf = __uint_as_float((n & 1) ? (ws & 0xFFFF0000u) : (ws << 16)) * (float)(1 << kTcScaleShift);
            const __half2 s2 = __float2half2_rn(sf), s16 = __float2half2_rn(sf * 0.0625f);
            __half2 fa, fb;
            if constexpr (C == kCodecMxfp4) mx_factors(sf, fa, fb);
            uint32_t q0[4], q1[4], q2[4], q3[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const uint32_t w = h ? cw[m].y : cw[m].x;
              if constexpr (C == kCodecMxfp4) {
                q0[m] = mx_pair(deq_e2m1<0>(w), fa, fb);   // K c, c+1
                q1[m] = mx_pair(deq_e2m1<4>(w), fa, fb);   // c+8, c+9
                q2[m] = mx_pair(deq_e2m1<8>(w), fa, fb);   // c+16, c+17
                q3[m] = mx_pair(deq_e2m1<12>(w), fa, fb);  // c+24, c+25
                continue;
              }
              uint32_t v0, v1, v2, v3;
              asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(v0) : "r"(w));
              asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xEA;" : "=r"(v1) : "r"(w));
              asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(v2) : "r"(w >> 8));
              asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xEA;" : "=r"(v3) : "r"(w >> 8));
              q0[m] = deq_pair(v0, s2, be);
              q1[m] = deq_pair(v1, s16, bo);
              q2[m] = deq_pair(v2, s2, be);
              q3[m] = deq_pair(v3, s16, bo);
            }
            const int c0 = 4 * h;
            *reinterpret_cast<uint4*>(a + (((c0 + 0) ^ (r & 7)) << 4)) = make_uint4(q0[0], q0[1], q0[2], q0[3]);
            *reinterpret_cast<uint4*>(a + (((c0 + 1) ^ (r & 7)) << 4)) = make_uint4(q1[0], q1[1], q1[2], q1[3]);
            *reinterpret_cast<uint4*>(a + (((c0 + 2) ^ (r & 7)) << 4)) = make_uint4(q2[0], q2[1], q2[2], q2[3]);
            *reinterpret_cast<uint4*>(a + (((c0 + 3) ^ (r & 7)) << 4)) = make_uint4(q3[0], q3[1], q3[2], q3[3]);
          }
        }
        fence_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_a[s]);
    }
    cp_async_wait_all();
  } else if (warp < kMmaWarp) {
    // ------------------------------------------------ epilogue: TMEM lanes 32 qd .. 32 qd + 31
    const int qd = warp & 3;
    const int l = 32 * qd + lane;  // accumulator row within an M-half
    float* facw = fac_s + (warp - kPW) * (2 * kTcTileN);
#pragma unroll 1
    for (int j = 0; j < ntl; ++j) {
      const int b = j & 1;
      const int4 tl = tiles[blockIdx.x + j * gridDim.x];
      const int mt = tl.y, pos0 = tl.z, n = tl.w, nmma = (n + 15) & ~15;
      const bool shared = tl.x >= p.E;
      // per-column factors, fetched while the tile is still accumulating:
      // gate/up the token's 2^sigma, down the pair's routing weight
      float* fb = facw + b * kTcTileN;
      for (int c = lane; c < n; c += 32) {
        const int pos = pos0 + c;
        float f;
        if (MODE == 0) f = p.xscale[shared ? pos - p.P : p.perm[pos] / p.k];
        else f = shared ? p.sh_scale[2] * (float)(1 << kTcScaleShift) : p.topk_w[p.perm[pos]];
        fb[c] = f;
      }
      __syncwarp();
      bool ok = true;
      if (lane == 0) ok = tc_wait(&accf[b], (j >> 1) & 1, p.err, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(32 * qd) << 16) + (uint32_t)(b * 256);
      if (MODE == 0) {
        const int i = (kTcTileM / 2) * mt + l;
        const float cg = shared ? p.sh_scale[0] : 1.f / (float)(1 << kTcScaleShift);
        const float cu = shared ? p.sh_scale[1] : 1.f / (float)(1 << kTcScaleShift);
        __half* hrow = p.h16 + (size_t)pos0 * (2 * kI) + i;
#pragma unroll 1
        for (int c0 = 0; c0 < nmma; c0 += 16) {
          float g[16], u[16];
          tmem_ld16x2(tb + c0, tb + 128 + c0, g, u);
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {
            const int col = c0 + cc;
            if (col < n) {
              const float f = fb[col];
              // h / c_t^2 = (x-scaled gate/up product) * 2^-2*kGrpUnitShift, then the fp16 shift
              const float hv = tc_silu_mul_scaled(g[cc] * cg, u[cc] * cu, f) *
                               (1.f / (float)(1 << kTcScaleShift)) * (1.f / (float)(1 << (2 * kGrpUnitShift)));
              const __half hi = __float2half_rn(hv);
              hrow[(size_t)col * (2 * kI)] = hi;
              hrow[(size_t)col * (2 * kI) + kI] = __float2half_rn(hv - __half2float(hi));
            }
          }
        }
      } else {
#pragma unroll 1
        for (int mh = 0; mh < 2; ++mh) {
          float* yrow = p.y + (size_t)pos0 * kH + kTcTileM * mt + mh * 128 + l;
#pragma unroll 1
          for (int c0 = 0; c0 < nmma; c0 += 32) {
            float v0[16], v1[16];
            tmem_ld16x2(tb + mh * 128 + c0, tb + mh * 128 + c0 + 16, v0, v1);
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
              const int col = c0 + cc;
              if (col < n) yrow[(size_t)col * kH] = v0[cc] * fb[col];
            }
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
              const int col = c0 + 16 + cc;
              if (col < n) yrow[(size_t)col * kH] = v1[cc] * fb[col];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[b]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issue (one thread)
    if (lane == 0) {
      int g = 0;
      bool ok = true;
#pragma unroll 1
      for (int j = 0; j < ntl && ok; ++j) {
        const int b = j & 1;
        const int4 tl = tiles[blockIdx.x + j * gridDim.x];
        const int nmma = (tl.w + 15) & ~15;
        if (j >= 2 && !tc_wait(&acce[b], ((j >> 1) - 1) & 1, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t idesc = make_idesc(nmma);
        const uint32_t dcol = tmem + (uint32_t)(b * 256);
#pragma unroll 1
        for (int kk = 0; kk < NK; ++kk, ++g) {
          const int s = g % S;
          const uint32_t ph = (g / S) & 1;
          if (!tc_wait(&full_a[s], ph, p.err, abort_flag) || !tc_wait(&full_b[s], ph, p.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kStageA), b0 = smem_u32(sB + s * NB * kStageBPart);
#pragma unroll
          for (int k4 = 0; k4 < kTcK / 16; ++k4)
#pragma unroll
            for (int mh = 0; mh < 2; ++mh)
#pragma unroll
              for (int part = 0; part < NB; ++part)
                tc_mma(dcol + mh * 128, sw128_desc(a0 + mh * (kStageA / 2) + 32 * k4),
                       sw128_desc(b0 + part * kStageBPart + 32 * k4), idesc, (kk | k4 | part) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(&accf[b]);
      }
      // no MMA may still be writing TMEM when it is freed
      tc_commit(drain);
      mbar_wait(drain, 0, kTcWaitNs, p.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ TMA issue (one thread)
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      if (ntl > 0) prefetch_tile<MODE>(p, tiles[blockIdx.x], p.xg, p.h16, p.shgu16, p.shdn16);
#pragma unroll 1
      for (int j = 0; j < ntl && ok; ++j) {
        const int4 tl = tiles[blockIdx.x + j * gridDim.x];
        if (j + 1 < ntl)
          prefetch_tile<MODE>(p, tiles[blockIdx.x + (j + 1) * gridDim.x], p.xg, p.h16, p.shgu16, p.shdn16);
        const int nmma = (tl.w + 15) & ~15, nbox = (nmma + kBoxRows - 1) / kBoxRows;
        const bool shared = tl.x >= p.E;
        const uint32_t bytes = (uint32_t)(NB * nbox * kBoxBytes + (shared ? kStageA : 0));
#pragma unroll 1
        for (int kk = 0; kk < NK; ++kk, ++g) {
          const int s = g % S;
          if (!tc_wait(&empty[s], ((g / S) & 1) ^ 1, p.err, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_b[s], bytes);
          const uint32_t bdst = smem_u32(sB + s * NB * kStageBPart);
#pragma unroll
          for (int part = 0; part < NB; ++part)
            for (int bx = 0; bx < nbox; ++bx)
              tma_load_2d(bdst + part * kStageBPart + bx * kBoxBytes, &tmB, part * kI + kk * kTcK,
                          tl.z + bx * kBoxRows, &full_b[s]);
          if (shared) {
            const uint32_t adst = smem_u32(sA + s * kStageA);
            for (int hf = 0; hf < kTcTileM / kShBoxRows; ++hf)
              tma_load_2d(adst + hf * (kShBoxRows * 128), &tmA, kk * kTcK, kTcTileM * tl.y + hf * kShBoxRows,
                          &full_b[s]);
          }
        }
      }
      // after an abort, loads may still be landing: wait for every armed stage
      for (int q = g - S > 0 ? g - S : 0; q < g; ++q) mbar_wait(&full_b[q % S], (q / S) & 1, kTcWaitNs, p.err);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------- host
template <int C>
static cudaError_t setup_c() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(tc_grouped_kernel<0, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)tc_smem(0))) != cudaSuccess)
    return e;
  return cudaFuncSetAttribute(tc_grouped_kernel<1, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)tc_smem(1));
}

cudaError_t setup_grouped_tc() {
  const cudaError_t e = setup_c<kCodecInt4>();
  return e != cudaSuccess ? e : setup_c<kCodecMxfp4>();
}

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// fp16 matrix [rows, cols] row-major; boxes of 64 columns (128 B) x box_rows,
// 128-byte swizzle, zero fill outside the matrix
cudaError_t encode_2d(CUtensorMap* m, const __half* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * sizeof(__half)};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
}  // namespace

cudaError_t tc_encode_maps(TcMaps* m, const __half* xg, const __half* h16, int rows, const __half* shgu16,
                           const __half* shdn16) {
  cudaError_t e;
  if ((e = encode_2d(&m->b_x, xg, rows, kH, kBoxRows)) != cudaSuccess) return e;
  if ((e = encode_2d(&m->b_h, h16, rows, 2 * kI, kBoxRows)) != cudaSuccess) return e;
  if ((e = encode_2d(&m->a_shgu, shgu16, 2 * kI, kH, kShBoxRows)) != cudaSuccess) return e;
  return encode_2d(&m->a_shdn, shdn16, kH, kI, kShBoxRows);
}

cudaError_t launch_tc_gemm(int mode, const TcMaps& m, const TcParams& p, int nctas, cudaStream_t s) {
  if (p.codec == kCodecMxfp4) {
    if (mode == 0) tc_grouped_kernel<0, kCodecMxfp4><<<nctas, tc_threads(0), tc_smem(0), s>>>(m.b_x, m.a_shgu, p);
    else tc_grouped_kernel<1, kCodecMxfp4><<<nctas, tc_threads(1), tc_smem(1), s>>>(m.b_h, m.a_shdn, p);
  } else {
    if (mode == 0) tc_grouped_kernel<0, kCodecInt4><<<nctas, tc_threads(0), tc_smem(0), s>>>(m.b_x, m.a_shgu, p);
    else tc_grouped_kernel<1, kCodecInt4><<<nctas, tc_threads(1), tc_smem(1), s>>>(m.b_h, m.a_shdn, p);
  }
  return cudaGetLastError();
}

}  // namespace lingmoe
