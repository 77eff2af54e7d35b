// Tensor-core grouped GEMMs of the token-grouped path (tcgen05, sm_100a).
//
// For every routed expert e with m_e tokens (after the stable sort by expert):
//   gate/up:  H_e[m_e, 768]  = SiLU(X_e Wg_e^T) * (X_e Wu_e^T)     K = 2560
//   down:     Y_e[m_e, 2560] = w * (H_e Wd_e^T)                    K = 768
// as tiles of M = 128 weight rows x N <= 128 tokens.  The weights are the
// A operand: producer warps dequantise the repacked int4 codes into exact
// fp16 values q*s (q has at most 4 significant bits and s is a bf16, so the
// product fits fp16's 11 bits) and write them into 128-byte-swizzled K-major
// shared-memory tiles.  The activations are the B operand, stored in fp16 in
// the same per-8-element K order as the dequantised codes (the order a LOP3
// extracts nibbles in), so no permutation is needed inside the main loop.
// One elected thread issues tcgen05.mma into a TMEM accumulator; tcgen05.commit
// releases each pipeline stage and finally signals the epilogue, which reads
// the accumulator with tcgen05.ld.
//
// Source of the layer: vLLM recipe page "inclusionAI/Ling-3.0-flash"
// ("Single-GPU int4": symmetric W4, group 32; "Launching the Server":
// chunked prefill) and the bpdata article "Harom optimalizacio a
// Ling-3.0-flash MoE inferenciajanak" ("Modell es kiindulo konfiguracio").
#include "common.cuh"
#include "grouped_tc.h"

namespace lingmoe {

constexpr int kTcThreads = 160;      // warps 0-3: producers + epilogue, warp 4: MMA issue
constexpr int kTcStages = 4;
constexpr int kTcM = 128;            // weight rows per tile
constexpr int kTcN = 128;            // tokens per tile (max)
constexpr int kTcK = 64;             // K per stage (one 128-byte swizzle row of fp16)
constexpr int kStageA = kTcM * kTcK * 2;  // 16 KB
constexpr int kStageB = kTcN * kTcK * 2;  // 16 KB per B part
constexpr int kTmemCols = 128;
// B parts per stage: gate/up reads x (exact in fp16), down reads h as the two
// fp16 terms hi + lo, so that h keeps ~22 bits through the contraction.
__host__ __device__ constexpr int tc_bparts(int mode) { return mode == 0 ? 1 : 2; }
__host__ __device__ constexpr size_t tc_smem(int mode) {
  return 1024 /*align slack*/ + (size_t)kTcStages * (kStageA + tc_bparts(mode) * kStageB) + 1024;
}
constexpr unsigned long long kTcWaitNs = 2000000000ull;

// K order inside each group of 8 elements: position p holds element kPerm[p];
// kInvPerm maps an element to its position.  It is the order in which
// (w >> 4s) & 0x000F000F yields nibble pairs (e_s, e_{s+4}).
__host__ __device__ constexpr int perm_pos(int o) { return (o < 4) ? 2 * o : 2 * (o - 4) + 1; }

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  // K-major, 128B swizzle: 8-row atoms of 128 B, atoms 1024 B apart (SBO),
  // LBO unused (1), descriptor version 1, layout type 2.
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ uint32_t make_idesc(int n) {
  // D = f32, A = B = f16, both K-major, M = 128, N = n
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTcM >> 4) << 24);
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
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
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

// Two exact fp16 weights q*s from a nibble pair (1024 + n in each half):
// v - 1032 = q is exact, and so is q * s (q has at most 4 significant bits,
// s at most 8).  Folding the bias into one fma would round -1032 * s.
__device__ __forceinline__ uint32_t deq_pair(uint32_t v, __half2 s2, __half2 b2) {
  const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&v), b2);
  const __half2 r = __hmul2(q, s2);
  return *reinterpret_cast<const uint32_t*>(&r);
}
// 32 codes (16 bytes, offset-binary nibbles) of one group with scale s ->
// 32 fp16 in permuted K order, written as 4 x 16 bytes to dst chunks.
__device__ __forceinline__ void deq_group(uint4 q, float s, uint4 out[4]) {
  const __half sh = __float2half_rn(s);
  const __half2 s2 = __halves2half2(sh, sh);
  const __half bh = __float2half_rn(1032.0f);
  const __half2 b2 = __halves2half2(bh, bh);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t p[4];
#pragma unroll
    for (int sft = 0; sft < 4; ++sft) {
      uint32_t v;
      asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(v) : "r"(w[i] >> (4 * sft)));
      p[sft] = deq_pair(v, s2, b2);  // (e_sft, e_{sft+4}) -> positions 2 sft, 2 sft + 1
    }
    out[i] = make_uint4(p[0], p[1], p[2], p[3]);
  }
}

// ---------------------------------------------------------------- x -> fp16 (permuted)
// x [T, H] bf16 -> x16 [T, H] fp16 in the permuted K order, scaled by
// 2^-sigma_t so that max|x_t| stays inside fp16; xscale[t] = 2^sigma_t.
__global__ void __launch_bounds__(256) x16_kernel(const __nv_bfloat16* __restrict__ x, int T,
                                                  __half* __restrict__ x16, float* __restrict__ xscale) {
  const int t = blockIdx.x;
  if (t >= T) return;
  __shared__ uint32_t smax;
  if (threadIdx.x == 0) smax = 0;
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * kH);
  for (int c = threadIdx.x; c < kH / 8; c += blockDim.x) {
    const uint4 w = src[c];
    const float m = fmaxf(fmaxf(fmaxf(fabsf(bf16lo(w.x)), fabsf(bf16hi(w.x))), fmaxf(fabsf(bf16lo(w.y)), fabsf(bf16hi(w.y)))),
                          fmaxf(fmaxf(fabsf(bf16lo(w.z)), fabsf(bf16hi(w.z))), fmaxf(fabsf(bf16lo(w.w)), fabsf(bf16hi(w.w)))));
    atomicMax(&smax, __float_as_uint(fminf(m, 3.0e38f)));
  }
  __syncthreads();
  const int e = (int)(smax >> 23) - 127;
  const int sigma = e >= 14 ? e - 13 : 0;
  const float inv = __uint_as_float((uint32_t)(127 - sigma) << 23);
  if (threadIdx.x == 0) xscale[t] = __uint_as_float((uint32_t)(127 + sigma) << 23);
  uint4* dst = reinterpret_cast<uint4*>(x16 + (size_t)t * kH);
  for (int c = threadIdx.x; c < kH / 8; c += blockDim.x) {
    const uint4 w = src[c];
    const float f[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                        bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
    __half h[8];
#pragma unroll
    for (int o = 0; o < 8; ++o) h[perm_pos(o)] = __float2half_rn(f[o] * inv);
    dst[c] = *reinterpret_cast<const uint4*>(h);
  }
}

// ---------------------------------------------------------------- tile lists
// One thread: tiles (expert, m-tile, first token position, tokens) in expert
// order, for both GEMMs.
__global__ void tc_tiles_kernel(const int32_t* cnt, const int32_t* off, int E, int4* gu_tiles, int4* dn_tiles,
                                int32_t* ntiles) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int ng = 0, nd = 0;
  for (int e = 0; e < E; ++e) {
    const int m = cnt[e];
    for (int n0 = 0; n0 < m; n0 += kTcN) {
      const int n = min(kTcN, m - n0);
      for (int mt = 0; mt < kI * 2 / kTcM; ++mt) gu_tiles[ng++] = make_int4(e, mt, off[e] + n0, n);
      for (int mt = 0; mt < kH / kTcM; ++mt) dn_tiles[nd++] = make_int4(e, mt, off[e] + n0, n);
    }
  }
  ntiles[0] = ng;
  ntiles[1] = nd;
}

// ---------------------------------------------------------------- the GEMM
// MODE 0: gate/up (A = gate/up rows interleaved: tile row 2j = gate, 2j+1 = up
// of intermediate row 64*mt + j; B = x16 rows of the tile's tokens; output h16
// [positions, 768] fp16 in permuted K order).
// MODE 1: down (A = down rows 128*mt..+127; B = the hi and lo halves of the
// h16 rows, both accumulated into one TMEM tile; output y [positions, 2560]
// fp32 scaled by the pair's routing weight).
template <int MODE>
__global__ void __launch_bounds__(kTcThreads, 1) tc_grouped_kernel(TcParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw_tc[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw_tc) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = smem;
  constexpr int NB = tc_bparts(MODE);
  unsigned char* sB = smem + kTcStages * kStageA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kTcStages * NB * kStageB);
  uint64_t* empty = full + kTcStages;
  uint64_t* accf = empty + kTcStages;
  uint64_t* acce = accf + 1;
  uint64_t* drain = acce + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int KTOT = MODE == 0 ? kH : kI;
  constexpr int NK = KTOT / kTcK;
  const int4* tiles = MODE == 0 ? p.gu_tiles : p.dn_tiles;
  const int ntiles = p.ntiles[MODE];

  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    mbar_init(acce, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int g = 0;     // global stage counter (same sequence in every role)
  int tj = 0;    // tiles done by this CTA
  for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x, ++tj) {
    const int4 tl = tiles[ti];
    const int e = tl.x, mt = tl.y, pos0 = tl.z, nrow = tl.w;
    const int nmma = (nrow + 15) & ~15;  // N of the MMA: multiple of 16, >= 16
    if (warp < 4) {
      // ------------------------------------------------ producers
      const int r = tid;  // A row and B row handled by this thread
      // A source for row r
      const uint8_t* abase;
      int alane;
      if (MODE == 0) {
        const int i = 64 * mt + (r >> 1);          // intermediate row
        const int rin = (r & 1) ? 4 + (i & 3) : (i & 3);  // row within the unit (gate 0-3, up 4-7)
        abase = p.gu + ((size_t)e * kGuUnits + (i >> 2)) * kGuUnitBytes;
        alane = rin;                                 // + 8 * quarter, below
      } else {
        const int n = kTcM * mt + r;                 // output row
        abase = p.dn + ((size_t)e * kDnUnits + (n >> 2)) * kDnUnitBytes;
        alane = n & 3;                               // + 4 * slice, below
      }
      // B source for row r (token or position)
      const bool bvalid = r < nrow;
      const unsigned char* bsrc;
      if (MODE == 0) {
        const int tok = bvalid ? p.perm[pos0 + r] / p.k : 0;
        bsrc = reinterpret_cast<const unsigned char*>(p.x16 + (size_t)tok * kH);
      } else {
        bsrc = reinterpret_cast<const unsigned char*>(p.h16 + (size_t)(pos0 + (bvalid ? r : 0)) * 2 * kI);
      }
      for (int kk = 0; kk < NK; ++kk, ++g) {
        const int s = g % kTcStages;
        if (!tc_wait(&empty[s], ((g / kTcStages) & 1) ^ 1, p.err, abort_flag)) break;
        // two groups of 32 codes: groups 2kk, 2kk+1 of this row
        uint4 outv[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int G = 2 * kk + h;
          uint4 q;
          float sc;
          if (MODE == 0) {
            const int quarter = G / kGuChunks, j = G - quarter * kGuChunks, ln = alane + 8 * quarter;
            q = *reinterpret_cast<const uint4*>(abase + j * 512 + 16 * ln);
            sc = bf16_to_f32(*reinterpret_cast<const unsigned short*>(abase + kGuScaleOff + (j >> 2) * 256 + 8 * ln + 2 * (j & 3)));
          } else {
            const int slice = G / kDnChunks, j = G - slice * kDnChunks, ln = alane + 4 * slice;
            q = *reinterpret_cast<const uint4*>(abase + j * 512 + 16 * ln);
            sc = bf16_to_f32(*reinterpret_cast<const unsigned short*>(abase + kDnScaleOff + j * 64 + 2 * ln));
          }
          deq_group(q, sc, outv + 4 * h);
        }
        unsigned char* a = sA + s * kStageA + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(a + ((c ^ (r & 7)) << 4)) = outv[c];
#pragma unroll
        for (int part = 0; part < NB; ++part) {
          unsigned char* b = sB + (s * NB + part) * kStageB + r * 128;
          const uint4* bs = reinterpret_cast<const uint4*>(bsrc + part * 2 * kI + kk * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(b + ((c ^ (r & 7)) << 4)) = bvalid ? bs[c] : make_uint4(0, 0, 0, 0);
        }
        fence_async_smem();
        mbar_arrive(&full[s]);
      }
      // ------------------------------------------------ epilogue
      if (!tc_wait(accf, tj & 1, p.err, abort_flag)) break;
      tc_fence_after();
      const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
      for (int c0 = 0; c0 < nmma; c0 += 16) {
        float v[16];
        tmem_ld16(trow + c0, v);
        if (MODE == 0) {
          const int rr = warp * 32 + lane, j = rr >> 1, i = 64 * mt + j;
          const int ip = (i & ~7) + perm_pos(i & 7);
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {
            const float other = __shfl_xor_sync(0xffffffffu, v[cc], 1);
            const int col = c0 + cc;
            if (!(lane & 1) && col < nrow) {
              const int pos = pos0 + col;
              const float xs = p.xscale[p.perm[pos] / p.k];
              const float hv = silu_mul(v[cc] * xs, other * xs);
              const __half hi = __float2half_rn(hv);
              p.h16[(size_t)pos * 2 * kI + ip] = hi;
              p.h16[(size_t)pos * 2 * kI + kI + ip] = __float2half_rn(hv - __half2float(hi));
            }
          }
        } else {
          const int n = kTcM * mt + warp * 32 + lane;
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {
            const int col = c0 + cc;
            if (col < nrow) {
              const int pos = pos0 + col;
              p.y[(size_t)pos * kH + n] = v[cc] * p.topk_w[p.perm[pos]];
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acce);
    } else {
      // ------------------------------------------------ MMA issue (one thread)
      bool ok = true;
      if (lane == 0) {
        if (tj > 0) ok = tc_wait(acce, (tj - 1) & 1, p.err, abort_flag);
        tc_fence_after();
        const uint32_t idesc = make_idesc(nmma);
        for (int kk = 0; kk < NK && ok; ++kk, ++g) {
          const int s = g % kTcStages;
          if (!tc_wait(&full[s], (g / kTcStages) & 1, p.err, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kStageA), b0 = smem_u32(sB + s * NB * kStageB);
#pragma unroll
          for (int k4 = 0; k4 < kTcK / 16; ++k4)
#pragma unroll
            for (int part = 0; part < NB; ++part)
              tc_mma(tmem, sw128_desc(a0 + 32 * k4), sw128_desc(b0 + part * kStageB + 32 * k4), idesc,
                     (kk | k4 | part) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(accf);
      }
      g = __shfl_sync(0xffffffffu, g, 0);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
    }
    if (*reinterpret_cast<volatile int*>(abort_flag)) break;
  }
  // teardown: no MMA may still be writing TMEM when it is freed
  if (warp == 4 && lane == 0) {
    tc_commit(drain);
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kTcWaitNs) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
}

size_t tc_smem_bytes() { return tc_smem(1); }

cudaError_t setup_grouped_tc() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(tc_grouped_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc_smem(0))) != cudaSuccess)
    return e;
  return cudaFuncSetAttribute(tc_grouped_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc_smem(1));
}

cudaError_t launch_x16(const __nv_bfloat16* x, int T, __half* x16, float* xscale, cudaStream_t s) {
  x16_kernel<<<T, 256, 0, s>>>(x, T, x16, xscale);
  return cudaGetLastError();
}

cudaError_t launch_tc_tiles(const int32_t* cnt, const int32_t* off, int E, int4* gu_tiles, int4* dn_tiles,
                            int32_t* ntiles, cudaStream_t s) {
  tc_tiles_kernel<<<1, 32, 0, s>>>(cnt, off, E, gu_tiles, dn_tiles, ntiles);
  return cudaGetLastError();
}

cudaError_t launch_tc_gemm(int mode, const TcParams& p, int nctas, cudaStream_t s) {
  if (mode == 0) tc_grouped_kernel<0><<<nctas, kTcThreads, tc_smem(0), s>>>(p);
  else tc_grouped_kernel<1><<<nctas, kTcThreads, tc_smem(1), s>>>(p);
  return cudaGetLastError();
}

}  // namespace lingmoe
