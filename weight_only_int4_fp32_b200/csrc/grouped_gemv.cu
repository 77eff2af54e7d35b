// Grouped path, GEMV side: routed experts that hold only 1..kGvMaxTok tokens of
// the call.  For them a dense tensor-core tile would be almost all padding, so
// their weights are streamed once and multiplied on the CUDA cores / mma.sync
// instead, with the decode path's machinery:
//   gate/up  a task is (expert, quarter of its 96 units); the CTA stages the
//            expert's x rows in MMA B-fragment order, and each warp pair runs
//            the two K halves of a unit: per 16x16 block one fragment word per
//            lane -> exact codes q (LOP3 + HSUB2) -> one m16n8k16 MMA whose
//            columns are the expert's tokens; per 32-K group the fp32 result is
//            scaled by the group's bf16 scale; SiLU(g) * u is written as the
//            fp16 hi + lo terms (times 2^-8) that the down GEMM reads.
//   down     a task is (expert, quarter of the output rows); the CTA stages
//            h as fp16 hi + lo A fragments, streams the 8-row down units
//            (double-buffered bulk copies) and runs them on mma.sync with the
//            expert's tokens as A rows; it writes w * (Wd h) per position.
// The tensor-core tiles (grouped_tc.cu) take the experts with more tokens and
// the shared expert; both write the same h16 / y buffers.
//
// Source of the layer: vLLM recipe page "inclusionAI/Ling-3.0-flash"
// ("Single-GPU int4": symmetric W4, group 32) and the bpdata article "Harom
// optimalizacio a Ling-3.0-flash MoE inferenciajanak" ("Modell es kiindulo
// konfiguracio").
#include "common.cuh"
#include "grouped_gemv.h"
#include "grouped_tc.h"

namespace lingmoe {

constexpr int kGvThreads = 384;
constexpr int kGvWarps = kGvThreads / 32;    // 12
constexpr int kGvPairs = kGvWarps / 2;       // 6
constexpr int kGvGuTasks = 4;                // gate/up tasks per expert
constexpr int kGvGuUnits = kGuUnits / kGvGuTasks;  // 24 units per task
constexpr int kGvGuRounds = kGvGuUnits / kGvPairs;  // 4
static_assert(kGvGuUnits % kGvPairs == 0, "a task's units split evenly over the warp pairs");
constexpr int kGvXfTok = (kH / 64) * 128;    // 5120 B per token in B-fragment order
constexpr int kGvPiece = kGuHalfCodes / 4;   // 2560 B
// gate/up shared memory: mbarriers [12][6] | x fragments [8][5120] | pair
// combine [6][2][32][4] floats | per warp: 4 code pieces + 2 scale slots
constexpr int kGvGuWarpBytes = 4 * kGvPiece + 2 * kGuHalfScales;  // 12800
constexpr size_t kGvGuXf = 1024;
constexpr size_t kGvGuComb = kGvGuXf + (size_t)kGvMaxTok * kGvXfTok;
constexpr size_t kGvGuBuf = kGvGuComb + (size_t)kGvPairs * 2 * 32 * 16;
constexpr size_t kGvGuSmem = kGvGuBuf + (size_t)kGvWarps * kGvGuWarpBytes;
static_assert(kGvGuSmem <= 227 * 1024, "GEMV gate/up shared memory over budget");

constexpr int kGvDnTasks = 4;                          // down tasks per expert: 80 units (640 rows)
constexpr int kGvDnChunks = 4;                         // streamed chunks per task
constexpr int kGvDnUnits = kDnUnits / (kGvDnTasks * kGvDnChunks);  // 20 units of 8 rows per chunk
constexpr int kGvDnThirds = 3;                         // a unit's K in thirds: 60 items per chunk
constexpr int kGvDnItems = kGvDnUnits * kGvDnThirds;
static_assert(kGvDnItems % kGvWarps == 0, "a chunk's items split evenly over the warps");
static_assert(kDnChunks % kGvDnThirds == 0, "a third of K is whole 128-K chunks");
// down shared memory: mbarriers [2 buffers][2 pieces] | h fragments [8 tokens]
// | partial sums [2][units][thirds][8 tokens][4 lanes][2] | 2 chunk buffers
constexpr size_t kGvDnHOff = 256;
constexpr size_t kGvDnPartOff = kGvDnHOff + (size_t)kGvMaxTok * kHfStride;
constexpr size_t kGvDnPartBytes = (size_t)kGvDnItems * kGvMaxTok * 8 * 4;  // 15360
constexpr size_t kGvDnUnitsOff = kGvDnPartOff + 2 * kGvDnPartBytes;
constexpr size_t kGvDnUnitsBytes = (size_t)kGvDnUnits * kDnUnitBytes;  // 69120
constexpr size_t kGvDnSmem = kGvDnUnitsOff + 2 * kGvDnUnitsBytes;
static_assert(kGvDnPartOff % 16 == 0 && kGvDnUnitsOff % 16 == 0 && kGvDnUnitsBytes % 16 == 0,
              "bulk copies need 16-byte alignment");
static_assert(kGvDnSmem <= 227 * 1024, "GEMV down shared memory over budget");

// ---------------------------------------------------------------- gate/up
// A warp walks rounds g = 0, 1, ... over its CTA's tasks (4 rounds per task);
// in round g it computes one K half of unit b(g).  Its buffer holds four
// pieces of 2560 B; as soon as piece pc of round g is consumed, piece pc of
// round g + 1 is requested into the same slot, and the scales of round g + 1
// go to the second of two scale slots, so the weights stream continuously.
// C: the codec of the routed weights (kCodecInt4 or kCodecMxfp4, layout.h).
template <int C>
__global__ void __launch_bounds__(kGvThreads, 1) gv_gu_kernel(const GvParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm);
  unsigned char* xf = sm + kGvGuXf;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pair = warp >> 1, half = warp & 1;
  float* comb = reinterpret_cast<float*>(sm + kGvGuComb) + (size_t)pair * (2 * 32 * 4);
  unsigned char* buf = sm + kGvGuBuf + (size_t)warp * kGvGuWarpBytes;  // 4 pieces, then 2 scale slots
  uint64_t* bar = mbar + warp * 6;  // [0..3] pieces, [4..5] scale slots
  if (lane == 0) {
    for (int i = 0; i < 6; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int ntask = *p.nsmall * kGvGuTasks;
  const int nmine = ntask > (int)blockIdx.x ? (ntask - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int nround = nmine * kGvGuRounds;
  // weights of round g for this warp
  auto unit_src = [&](int g) -> const uint8_t* {
    const int task = blockIdx.x + (g / kGvGuRounds) * gridDim.x;
    const int4 se = p.small[task / kGvGuTasks];
    const int b = (task % kGvGuTasks) * kGvGuUnits + pair + kGvPairs * (g % kGvGuRounds);
    return p.gu + ((size_t)se.x * kGuUnits + b) * kGuUnitBytes;
  };
  auto issue_scales = [&](int g) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar[4 + (g & 1)], kGuHalfScales);
      bulk_g2s(buf + 4 * kGvPiece + (g & 1) * kGuHalfScales, unit_src(g) + kGuScaleOff + half * kGuHalfScales,
               kGuHalfScales, &bar[4 + (g & 1)]);
    }
  };
  auto issue_piece = [&](int g, int pc) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar[pc], kGvPiece);
      bulk_g2s(buf + pc * kGvPiece, unit_src(g) + half * kGuHalfCodes + pc * kGvPiece, kGvPiece, &bar[pc]);
    }
  };
  bool dead = false;  // a wait ran out: no further copies, barriers still met
  if (nround > 0) {
    issue_scales(0);
    for (int pc = 0; pc < 4; ++pc) issue_piece(0, pc);
  }
  const int n = lane >> 2, mm = lane & 3;  // B column (token of the expert) / lane class
  int pos0 = 0, m = 0, q4 = 0;
#pragma unroll 1
  for (int g = 0; g < nround; ++g) {
    const int r = g % kGvGuRounds;
    if (r == 0) {
      const int task = blockIdx.x + (g / kGvGuRounds) * gridDim.x;
      const int4 se = p.small[task / kGvGuTasks];
      pos0 = se.y;
      m = se.z;
      q4 = task % kGvGuTasks;
      __syncthreads();  // the previous task is done with xf
      // x rows of the expert's positions in B-fragment order: per 16-K block kb
      // and lane class mm, (x[c], x[c+1]) and (x[c+8], x[c+9]), c = 16 kb + 2 mm;
      // int4: the second pair / 16 (it meets codes dequantised as 16 q)
      for (int v = tid; v < m * (kH / 4); v += kGvThreads) {
        const int t = v / (kH / 4), rr = v - t * (kH / 4), kb = rr >> 2, c = 16 * kb + 2 * (rr & 3);
        const __half* row = p.xg + (size_t)(pos0 + t) * kH;
        const uint32_t lo = *reinterpret_cast<const uint32_t*>(row + c);
        const __half2 hi = C == kCodecInt4
                               ? __hmul2(*reinterpret_cast<const __half2*>(row + c + 8), __float2half2_rn(0.0625f))
                               : *reinterpret_cast<const __half2*>(row + c + 8);
        *reinterpret_cast<uint2*>(xf + t * kGvXfTok + (kb >> 2) * 128 + (rr & 3) * 32 + (kb & 3) * 8) =
            make_uint2(lo, *reinterpret_cast<const uint32_t*>(&hi));
      }
      __syncthreads();
    }
    const bool more = !dead && g + 1 < nround;
    if (more) issue_scales(g + 1);  // its slot was last used by round g - 1
    const bool bval = n < m;
    const unsigned char* xrow = xf + (bval ? n : 0) * kGvXfTok + mm * 32 + half * (kGuChunks / 2) * 128;
    const unsigned char* sc = buf + 4 * kGvPiece + (g & 1) * kGuHalfScales;
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
    bool ok = !dead && mbar_wait_warp(&bar[4 + (g & 1)], (uint32_t)((g >> 1) & 1), p.wait_limit_ns, p.err);
#pragma unroll 1
    for (int pc = 0; pc < 4 && ok; ++pc) {
      ok = mbar_wait_warp(&bar[pc], (uint32_t)(g & 1), p.wait_limit_ns, p.err);
      if (!ok) break;
#pragma unroll
      for (int jj = 0; jj < kGuChunks / 8; ++jj) {
        const int jl = pc * (kGuChunks / 8) + jj;
        const uint4 wv = lds128(buf + jl * 512 + 16 * lane);
        const uint4 xa = lds128(xrow + jl * 128);  // a column without a token reads token 0
        const uint4 xc = lds128(xrow + jl * 128 + 16);
        const uint32_t s01 = *reinterpret_cast<const uint32_t*>(sc + (2 * jl) * 32 + 4 * n);
        const uint32_t s23 = *reinterpret_cast<const uint32_t*>(sc + (2 * jl + 1) * 32 + 4 * n);
        const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
        const uint32_t bx[8] = {xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w};
        float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t a0, a1, a2, a3;
          if constexpr (C == kCodecMxfp4) {
            a0 = deq_e2m1<0>(wd[w]);
            a2 = deq_e2m1<4>(wd[w]);
            a1 = deq_e2m1<8>(wd[w]);
            a3 = deq_e2m1<12>(wd[w]);
          } else {
            a0 = deq_q_even(wd[w]);
            a2 = deq_q_odd16(wd[w]);
            a1 = deq_q_even(wd[w] >> 8);
            a3 = deq_q_odd16(wd[w] >> 8);
          }
          if (w & 1) {
            mma_16816(d0, d1, d2, d3, a0, a1, a2, a3, bx[2 * w], bx[2 * w + 1], d0, d1, d2, d3);
            const uint32_t sw = (w == 1) ? s01 : s23;
            const float sg = bf16lo(sw), su = bf16hi(sw);
            acc0 = fmaf(sg, d0, acc0);
            acc1 = fmaf(sg, d1, acc1);
            acc2 = fmaf(su, d2, acc2);
            acc3 = fmaf(su, d3, acc3);
          } else {
            mma_16816(d0, d1, d2, d3, a0, a1, a2, a3, bx[2 * w], bx[2 * w + 1], 0.f, 0.f, 0.f, 0.f);
          }
        }
      }
      __syncwarp();  // every lane is done with piece pc
      if (more) issue_piece(g + 1, pc);
    }
    if (!ok && !dead) {
      dead = true;
      if (lane == 0) {  // copies of this and the next round may still be landing: wait (bounded)
        mbar_wait(&bar[4 + (g & 1)], (uint32_t)((g >> 1) & 1), p.wait_limit_ns, p.err);
        for (int pc = 0; pc < 4; ++pc) mbar_wait(&bar[pc], (uint32_t)(g & 1), p.wait_limit_ns, p.err);
        if (more) {
          mbar_wait(&bar[4 + ((g + 1) & 1)], (uint32_t)(((g + 1) >> 1) & 1), p.wait_limit_ns, p.err);
        }
      }
      __syncwarp();
    }
    // the two K halves meet in shared memory (double-buffered by round parity)
    float* cb = comb + (g & 1) * (32 * 4) + lane * 4;
    if (half == 1) *reinterpret_cast<float4*>(cb) = make_float4(acc0, acc1, acc2, acc3);
    asm volatile("bar.sync %0, %1;" :: "r"(1 + pair), "r"(64) : "memory");
    const bool pair_dead = __shfl_sync(0xffffffffu, dead, 0);
    if (half == 0 && !pair_dead) {
      const float4 o = *reinterpret_cast<const float4*>(cb);
      acc0 += o.x;
      acc1 += o.y;
      acc2 += o.z;
      acc3 += o.w;
      const int b = q4 * kGvGuUnits + pair + kGvPairs * r;
      const int i = 8 * b + n;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int col = 2 * mm + cc;
        if (col < m) {
          const int pos = pos0 + col;
          // h / c_t^2 (the tensor-core tiles' convention), then the fp16 shift
          const float xs = p.xscale[p.perm[pos] / p.k];
          const float hv = silu_mul_scaled(cc ? acc1 : acc0, cc ? acc3 : acc2, xs) *
                           (1.f / (float)(1 << kTcScaleShift)) * (1.f / (float)(1 << (2 * kGrpUnitShift)));
          const __half hh = __float2half_rn(hv);
          __half* dst = p.h16 + (size_t)pos * (2 * kI) + i;
          dst[0] = hh;
          dst[kI] = __float2half_rn(hv - __half2float(hh));
        }
      }
    }
  }
}

// ---------------------------------------------------------------- down
// A task is a quarter of an expert's output rows (80 units of 8 rows); h is
// staged once per task as MMA A fragments.  The CTA walks its tasks as a flat
// sequence of 20-unit chunks through two buffers: while one chunk is
// computed, the next one (possibly of the next task) streams into the other.
// A chunk is 60 items (unit, third of K) spread evenly over the 12 warps;
// the three partial sums of a row meet in shared memory in a fixed order.
__device__ __forceinline__ void gv_dn_issue(const GvParams& p, int gc, unsigned char* sm) {
  const int task = blockIdx.x + (gc / kGvDnChunks) * gridDim.x;
  const int4 se = p.small[task / kGvDnTasks];
  const int v0 = (task % kGvDnTasks) * (kGvDnChunks * kGvDnUnits) + (gc % kGvDnChunks) * kGvDnUnits;
  const uint8_t* src = p.dn + ((size_t)se.x * kDnUnits + v0) * kDnUnitBytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm) + 2 * (gc & 1);
  unsigned char* dst = sm + kGvDnUnitsOff + (size_t)(gc & 1) * kGvDnUnitsBytes;
  constexpr uint32_t kPieceBytes = (kGvDnUnits / 2) * kDnUnitBytes;
  for (int pc = 0; pc < 2; ++pc) {
    mbar_arrive_expect_tx(&bar[pc], kPieceBytes);
    bulk_g2s(dst + pc * kPieceBytes, src + pc * kPieceBytes, kPieceBytes, &bar[pc]);
  }
}

template <int C>
__global__ void __launch_bounds__(kGvThreads, 1) gv_dn_kernel(const GvParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm);  // [buffer][piece]
  unsigned char* hf = sm + kGvDnHOff;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&mbar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int ntask = *p.nsmall * kGvDnTasks;
  const int nmine = ntask > (int)blockIdx.x ? (ntask - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int nchunk = nmine * kGvDnChunks;
  const int g = lane >> 2, c = lane & 3;  // token (A row) / lane class
  int dead = 0;
  if (tid == 0 && nchunk > 0) gv_dn_issue(p, 0, sm);
  int pos0 = 0, m = 0;
#pragma unroll 1
  for (int gc = 0; gc < nchunk; ++gc) {
    const int task = blockIdx.x + (gc / kGvDnChunks) * gridDim.x;
    if (gc % kGvDnChunks == 0) {
      const int4 se = p.small[task / kGvDnTasks];
      pos0 = se.y;
      m = se.z;
      // h of the expert's positions (fp16 hi + lo, natural K order) into A
      // fragments: per (token, 16-K block, lane class) 4 words
      for (int v = tid; v < m * (kI / 4); v += kGvThreads) {
        const int t = v / (kI / 4), r = v - t * (kI / 4), k = 16 * (r >> 2) + 2 * (r & 3);
        const __half* row = p.h16 + (size_t)(pos0 + t) * (2 * kI);
        const uint32_t hi0 = *reinterpret_cast<const uint32_t*>(row + k);
        const uint32_t lo0 = *reinterpret_cast<const uint32_t*>(row + kI + k);
        const uint32_t hi8 = *reinterpret_cast<const uint32_t*>(row + k + 8);
        const uint32_t lo8 = *reinterpret_cast<const uint32_t*>(row + kI + k + 8);
        *reinterpret_cast<uint4*>(hf + (size_t)t * kHfStride + hf_off(k)) = make_uint4(hi0, lo0, hi8, lo8);
      }
      __syncthreads();
    }
    // the next chunk streams into the other buffer (its last chunk is done:
    // every warp passed the barrier at the end of the previous iteration)
    if (tid == 0 && gc + 1 < nchunk && !dead) gv_dn_issue(p, gc + 1, sm);
    const unsigned char* units = sm + kGvDnUnitsOff + (size_t)(gc & 1) * kGvDnUnitsBytes;
    float* part = reinterpret_cast<float*>(sm + kGvDnPartOff + (size_t)(gc & 1) * kGvDnPartBytes);
    const uint32_t par = (uint32_t)((gc >> 1) & 1);
    const bool act = g < m;
    const unsigned char* hfl = hf + (size_t)(act ? g : 0) * kHfStride + 16 * c;
#pragma unroll 1
    for (int it = warp; it < kGvDnItems && !dead; it += kGvWarps) {
      const int u = it / kGvDnThirds, th = it - u * kGvDnThirds;
      if (!mbar_wait_warp(&mbar[2 * (gc & 1) + u / (kGvDnUnits / 2)], par, p.wait_limit_ns, p.err)) {
        dead = 1;
        break;
      }
      float r0, r1;
      constexpr int kJ = kDnChunks / kGvDnThirds;
      dn_unit_mma<C>(units + (size_t)u * kDnUnitBytes, hfl, lane, r0, r1, kJ * th, kJ * th + kJ);
      if (act) *reinterpret_cast<float2*>(part + ((size_t)it * kGvMaxTok + g) * 8 + 2 * c) = make_float2(r0, r1);
    }
    dead = __syncthreads_or(dead);
    if (dead) {
      // a wait ran out: let every copy issued so far land (bounded) before leaving
      if (tid == 0) {
        for (int pc = 0; pc < 2; ++pc) mbar_wait(&mbar[2 * (gc & 1) + pc], par, p.wait_limit_ns, p.err);
        if (gc + 1 < nchunk)  // the next chunk was issued into the other buffer
          for (int pc = 0; pc < 2; ++pc)
            mbar_wait(&mbar[2 * ((gc + 1) & 1) + pc], (uint32_t)(((gc + 1) >> 1) & 1), p.wait_limit_ns, p.err);
      }
      break;
    }
    // the thirds of K add up in a fixed order; y = w * 2^8 * sum per position
    const int v0 = (task % kGvDnTasks) * (kGvDnChunks * kGvDnUnits) + (gc % kGvDnChunks) * kGvDnUnits;
    for (int v = tid; v < kGvDnUnits * m * kDnUnitRows; v += kGvThreads) {
      const int u = v / (m * kDnUnitRows), rem = v - u * (m * kDnUnitRows), t = rem >> 3, r = rem & 7;
      const float* pp = part + ((size_t)(u * kGvDnThirds) * kGvMaxTok + t) * 8 + r;
      const float sum = (pp[0] + pp[kGvMaxTok * 8]) + pp[2 * kGvMaxTok * 8];
      const int pos = pos0 + t;
      p.y[(size_t)pos * kH + kDnUnitRows * (v0 + u) + r] =
          (float)(1 << kHShift) * sum * p.topk_w[p.perm[pos]];
    }
  }
}

template <int C>
static cudaError_t setup_c() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(gv_gu_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGvGuSmem)) !=
      cudaSuccess)
    return e;
  return cudaFuncSetAttribute(gv_dn_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGvDnSmem);
}

cudaError_t setup_grouped_gemv() {
  const cudaError_t e = setup_c<kCodecInt4>();
  return e != cudaSuccess ? e : setup_c<kCodecMxfp4>();
}

cudaError_t launch_gemv_gu(const GvParams& p, int nctas, cudaStream_t s) {
  if (p.codec == kCodecMxfp4) gv_gu_kernel<kCodecMxfp4><<<nctas, kGvThreads, kGvGuSmem, s>>>(p);
  else gv_gu_kernel<kCodecInt4><<<nctas, kGvThreads, kGvGuSmem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemv_dn(const GvParams& p, int nctas, cudaStream_t s) {
  if (p.codec == kCodecMxfp4) gv_dn_kernel<kCodecMxfp4><<<nctas, kGvThreads, kGvDnSmem, s>>>(p);
  else gv_dn_kernel<kCodecInt4><<<nctas, kGvThreads, kGvDnSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace lingmoe
