// Decode / verify path (1 <= T <= kMaxDecodeT) of the W4 g32 MoE layer.
//
// One persistent launch per call, one CTA per SM, co-resident (cooperative
// launch).  The work is a chain router -> top-k -> routed gate/up -> down,
// so the CTAs meet at three bounded grid barriers:
//
//   phase 1  router logits (bf16 GEMV, fp32)            -> barrier A
//   phase 2  shared-expert gate/up + SiLU*up (bf16)     -> barrier B
//   phase 3  wait A; every CTA selects the top-k itself; routed gate/up
//            (W4 g32, dequantised in registers) + SiLU*up -> barrier C
//   phase 4  wait B, C; routed down (W4 g32) weighted by the routing weights,
//            shared down (bf16), summed in a fixed order, one bf16 rounding.
//
// Bytes that do not depend on the routing (shared expert) are prefetched into
// L2 at the start, and the routed down weights as soon as the routing is
// known, so HBM keeps streaming across the barriers.
//
// Layer definition: vLLM recipe page "inclusionAI/Ling-3.0-flash" (Overview;
// "Single-GPU int4": symmetric W4, group 32, routed experts only) and the
// bpdata article "Harom optimalizacio a Ling-3.0-flash MoE inferenciajanak"
// ("Modell es kiindulo konfiguracio": 8 of 512 routed experts + 1 shared).
#include "common.cuh"
#include "decode.h"

namespace lingmoe {

// ---------------------------------------------------------------- smem plan
constexpr int kMaxPairs = kMaxDecodeT * kMaxTopK;      // 32
constexpr int kMaxBlkPerCta = 8;                       // down row-blocks per CTA (>= 640 / nctas)

struct __align__(16) SmemHeader {
  int topi[kMaxDecodeT][kMaxTopK];
  float topw[kMaxDecodeT][kMaxTopK];
  int nuniq;
  int uniq_e[kMaxPairs];
  int uniq_cnt[kMaxPairs];
  int uniq_pair[kMaxPairs][kMaxDecodeT];
  int flag;
};

constexpr size_t kPhase13Floats = (size_t)kMaxDecodeT * kXTok + kMaxDecodeT * kXGroups;
constexpr size_t kPhase4Floats = (size_t)kMaxPairs * kHpStride + kMaxPairs * kHGroups +
                                 (size_t)kMaxDecodeT * kHsTok +
                                 (size_t)kMaxBlkPerCta * (kMaxPairs + kMaxDecodeT) * 4;
constexpr size_t kBodyFloats = kPhase13Floats > kPhase4Floats ? kPhase13Floats : kPhase4Floats;
constexpr size_t kDecodeSmemBytes = sizeof(SmemHeader) + kBodyFloats * sizeof(float);

size_t decode_smem_bytes() { return kDecodeSmemBytes; }

// ---------------------------------------------------------------- helpers
// ---------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kDecodeThreads, 1)
moe_decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SmemHeader& hd = *reinterpret_cast<SmemHeader*>(smem_raw);
  float* body = reinterpret_cast<float*>(smem_raw + sizeof(SmemHeader));

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cta = blockIdx.x, ncta = gridDim.x;
  const int T = p.T, E = p.E, K = p.k;

  // barrier generations (read before this CTA arrives anywhere)
  const unsigned long long genA = ld_acquire_u64(p.bar + 0) / ncta;
  const unsigned long long genB = ld_acquire_u64(p.bar + 1) / ncta;
  const unsigned long long genC = ld_acquire_u64(p.bar + 2) / ncta;
  const bool skip = (cta == p.skip_arrive_cta);

  // this CTA's slices
  const int r0 = (int)((long long)cta * E / ncta), r1 = (int)((long long)(cta + 1) * E / ncta);
  const int s0 = cta * kI / ncta, s1 = (cta + 1) * kI / ncta;
  const int b0 = cta * kDnUnits / ncta, b1 = (cta + 1) * kDnUnits / ncta;
  const int nblk = b1 - b0;

  // L2 prefetch of routing-independent bytes: shared gate/up rows, shared down rows
  if (warp == kDecodeWarps - 1) {
    const uint32_t row_bytes = kH * 2;
    for (int i = s0 + lane; i < s1; i += 32) {
      prefetch_l2_bulk(p.sh_gate + (size_t)i * kH, row_bytes);
      prefetch_l2_bulk(p.sh_up + (size_t)i * kH, row_bytes);
    }
    if (lane == 0 && nblk > 0)
      prefetch_l2_bulk(p.sh_down + (size_t)b0 * 4 * kI, (uint32_t)nblk * 4 * kI * 2);
  }

  // ---- stage x (fp32 planes) and the group sums
  float* xs = body;
  float* cx = body + (size_t)kMaxDecodeT * kXTok;
  for (int v = tid; v < T * kXChunks; v += kDecodeThreads) {
    const int t = v / kXChunks, c = v - t * kXChunks;
    const uint4 w = *reinterpret_cast<const uint4*>(p.x + (size_t)t * kH + 8 * c);
    float* d = xs + (size_t)t * kXTok + xoff(c);
    *reinterpret_cast<float4*>(d) = make_float4(bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y));
    *reinterpret_cast<float4*>(d + kXPlane) =
        make_float4(bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w));
  }
  __syncthreads();
  for (int v = tid; v < T * kXGroups; v += kDecodeThreads) {
    const int t = v / kXGroups, G = v - t * kXGroups;
    const float* xt = xs + (size_t)t * kXTok;
    float s = 0.f;
    for (int i = 0; i < 4; ++i) {
      const int c = 4 * G + i;
      const float4 a = *reinterpret_cast<const float4*>(xt + xoff(c));
      const float4 b = *reinterpret_cast<const float4*>(xt + kXPlane + xoff(c));
      s += a.x + a.y + a.z + a.w + b.x + b.y + b.z + b.w;
    }
    cx[t * kXGroups + G] = kBiasCoef * s;
  }
  __syncthreads();

  // ---- phase 1: router logits for rows [r0, r1)
  for (int e = r0 + warp; e < r1; e += kDecodeWarps) {
    const __nv_bfloat16* wr = p.router_w + (size_t)e * kH;
    uint4 w[kXChunks / 32];
#pragma unroll
    for (int m = 0; m < kXChunks / 32; ++m) w[m] = ldg_stream(wr + 8 * (lane + 32 * m));
    const float bias = p.router_bias ? p.router_bias[e] : 0.f;
    float acc[kMaxDecodeT];
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) acc[t] = 0.f;
#pragma unroll
    for (int m = 0; m < kXChunks / 32; ++m) {
      const int o = xoff(lane + 32 * m);
#pragma unroll
      for (int t = 0; t < kMaxDecodeT; ++t) {
        if (t < T) {
          const float* xt = xs + (size_t)t * kXTok + o;
          acc[t] = dot8_bf16(w[m], *reinterpret_cast<const float4*>(xt),
                             *reinterpret_cast<const float4*>(xt + kXPlane), acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) {
      if (t < T) {
        const float v = warp_sum(acc[t]);
        if (lane == 0) p.logits[(size_t)t * E + e] = v + bias;
      }
    }
  }
  grid_arrive(p.bar + 0, skip);

  // ---- phase 2: shared expert gate/up rows [s0, s1)
  for (int i = s0 + warp; i < s1; i += kDecodeWarps) {
    const __nv_bfloat16* wg = p.sh_gate + (size_t)i * kH;
    const __nv_bfloat16* wu = p.sh_up + (size_t)i * kH;
    uint4 g[kXChunks / 32], u[kXChunks / 32];
#pragma unroll
    for (int m = 0; m < kXChunks / 32; ++m) {
      g[m] = ldg_stream(wg + 8 * (lane + 32 * m));
      u[m] = ldg_stream(wu + 8 * (lane + 32 * m));
    }
    float ag[kMaxDecodeT], au[kMaxDecodeT];
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) ag[t] = au[t] = 0.f;
#pragma unroll
    for (int m = 0; m < kXChunks / 32; ++m) {
      const int o = xoff(lane + 32 * m);
#pragma unroll
      for (int t = 0; t < kMaxDecodeT; ++t) {
        if (t < T) {
          const float* xt = xs + (size_t)t * kXTok + o;
          const float4 a = *reinterpret_cast<const float4*>(xt);
          const float4 b = *reinterpret_cast<const float4*>(xt + kXPlane);
          ag[t] = dot8_bf16(g[m], a, b, ag[t]);
          au[t] = dot8_bf16(u[m], a, b, au[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) {
      if (t < T) {
        const float vg = warp_sum(ag[t]);
        const float vu = warp_sum(au[t]);
        if (lane == 0) p.h_s[(size_t)t * kI + i] = silu_mul(vg, vu);
      }
    }
  }
  grid_arrive(p.bar + 1, skip);

  // ---- phase 3: routing (every CTA, redundantly), then routed gate/up
  if (!grid_wait(p.bar + 0, (genA + 1) * ncta, p.wait_limit_ns, p.err, &hd.flag)) return;
  if (warp < T) warp_topk(p.logits + (size_t)warp * E, E, K, hd.topi[warp], hd.topw[warp]);
  __syncthreads();
  if (warp == 0) {
    // union of the selected experts, in first-occurrence order (t-major)
    const int npairs = T * K;
    const int pe = (lane < npairs) ? hd.topi[lane / K][lane % K] : -1 - lane;
    bool first = lane < npairs;
    for (int j = 0; j < 32; ++j) {
      const int ej = __shfl_sync(0xffffffffu, pe, j);
      if (j < lane && ej == pe) first = false;
    }
    const unsigned fm = __ballot_sync(0xffffffffu, first);
    const int myu = first ? __popc(fm & ((1u << lane) - 1u)) : -1;
    if (first) hd.uniq_e[myu] = pe;
    // token lists (pair indices t*K+slot, ascending) of each unique expert
    int cnt = 0;
    for (int j = 0; j < npairs; ++j) {
      const int ej = __shfl_sync(0xffffffffu, pe, j);
      if (first && ej == pe) hd.uniq_pair[myu][cnt++] = j;
    }
    if (first) hd.uniq_cnt[myu] = cnt;
    if (lane == 0) hd.nuniq = __popc(fm);
    if (cta == 0 && lane < npairs) {
      const int t = lane / K, s = lane % K;
      p.topk_idx_ws[lane] = hd.topi[t][s];
      p.topk_w_ws[lane] = hd.topw[t][s];
      if (p.topk_idx_out) p.topk_idx_out[lane] = hd.topi[t][s];
      if (p.topk_w_out) p.topk_w_out[lane] = hd.topw[t][s];
    }
  }
  __syncthreads();
  const int U = hd.nuniq;

  // prefetch this CTA's routed down units (contiguous per expert) into L2
  if (warp == kDecodeWarps - 1 && nblk > 0) {
    for (int u = lane; u < U; u += 32) {
      const uint8_t* src = p.dn + ((size_t)hd.uniq_e[u] * kDnUnits + b0) * kDnUnitBytes;
      prefetch_l2_bulk(src, (uint32_t)nblk * kDnUnitBytes);
    }
  }

  {
    const int n3 = U * kGuUnits;
    const int u0 = (int)((long long)cta * n3 / ncta), u1 = (int)((long long)(cta + 1) * n3 / ncta);
    const int r = lane & 7, q = lane >> 3;
    for (int unit = u0 + warp; unit < u1; unit += kDecodeWarps) {
      const int u = unit / kGuUnits, b = unit - u * kGuUnits;
      const uint8_t* base = p.gu + ((size_t)hd.uniq_e[u] * kGuUnits + b) * kGuUnitBytes;
      uint4 wq[kGuChunks];
      uint2 sc[kGuChunks / 4];
#pragma unroll
      for (int j = 0; j < kGuChunks; ++j) wq[j] = ldg_stream(base + j * 512 + 16 * lane);
#pragma unroll
      for (int j = 0; j < kGuChunks / 4; ++j) sc[j] = ldg_stream64(base + kGuScaleOff + j * 256 + 8 * lane);
      const int cnt = hd.uniq_cnt[u];
      // per-token bases: chunk 4G+i of quarter q sits at 324q + 16j + 4i
      const float* xb[kMaxDecodeT];
      const float* cb[kMaxDecodeT];
      float acc[kMaxDecodeT];
#pragma unroll
      for (int tt = 0; tt < kMaxDecodeT; ++tt) {
        const int t = (tt < cnt) ? hd.uniq_pair[u][tt] / K : 0;
        xb[tt] = xs + (size_t)t * kXTok + 324 * q;
        cb[tt] = cx + t * kXGroups + q * kGuChunks;
        acc[tt] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < kGuChunks; ++j) {
        float part[kMaxDecodeT];
#pragma unroll
        for (int tt = 0; tt < kMaxDecodeT; ++tt) part[tt] = (tt < cnt) ? cb[tt][j] : 0.f;
        const uint32_t wj[4] = {wq[j].x, wq[j].y, wq[j].z, wq[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float f[8];
          dequant8(wj[i], f);
#pragma unroll
          for (int tt = 0; tt < kMaxDecodeT; ++tt) {
            if (tt < cnt) {
              const float* xq = xb[tt] + 16 * j + 4 * i;
              part[tt] = dot8_f(f, *reinterpret_cast<const float4*>(xq),
                                *reinterpret_cast<const float4*>(xq + kXPlane), part[tt]);
            }
          }
        }
        const float s = scale_of(sc[j >> 2], j & 3);
#pragma unroll
        for (int tt = 0; tt < kMaxDecodeT; ++tt) acc[tt] = fmaf(s, part[tt], acc[tt]);
      }
#pragma unroll
      for (int tt = 0; tt < kMaxDecodeT; ++tt) {
        if (tt < cnt) {
          float v = acc[tt];
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          const float up = __shfl_sync(0xffffffffu, v, (lane & ~7) | ((r + 4) & 7));
          if (r < 4 && q == tt) {
            const int pr = hd.uniq_pair[u][tt];
            p.h_pair[(size_t)pr * kI + 4 * b + r] = silu_mul(kCodeScale * v, kCodeScale * up);
          }
        }
      }
    }
  }
  grid_arrive(p.bar + 2, skip);

  // ---- phase 4: down projections and the output
  if (!grid_wait(p.bar + 1, (genB + 1) * ncta, p.wait_limit_ns, p.err, &hd.flag)) return;
  if (!grid_wait(p.bar + 2, (genC + 1) * ncta, p.wait_limit_ns, p.err, &hd.flag)) return;

  const int npairs = T * K;
  float* hp = body;                                           // [pairs][kHpStride]
  float* chp = hp + (size_t)kMaxPairs * kHpStride;            // [pairs][kHGroups]
  float* hs = chp + (size_t)kMaxPairs * kHGroups;             // [T][kHsTok]
  float* part = hs + (size_t)kMaxDecodeT * kHsTok;            // [blk][pairs + T][4]
  for (int v = tid; v < npairs * (kI / 4); v += kDecodeThreads) {
    const int pr = v / (kI / 4), c4 = v - pr * (kI / 4);
    const float4 h = ldcg_f4(reinterpret_cast<const float4*>(p.h_pair + (size_t)pr * kI) + c4);
    const int e0 = 4 * c4;
    *reinterpret_cast<float4*>(hp + (size_t)pr * kHpStride + e0 + 4 * (e0 / 96)) = h;
  }
  for (int v = tid; v < T * (kI / 4); v += kDecodeThreads) {
    const int t = v / (kI / 4), c4 = v - t * (kI / 4);
    const float4 h = ldcg_f4(reinterpret_cast<const float4*>(p.h_s + (size_t)t * kI) + c4);
    const int c = c4 >> 1, pl = c4 & 1;
    *reinterpret_cast<float4*>(hs + (size_t)t * kHsTok + pl * kHsPlane + 4 * c) = h;
  }
  __syncthreads();
  for (int v = tid; v < npairs * kHGroups; v += kDecodeThreads) {
    const int pr = v / kHGroups, G = v - pr * kHGroups;
    const float* src = hp + (size_t)pr * kHpStride + 32 * G + 4 * (G / 3);
    float s = 0.f;
    for (int i = 0; i < 32; ++i) s += src[i];
    chp[pr * kHGroups + G] = kBiasCoef * s;
  }
  __syncthreads();

  // routed items (blk, u): 4 output rows x one unique expert, for its tokens
  {
    const int r = lane & 3, q = lane >> 2;
    const int nitems = nblk * U;
    for (int it0 = warp; it0 < nitems; it0 += 4 * kDecodeWarps) {
      uint4 wq[4][kDnChunks];
      unsigned short sc[4][kDnChunks];
#pragma unroll
      for (int bI = 0; bI < 4; ++bI) {
        const int it = it0 + bI * kDecodeWarps;
        if (it < nitems) {
          const int blk = it / U, u = it - blk * U;
          const uint8_t* base = p.dn + ((size_t)hd.uniq_e[u] * kDnUnits + b0 + blk) * kDnUnitBytes;
#pragma unroll
          for (int j = 0; j < kDnChunks; ++j) {
            wq[bI][j] = ldg_stream(base + j * 512 + 16 * lane);
            sc[bI][j] = ldg_stream16(base + kDnScaleOff + j * 64 + 2 * lane);
          }
        }
      }
#pragma unroll
      for (int bI = 0; bI < 4; ++bI) {
        const int it = it0 + bI * kDecodeWarps;
        if (it < nitems) {
          const int blk = it / U, u = it - blk * U;
          const int cnt = hd.uniq_cnt[u];
          float acc[kMaxDecodeT];
#pragma unroll
          for (int tt = 0; tt < kMaxDecodeT; ++tt) acc[tt] = 0.f;
          const float* hb[kMaxDecodeT];
          const float* cb[kMaxDecodeT];
#pragma unroll
          for (int tt = 0; tt < kMaxDecodeT; ++tt) {
            const int pr = (tt < cnt) ? hd.uniq_pair[u][tt] : 0;
            hb[tt] = hp + (size_t)pr * kHpStride + 100 * q;
            cb[tt] = chp + pr * kHGroups + q * kDnChunks;
          }
#pragma unroll
          for (int j = 0; j < kDnChunks; ++j) {
            float part[kMaxDecodeT];
#pragma unroll
            for (int tt = 0; tt < kMaxDecodeT; ++tt) part[tt] = (tt < cnt) ? cb[tt][j] : 0.f;
            const uint32_t wj[4] = {wq[bI][j].x, wq[bI][j].y, wq[bI][j].z, wq[bI][j].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float f[8];
              dequant8(wj[i], f);
#pragma unroll
              for (int tt = 0; tt < kMaxDecodeT; ++tt) {
                if (tt < cnt) {
                  const float* hq = hb[tt] + 32 * j + 8 * i;
                  part[tt] = dot8_f(f, *reinterpret_cast<const float4*>(hq),
                                    *reinterpret_cast<const float4*>(hq + 4), part[tt]);
                }
              }
            }
            const float sj = bf16_to_f32(sc[bI][j]);
#pragma unroll
            for (int tt = 0; tt < kMaxDecodeT; ++tt) acc[tt] = fmaf(sj, part[tt], acc[tt]);
          }
#pragma unroll
          for (int tt = 0; tt < kMaxDecodeT; ++tt) {
            if (tt < cnt) {
              float v = acc[tt];
              v += __shfl_xor_sync(0xffffffffu, v, 4);
              v += __shfl_xor_sync(0xffffffffu, v, 8);
              v += __shfl_xor_sync(0xffffffffu, v, 16);
              if (q == 0) {
                const int pr = hd.uniq_pair[u][tt];
                const float wgt = hd.topw[pr / K][pr % K];
                part[((size_t)blk * (kMaxPairs + kMaxDecodeT) + pr) * 4 + r] = kCodeScale * v * wgt;
              }
            }
          }
        }
      }
    }
  }
  // shared items: one 4-row block of the shared down projection, all tokens
  {
    const int r = lane & 3, q = lane >> 2;
    for (int blk = kDecodeWarps - 1 - warp; blk < nblk; blk += kDecodeWarps) {
      const int n = 4 * (b0 + blk) + r;
      const __nv_bfloat16* wd = p.sh_down + (size_t)n * kI;
      uint4 w[kI / 64];
#pragma unroll
      for (int m = 0; m < kI / 64; ++m) w[m] = ldg_stream(wd + 8 * (q + 8 * m));
      float acc[kMaxDecodeT];
#pragma unroll
      for (int t = 0; t < kMaxDecodeT; ++t) acc[t] = 0.f;
#pragma unroll
      for (int m = 0; m < kI / 64; ++m) {
        const int c = q + 8 * m;
#pragma unroll
        for (int t = 0; t < kMaxDecodeT; ++t) {
          if (t < T) {
            const float* ht = hs + (size_t)t * kHsTok + 4 * c;
            acc[t] = dot8_bf16(w[m], *reinterpret_cast<const float4*>(ht),
                               *reinterpret_cast<const float4*>(ht + kHsPlane), acc[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kMaxDecodeT; ++t) {
        if (t < T) {
          float v = acc[t];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          if (q == 0) part[((size_t)blk * (kMaxPairs + kMaxDecodeT) + kMaxPairs + t) * 4 + r] = v;
        }
      }
    }
  }
  __syncthreads();
  // fixed-order sum: routed slots 0..k-1, then the shared expert
  for (int v = tid; v < nblk * T * 4; v += kDecodeThreads) {
    const int blk = v / (T * 4), rem = v - blk * T * 4, t = rem >> 2, r = rem & 3;
    const float* pb = part + (size_t)blk * (kMaxPairs + kMaxDecodeT) * 4;
    float s = 0.f;
    for (int sl = 0; sl < K; ++sl) s += pb[(t * K + sl) * 4 + r];
    s += pb[(kMaxPairs + t) * 4 + r];
    p.out[(size_t)t * kH + 4 * (b0 + blk) + r] = __float2bfloat16_rn(s);
  }
}

cudaError_t launch_decode(const DecodeParams& p, int nctas, cudaStream_t stream) {
  static_assert(kDecodeSmemBytes <= 227 * 1024, "decode smem over budget");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = kDecodeSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe_decode_kernel, p);
}

cudaError_t setup_decode() {
  return cudaFuncSetAttribute(moe_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kDecodeSmemBytes);
}

int decode_max_ctas_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, moe_decode_kernel, kDecodeThreads,
                                                    kDecodeSmemBytes) != cudaSuccess)
    return 0;
  return n;
}

}  // namespace lingmoe
