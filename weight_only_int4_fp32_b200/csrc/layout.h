// Layer shape and the repacked weight layouts (host and device).
#pragma once

#include <cstddef>

namespace lingmoe {

// ---------------------------------------------------------------- shape
// The layer shape the kernels are specialised for (Ling-3.0-flash MoE:
// hidden 2560, moe_intermediate_size 768, int4 groups of 32 along K).
constexpr int kH = 2560;
constexpr int kI = 768;
constexpr int kGroup = 32;
constexpr int kMaxTopK = 8;
constexpr int kMaxExperts = 512;

// ---------------------------------------------------------------- repacked layouts
// Routed gate/up, per expert: kGuUnits units, one per block of 8 intermediate
// rows i = 8b..8b+7, each unit holding the 16 rows (gate i, up i) x K.  K is
// cut into blocks of 16; a block is 32 words, and word t (lane t of a warp)
// holds exactly the int4 codes of lane t's A fragment of an m16n8k16 MMA
// whose rows are (gate i_t, up i_t), i_t = 8b + t/4, and whose columns are
// c, c+1, c+8, c+9 with c = 16 kb + 2 (t % 4):
//   nibble 0: gate c    nibble 4: gate c+1    nibble 1: gate c+8   nibble 5: gate c+9
//   nibble 2: up c      nibble 6: up c+1      nibble 3: up c+8     nibble 7: up c+9
// as offset-binary codes (q + 8).  A chunk of 512 B covers 64 K (4 blocks):
// lane t's 16 bytes are its words for blocks 4j .. 4j+3.  The bf16 scales
// follow the kGuChunks chunks as [group][i (8)][gate, up].  The first and
// second halves of K (chunks 0..19 with groups 0..39, and the rest) are
// what the decode path streams as one work item each.
constexpr int kGuUnits = kI / 8;                  // 96
constexpr int kGuChunks = kH / 64;                // 40 chunks of 64 K
constexpr int kGuScaleOff = kGuChunks * 512;      // 20480
constexpr int kGuUnitBytes = kGuScaleOff + (kH / kGroup) * 32;  // 23040
constexpr size_t kGuExpertBytes = (size_t)kGuUnits * kGuUnitBytes;  // 2211840
constexpr int kGuHalfCodes = kGuScaleOff / 2;     // 10240: codes of one K half
constexpr int kGuHalfScales = (kH / kGroup) * 16; // 1280: scales of one K half
constexpr int kGuHalfBytes = kGuHalfCodes + kGuHalfScales;  // 11520

// Routed down, per expert: kDnUnits units, one per block of 8 output rows
// n = 8v..8v+7 (all 768 K).  K is cut into groups of 32; a group is 32
// words, and word t holds exactly the int4 codes of lane t's B fragments of
// the two m16n8k16 MMAs (K blocks 32G and 32G + 16) whose columns are the
// unit's 8 rows: row n_t = 8v + t/4, K = 32G + c, c + 1, c + 8, c + 9 and the
// same + 16, with c = 2 (t % 4):
//   nibble 0: c       nibble 4: c+1       nibble 1: c+8      nibble 5: c+9
//   nibble 2: c+16    nibble 6: c+17      nibble 3: c+24     nibble 7: c+25
// as offset-binary codes (q + 8), the nibble order of the gate/up words.  A
// chunk of 512 B covers 128 K (4 groups): lane t's 16 bytes are its words for
// groups 4j .. 4j+3.  The scales follow the kDnChunks chunks as 64-byte
// blocks [c/2 (4)][group within the chunk (4)] of 32-bit words, each the bf16
// pair (row 8v + c, row 8v + c + 1) of one group: the two output rows whose
// results lane t's accumulator fragment holds.
constexpr int kDnUnitRows = 8;
constexpr int kDnUnits = kH / kDnUnitRows;        // 320
constexpr int kDnChunks = kI / 128;               // 6 chunks of 128 K
constexpr int kDnScaleOff = kDnChunks * 512;      // 3072
constexpr int kDnUnitBytes = kDnScaleOff + kDnChunks * 64;  // 3456
constexpr size_t kDnExpertBytes = (size_t)kDnUnits * kDnUnitBytes;  // 1105920

// Routed-weight codecs.  kCodecInt4: symmetric int4 codes, stored
// offset-binary (q + 8), one bf16 scale per 32 K.  kCodecMxfp4: MXFP4 (OCP
// Microscaling) -- E2M1 codes (bit 3 sign, bits 2..1 exponent with bias 1,
// bit 0 mantissa) stored as they are, in the same nibble positions, with the
// per-32 E8M0 scale 2^(e - 127) stored as the bf16 2^(e - 127 + 14) (the
// kernels decode E2M1 as value * 2^-14).  Same unit layouts for both.
constexpr int kCodecInt4 = 0;
constexpr int kCodecMxfp4 = 1;

static_assert(kGuChunks % 2 == 0, "gate/up units split into two K halves");
static_assert(kH % 256 == 0 && kI % 256 == 0, "shape must tile by 256");

}  // namespace lingmoe
