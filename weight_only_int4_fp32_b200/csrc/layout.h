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
// Routed gate/up, per expert: kGuUnits units, one per block of 4 intermediate
// rows i = 4b..4b+3.  A unit holds 8 rows (gate i0..i3, up i0..i3) split into
// 4 K-quarters; lane l of a warp owns row (l & 7) and quarter (l >> 3).
// Chunk j (0..kGuChunks-1) is 32 lanes x 16 B; lane l's 16 B are the 32 int4
// codes of group G = quarter * kGuChunks + j of its row, as offset-binary
// nibbles (code + 8), low nibble = even K index.  The 4*kGuChunks bf16 scales
// of each lane follow, as kGuChunks/4 blocks of [32 lanes x 4 scales].
constexpr int kGuUnits = kI / 4;                  // 192
constexpr int kGuChunks = kH / 128;               // 20 groups per lane
constexpr int kGuScaleOff = kGuChunks * 512;      // 10240
constexpr int kGuUnitBytes = kGuScaleOff + kGuChunks * 64;  // 11520
constexpr size_t kGuExpertBytes = (size_t)kGuUnits * kGuUnitBytes;  // 2211840

// Routed down, per expert: kDnUnits units, one per block of 4 output rows
// n = 4v..4v+3; lane l owns row (l & 3) and K-slice (l >> 2) of 3 groups.
// Chunk j (0..2) is 32 lanes x 16 B (group 3*slice + j of the lane's row),
// then 3 blocks of [32 lanes x bf16 scale].
constexpr int kDnUnits = kH / 4;                  // 640
constexpr int kDnChunks = kI / 256;               // 3 groups per lane
constexpr int kDnScaleOff = kDnChunks * 512;      // 1536
constexpr int kDnUnitBytes = kDnScaleOff + kDnChunks * 64;  // 1728
constexpr size_t kDnExpertBytes = (size_t)kDnUnits * kDnUnitBytes;  // 1105920

static_assert(kGuChunks % 4 == 0, "gate/up scales are loaded 4 at a time");
static_assert(kH % 256 == 0 && kI % 256 == 0, "shape must tile by 256");

}  // namespace lingmoe
