// Layout of the tensor-core path's per-segment state (d = dv = 64).
//
// The packed feature rows are grouped in 16-row "half-strips": half-strip h
// holds the rows (i, j) for one i and j = jb .. jb + 15 (jb a multiple of 16).
// Only half-strips that contain some j >= i are kept: for jb = 16 b, i runs
// over 0 .. 16 b + 15, giving 16 + 32 + 48 + 64 = 160 half-strips = 2560 rows
// (the 2080 rows of the exact half triangle plus the 480 mirrored entries of
// the 16 diagonal blocks, which the readout weights by zero).
//
// The order of the half-strips follows the state builder's work split: 5
// CTAs per (head, segment), each with 4 accumulator tiles of 128 rows; tile
// lanes come in 8 slots of 16 lanes, and a slot keeps the same jb in all 4
// tiles of its CTA, so each builder thread reads its own key column once per
// token block.  With global slot gs = 8 c + s (CTA c, slot s) the slots of
// class b (jb = 16 b) are gs = 4 b (b + 1) / 2 .. ; slot u of class b covers
// i = 4 u + m in tile m.  Half-strip index: h = 32 c + 8 m + s, state row
// r = 16 h + (j - jb).
//
// Per (head, segment) the fp32 state is 2560 rows x 64 (the half-strips) then
// the packed normaliser z[r] = sum k_i k_j for the same 2560 rows; the bf16
// prefix copy read by the readout is the 2560 rows, then the dense
// Z = sum k k^T split into hi and lo bf16 parts (64 rows each).
#pragma once

namespace kata {
namespace tc {

constexpr int kD = 64;
constexpr int kHalfStrips = 160;
constexpr int kStateRows = 16 * kHalfStrips;        // 2560
constexpr long long kZPacked0 = (long long)kStateRows * kD;     // fp32 packed z offset
constexpr long long kF32PerSeg = kZPacked0 + kStateRows;        // 166,400 floats
constexpr int kBf16Rows = kStateRows + 2 * kD;      // 2688 rows of 64 bf16
constexpr int kZHiRow0 = kStateRows;                // bf16 Z hi rows
constexpr int kZLoRow0 = kStateRows + kD;           // bf16 Z lo rows

__host__ __device__ constexpr int hs_class(int gs) { return gs < 4 ? 0 : gs < 12 ? 1 : gs < 24 ? 2 : 3; }
__host__ __device__ constexpr int hs_class_start(int b) { return b == 0 ? 0 : b == 1 ? 4 : b == 2 ? 12 : 24; }

// i and jb of half-strip h.
__host__ __device__ constexpr int hs_i(int h) {
    return 4 * ((8 * (h / 32) + h % 8) - hs_class_start(hs_class(8 * (h / 32) + h % 8))) +
           (h / 8) % 4;
}
__host__ __device__ constexpr int hs_jb(int h) { return 16 * hs_class(8 * (h / 32) + h % 8); }

// Half-strip holding row (i, j) for i <= j (requires i <= 16 (j / 16) + 15).
__host__ __device__ constexpr int hs_index(int i, int j) {
    return 32 * ((hs_class_start(j / 16) + i / 4) / 8) + 8 * (i % 4) +
           (hs_class_start(j / 16) + i / 4) % 8;
}

}  // namespace tc
}  // namespace kata
