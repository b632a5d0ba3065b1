// Layout of the tensor-core path's per-segment state (d = dv = 64).
//
// The state is indexed by the packed symmetric feature rows (i, j), i <= j:
// phi(q) . S = sum_{i<=j} c_ij q_i q_j S_(i,j) with c_ij = 2 for i < j and 1
// for i = j, so 64 * 65 / 2 = 2080 rows carry the whole state.  They are laid
// out in 17 tiles of 128 rows (2176 rows; the 96 extra rows have i > j, are
// weighted by zero in the readout and never exported).  The order serves both
// tensor-core kernels:
//
//   tiles 0-11   off-diagonal blocks (i / 16 < j / 16) in 16-row groups of one
//                i and 16 consecutive j (a "half-strip").  Tile 4 c + m, lane
//                16 s + jj: global slot gs = 8 c + s selects the j block bj
//                (gs 0-3: bj = 1, 4-11: bj = 2, 12-23: bj = 3), i = 4 (gs -
//                first slot of bj) + m, j = 16 bj + jj.
//   tiles 12-16  the four diagonal 16 x 16 triangles, as column groups: group
//                (b, q, j) holds the rows (16 b + 4 q + m, j), m = 0..3, for
//                j = 16 b + 4 q .. 16 b + 15 (rows with i > j are the padding).
//                The groups run in the order of the runs (b, q) = (r % 4,
//                r / 4), r = 0..15, columns ascending; the first 128 groups
//                fill tiles 12-15 (lane = group, tile 12 + m = row m), the
//                last 32 fill tile 16 (lane 4 g + m).
//
// State builder: a work item is 4 tiles (tiles 4 c .. 4 c + 3, c = 0..3) or
// the single tile 16 (c = 4); a builder thread owns the same lane in each of
// its item's tiles, and within items 0-3 that lane's j is the same in all 4
// tiles, so the thread reads its key column k_j once per token block.
// Readout: two consecutive rows (one 32-bit word of the bf16 A operand) are
// always (i, j), (i, j + 1) with j even or (i, j), (i + 1, j) with i even, so
// every word of phi(q) is one bf16x2 product of register pairs.
//
// Per (head, segment) the fp32 state is the 2176 rows x 64 values, then the
// packed normaliser z[r] = sum k_i k_j of the same rows; the bf16 prefix copy
// read by the readout is the 2176 rows, then the dense Z = sum k k^T split
// into hi and lo bf16 parts (64 rows each).
#pragma once

#if defined(__CUDACC__)
#define KATA_HD __host__ __device__
#else
#define KATA_HD
#endif

namespace kata {
namespace tc {

constexpr int kD = 64;
constexpr int kStateTiles = 17;
constexpr int kStateRows = 128 * kStateTiles;       // 2176
constexpr int kPairRows = kD * (kD + 1) / 2;        // 2080 rows with i <= j
constexpr long long kZPacked0 = (long long)kStateRows * kD;     // fp32 packed z offset
constexpr long long kF32PerSeg = kZPacked0 + kStateRows;        // 141,440 floats
constexpr int kBf16Rows = kStateRows + 2 * kD;      // 2304 rows of 64 bf16
constexpr int kZHiRow0 = kStateRows;                // bf16 Z hi rows
constexpr int kZLoRow0 = kStateRows + kD;           // bf16 Z lo rows
constexpr int kBuildItems = 5;                      // builder items per (head, segment)

// Tiles of builder item c, and the state tile holding its tile m.
KATA_HD constexpr int build_item_tiles(int c) { return c < 4 ? 4 : 1; }
KATA_HD constexpr int build_item_tile(int c, int m) { return c < 4 ? 4 * c + m : 16; }

struct PairIJ {
    int i, j;
};

KATA_HD constexpr int od_class(int gs) { return gs < 4 ? 1 : gs < 12 ? 2 : 3; }
KATA_HD constexpr int od_first_slot(int bj) { return bj == 1 ? 0 : bj == 2 ? 4 : 12; }
KATA_HD constexpr int run_groups(int run) { return 16 - 4 * (run >> 2); }

// (i, j) of state row r (0 <= r < kStateRows); i > j marks a padding row.
KATA_HD constexpr PairIJ row_ij(int r) {
    const int tile = r / 128, lane = r % 128;
    if (tile < 12) {
        const int c = tile / 4, m = tile % 4, s = lane / 16, jj = lane % 16;
        const int gs = 8 * c + s, bj = od_class(gs);
        return PairIJ{4 * (gs - od_first_slot(bj)) + m, 16 * bj + jj};
    }
    const bool first = tile < 16;
    int g = first ? lane : lane / 4;
    const int m = first ? tile - 12 : lane % 4;
    int run = first ? 0 : 10;
    while (g >= run_groups(run)) {
        g -= run_groups(run);
        ++run;
    }
    const int b = run & 3, q = run >> 2;
    return PairIJ{16 * b + 4 * q + m, 16 * b + 4 * q + g};
}

// State row of the pair (i, j), i <= j.
KATA_HD constexpr int row_index(int i, int j) {
    if (i / 16 < j / 16) {
        const int bj = j / 16, jj = j % 16, gs = od_first_slot(bj) + i / 4, m = i % 4;
        return 128 * (4 * (gs / 8) + m) + 16 * (gs % 8) + jj;
    }
    const int b = i / 16, q = (i % 16) / 4, m = i % 4;
    const int run = 4 * q + b;
    const bool first = run < 10;
    int off = 0;
    for (int r = first ? 0 : 10; r < run; ++r) off += run_groups(r);
    const int g = off + (j - (16 * b + 4 * q));
    return first ? 128 * (12 + m) + g : 128 * 16 + 4 * g + m;
}

// ---------------------------------------------------------------------------
// KATA-Mg with g = 2 factors (coordinates 0-31 and 32-63, each its own
// rank-one PSD factor): the state holds only the pairs (i, j), i <= j, inside
// one factor, 2 x 32 * 33 / 2 = 1056 rows, in 9 tiles (1152 rows):
//   tiles 0-3   the off-diagonal 16 x 16 blocks of the two factors, (0-15,
//               16-31) and (32-47, 48-63), as half-strips: tile m, lane
//               16 s + jj holds i = 4 s + m, j = 16 + jj for s < 4 and
//               i = 32 + 4 (s - 4) + m, j = 48 + jj for s >= 4;
//   tiles 4-8   the four diagonal 16 x 16 triangles, laid out as tiles 12-16
//               of the single-factor layout.
// The same properties hold: builder item 0 (tiles 0-3) and item 1 (tiles
// 4-7) keep one j per lane across their 4 tiles, item 2 is tile 8, and every
// 32-bit word of phi(q) is one bf16x2 product.
// ---------------------------------------------------------------------------
KATA_HD constexpr int state_tiles(int G) { return G == 1 ? kStateTiles : 9; }
KATA_HD constexpr int state_rows(int G) { return 128 * state_tiles(G); }
KATA_HD constexpr long long z_packed0(int G) { return (long long)state_rows(G) * kD; }
KATA_HD constexpr long long f32_per_seg(int G) { return z_packed0(G) + state_rows(G); }
KATA_HD constexpr int bf16_rows(int G) { return state_rows(G) + 2 * kD; }
KATA_HD constexpr int zhi_row0(int G) { return state_rows(G); }
KATA_HD constexpr int zlo_row0(int G) { return state_rows(G) + kD; }
KATA_HD constexpr int build_items(int G) { return G == 1 ? kBuildItems : 3; }
KATA_HD constexpr int build_item_tiles(int G, int c) { return c < build_items(G) - 1 ? 4 : 1; }
KATA_HD constexpr int build_item_tile(int G, int c, int m) {
    return c < build_items(G) - 1 ? 4 * c + m : state_tiles(G) - 1;
}
// Tiles of the g = 2 layout taken over from the single-factor layout.
constexpr int kM2TileShift = 8;

// (i, j) of state row r of the layout with G factors.
KATA_HD constexpr PairIJ row_ij_g(int G, int r) {
    if (G == 1) return row_ij(r);
    const int tile = r / 128, lane = r % 128;
    if (tile < 4) {
        const int s = lane / 16, jj = lane % 16;
        return s < 4 ? PairIJ{4 * s + tile, 16 + jj} : PairIJ{32 + 4 * (s - 4) + tile, 48 + jj};
    }
    return row_ij(r + 128 * kM2TileShift);
}

// Both coordinates in the same factor of G (a pair the layout holds).
KATA_HD constexpr bool same_factor(int G, int i, int j) { return i / (kD / G) == j / (kD / G); }

// State row of the pair (i, j), i <= j, same_factor(G, i, j), in the layout with G factors.
KATA_HD constexpr int row_index_g(int G, int i, int j) {
    if (G == 1) return row_index(i, j);
    if (i / 16 < j / 16) {
        const int f = i / 32, ii = i - 32 * f;
        return 128 * (ii % 4) + 16 * (ii / 4 + 4 * f) + j % 16;
    }
    return row_index(i, j) - 128 * kM2TileShift;
}

}  // namespace tc
}  // namespace kata
