// KATA causal forward, tensor-core path (bf16 q, k, v, d = dv = 64, sm_100a;
// heads of d = 16 and 32 read as 64, on the two-factor layout).
//
// Exact chunked-state form (gist.science summary of "Kernelized Linear
// Attention: Breaking the Capacity Wall with Symmetric Cones", Technical
// summary 2.3: tensor cores inside a chunk, associative scan of chunk states
// across chunks; arXiv abstract: "exact O(T) chunked-state form").  States are
// stored every L tokens (a segment); inside a segment the causal quadratic
// form is used, which equals the chunk-by-chunk propagation exactly.
//
//   tc_build         per segment on tcgen05: dS = sum phi(k) v^T on the
//                    half-strip rows (tc_layout.cuh) and dZ = sum k k^T, fp32
//                    (the key tiles are transposed in shared memory on the way)
//   tc_seg_scan      exclusive prefix over segments (associative scan) into a
//                    bf16 copy for the readout, and the total: written as the
//                    dense exported state (one factor, and heads of d <= 32)
//                    or kept packed in fp32 (two factors of d = 64)
//   tc_read          per 256 queries: phi(Q) S_prev and q^T Z_prev q on tcgen05
//                    (phi(Q) generated from registers into tensor memory), the
//                    intra-segment squared-score term on tcgen05, the division
//   tc_state_expand  two factors of d = 64: fp32 packed total -> dense [d*d, d]
//                    state and [d, d] Z, zeros at the pairs across factors
#include <cuda_bf16.h>

#include <mutex>

#include "kata_internal.cuh"
#include "sm100.cuh"
#include "tc_layout.cuh"
#include "tmap.cuh"

namespace kata {
namespace tc {
namespace {

using namespace kata::sm100;

// bf16 prefix elements per (head, segment): the state rows, then Z hi and lo
KATA_HD constexpr long long bf16_per_seg(int G) { return (long long)bf16_rows(G) * kD; }

// ---------------------------------------------------------------------------
// Exclusive prefix over segments (the associative scan across chunk states)
// -> bf16 copy for the readout (Z split into hi and lo parts), and the total:
// the fp32 packed total (total != nullptr) and/or the dense exported state
// (state_out != nullptr: S [d*d][d] and Z [d][d] of head size d <= 64,
// written straight from the scan's registers; one factor only).  An initial
// state (the sum of n_in dense states of head size d) seeds the running sum,
// so every prefix and the total include it and segment 0 gets a prefix too;
// prefix == nullptr computes the total only.
// Reduce-then-scan per block of 128 consecutive elements of one head
// (32 lanes x float4): warp w takes a run of RUN consecutive segments,
// holds them in registers and forms their running sums; the 8 run totals are
// scanned across warps in shared memory in log2(8) = 3 steps; each warp adds
// its offset and writes its run.  Every global access is a coalesced 16-byte
// (fp32) or 8-byte (bf16) vector per lane.  RUN is the smallest of 2, 4, 8,
// 16 whose pass covers every segment (at most 16): with few segments a short
// run keeps the registers, and so the blocks resident per SM, that the
// latency of these short blocks needs.  G factors (KATA-Mg): the layout with
// G factors; the dense Z prefix then also gets zeros at the pairs across
// factors, which the readout's q^T Z q must not see.
// grid.x = n_eb * BH (the packed-z blocks of all heads first); block 256.
// ---------------------------------------------------------------------------
constexpr int kScanWarps = 8;

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// One thread's 4 consecutive elements of a (head, segment) state: where they
// sit (state rows or packed normaliser rows, and the pairs of the latter).
template <int G>
struct ScanLane {
    long long e0;
    bool z_part;
    int zr;
    int zi[4], zj[4];
    __device__ __forceinline__ ScanLane(long long e) : e0(e) {
        z_part = e0 >= z_packed0(G);
        zr = z_part ? (int)(e0 - z_packed0(G)) : 0;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const PairIJ pij = row_ij_g(G, zr + x);
            zi[x] = pij.i;
            zj[x] = pij.j;
        }
    }

    // The initial state of these 4 packed elements: the sum of n_in dense states
    // of head size d (<= 64: the coordinates past d are zero), added in order
    // n = 0, 1, ...; the loads of U states are in flight at a time.
    template <int U>
    __device__ __forceinline__ float4 init(long long bh, const float *init_s, const float *init_z,
                                           int n_in, long long s_stride, long long z_stride,
                                           int d) const {
        float4 carry = make_float4(0.f, 0.f, 0.f, 0.f);
        if (n_in <= 0) return carry;
        if (!z_part) {
            const PairIJ pij = row_ij_g(G, (int)(e0 / kD));
            const int e = (int)(e0 % kD);  // 4 consecutive values, all below d or none
            if (pij.i > pij.j || pij.j >= d || e >= d) return carry;
            const float *src = init_s + ((bh * d + pij.i) * d + pij.j) * d + e;
            int n = 0;
            for (; n + U <= n_in; n += U) {
                float4 a[U];
#pragma unroll
                for (int u = 0; u < U; ++u) a[u] = *reinterpret_cast<const float4 *>(src + (n + u) * s_stride);
#pragma unroll
                for (int u = 0; u < U; ++u) carry = f4add(carry, a[u]);
            }
            for (; n < n_in; ++n) carry = f4add(carry, *reinterpret_cast<const float4 *>(src + n * s_stride));
            return carry;
        }
        // packed normaliser entries: Z[i][j] of each of the 4 pairs
        int off[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) off[x] = zi[x] <= zj[x] && zj[x] < d ? zi[x] * d + zj[x] : -1;
        const float *zb = init_z + bh * d * d;
        int n = 0;
        for (; n + U <= n_in; n += U) {
            float a[U][4];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int x = 0; x < 4; ++x) a[u][x] = off[x] >= 0 ? zb[(n + u) * z_stride + off[x]] : 0.f;
#pragma unroll
            for (int u = 0; u < U; ++u) carry = f4add(carry, make_float4(a[u][0], a[u][1], a[u][2], a[u][3]));
        }
        for (; n < n_in; ++n) {
            float a[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) a[x] = off[x] >= 0 ? zb[n * z_stride + off[x]] : 0.f;
            carry = f4add(carry, make_float4(a[0], a[1], a[2], a[3]));
        }
        return carry;
    }

    // Writes the total t of these elements into the dense exported state of
    // head bh, head size d (<= 64): S [d*d][d] at state_out and Z [d][d] at
    // z_out, both (i, j) and (j, i).  One factor only: there every dense entry
    // is a pair of the layout, so the scan lanes cover the whole export.
    __device__ __forceinline__ void write_dense(float *state_out, float *z_out, long long bh, float4 t,
                                                int d) const {
        if (!z_part) {
            const PairIJ pij = row_ij_g(G, (int)(e0 / kD));
            const int e = (int)(e0 % kD);
            if (pij.i > pij.j || pij.j >= d || e >= d) return;
            float *s = state_out + bh * d * d * d;
            *reinterpret_cast<float4 *>(s + ((long long)pij.i * d + pij.j) * d + e) = t;
            if (pij.i != pij.j) *reinterpret_cast<float4 *>(s + ((long long)pij.j * d + pij.i) * d + e) = t;
            return;
        }
        const float tv[4] = {t.x, t.y, t.z, t.w};
        float *z = z_out + bh * d * d;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            if (zi[x] > zj[x] || zj[x] >= d) continue;
            z[zi[x] * d + zj[x]] = tv[x];
            z[zj[x] * d + zi[x]] = tv[x];
        }
    }

    // Writes the prefix p of these elements into one segment's bf16 prefix dst.
    __device__ __forceinline__ void write(__nv_bfloat16 *dst, float4 p, int lane) const {
        if (!z_part) {
            uint2 o;
            o.x = pack_bf16x2(p.x, p.y);
            o.y = pack_bf16x2(p.z, p.w);
            *reinterpret_cast<uint2 *>(dst + e0) = o;
            return;
        }
        // dense Z[i][j] and Z[j][i] as hi + lo bf16
        const float pv[4] = {p.x, p.y, p.z, p.w};
        __nv_bfloat16 *zh = dst + (long long)zhi_row0(G) * kD;
        __nv_bfloat16 *zl = dst + (long long)zlo_row0(G) * kD;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            if (zi[x] > zj[x]) continue;
            const __nv_bfloat16 hi = __float2bfloat16_rn(pv[x]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(pv[x] - __bfloat162float(hi));
            zh[zi[x] * kD + zj[x]] = hi;
            zl[zi[x] * kD + zj[x]] = lo;
            zh[zj[x] * kD + zi[x]] = hi;
            zl[zj[x] * kD + zi[x]] = lo;
        }
        if constexpr (G == 2) {
            // zeros at the pairs across the two factors: in each of Z hi and Z lo,
            // rows 0-31 columns 32-63 and rows 32-63 columns 0-31, as 16-byte runs
            // of 8 zeros (512 stores), spread over the lanes of the packed-z blocks
            constexpr int kStores = 2 * 64 * 4, kThr = 32 * (state_rows(G) / 128);
            const int zt = (zr / 128) * 32 + lane;
#pragma unroll
            for (int x = 0; x < (kStores + kThr - 1) / kThr; ++x) {
                const int si = zt + kThr * x;
                if (si >= kStores) break;
                const int row = (si % 256) / 4, col = (row < 32 ? 32 : 0) + 8 * (si % 4);
                __nv_bfloat16 *dz = (si < 256 ? zh : zl) + row * kD + col;
                *reinterpret_cast<uint4 *>(dz) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }
};

// Blocks per SM: RUN = 8 takes 3 at the cost of a few spilled registers
// (28 bytes; its 2 without spills were 14% slower on 64 segments per head).
template <int G, int RUN>
__global__ void __launch_bounds__(256, RUN == 4 ? 4 : RUN == 8 ? 3 : 2)
tc_seg_scan(const float *__restrict__ seg_state, __nv_bfloat16 *__restrict__ prefix,
            float *__restrict__ total, int n_seg, int n_valid, const float *__restrict__ init_s,
            const float *__restrict__ init_z, int n_in, long long s_stride, long long z_stride,
            int d, float *__restrict__ state_out, float *__restrict__ z_out) {
    // launched after the builder, perhaps as its programmatic dependent: the
    // readout may start launching now; the segment states are read after the
    // builder has finished
    griddep_launch_dependents();
    griddep_wait();
    __shared__ float4 part[2][kScanWarps][32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    constexpr long long E = f32_per_seg(G);
    constexpr long long n_eb = E / 128;
    // The packed-z blocks of every head (their dense Z prefix goes out in
    // scattered 2-byte stores) take the first CTAs, so they start in the first
    // wave; the state blocks follow, head-major.
    constexpr long long n_zb = state_rows(G) / 128, n_sb = n_eb - n_zb;
    const long long NZ = n_zb * (gridDim.x / n_eb), x = blockIdx.x;
    const long long bh = x < NZ ? x / n_zb : (x - NZ) / n_sb;
    const long long eb = x < NZ ? n_sb + x % n_zb : (x - NZ) % n_sb;
    const ScanLane<G> sl(eb * 128 + 4 * lane);
    const float *base = seg_state + bh * (long long)n_seg * E + sl.e0;
    __nv_bfloat16 *pbase = prefix ? prefix + bh * (long long)n_seg * bf16_per_seg(G) : nullptr;
    float4 carry = sl.template init<RUN <= 4 ? 2 : 4>(bh, init_s, init_z, n_in, s_stride, z_stride, d);
    const int g_first = n_in > 0 ? 0 : 1;  // without one, segment 0 has an empty prefix

    for (int g0 = 0; g0 < n_seg; g0 += kScanWarps * RUN) {
        const int gw = g0 + w * RUN;
        float4 v[RUN];
#pragma unroll
        for (int i = 0; i < RUN; ++i)
            v[i] = gw + i < n_valid ? *reinterpret_cast<const float4 *>(base + (long long)(gw + i) * E)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < RUN; ++i) {  // exclusive running sum within the run
            const float4 x = v[i];
            v[i] = run;
            run = f4add(run, x);
        }
        // inclusive Kogge-Stone scan of the 8 run totals across warps
        int buf = 0;
        part[0][w][lane] = run;
        __syncthreads();
#pragma unroll
        for (int off = 1; off < kScanWarps; off <<= 1) {
            float4 x = part[buf][w][lane];
            if (w >= off) x = f4add(x, part[buf][w - off][lane]);
            part[buf ^ 1][w][lane] = x;
            buf ^= 1;
            __syncthreads();
        }
        const float4 incl = part[buf][w][lane];
        const float4 all = part[buf][kScanWarps - 1][lane];
        const float4 off = f4add(carry, make_float4(incl.x - run.x, incl.y - run.y, incl.z - run.z,
                                                    incl.w - run.w));
        carry = f4add(carry, all);
        __syncthreads();  // part is rewritten by the next pass
#pragma unroll
        for (int i = 0; i < RUN; ++i) {
            const int g = gw + i;
            if (prefix == nullptr || g < g_first || g >= n_seg) continue;
            sl.write(pbase + (long long)g * bf16_per_seg(G), f4add(v[i], off), lane);
        }
    }
    if (w == 0) {
        if (total != nullptr) *reinterpret_cast<float4 *>(total + bh * E + sl.e0) = carry;
        if (state_out != nullptr) sl.write_dense(state_out, z_out, bh, carry, d);
    }
}

// The same scan for short sequences (at most RUN <= 16 segments): one warp
// per element block holds every segment in registers and scans them
// sequentially, eight element blocks per CTA, with no cross-warp exchange and
// no barrier.  A sequence of a few segments (a short prompt, one rank's block
// of a sequence split over GPUs) otherwise runs thousands of blocks that each
// move a few kilobytes between three barriers.
// grid.x = ceil(n_eb * BH / 8) (at least n_zb * BH); block 256.
template <int G, int RUN>
__global__ void __launch_bounds__(256, RUN > 8 ? 2 : RUN > 4 || G == 2 ? 3 : 4)  // blocks per SM without spills
tc_seg_scan_short(const float *__restrict__ seg_state, __nv_bfloat16 *__restrict__ prefix,
                  float *__restrict__ total, int n_seg, int n_valid, long long BH,
                  const float *__restrict__ init_s, const float *__restrict__ init_z, int n_in,
                  long long s_stride, long long z_stride, int d, float *__restrict__ state_out,
                  float *__restrict__ z_out) {
    griddep_launch_dependents();  // as tc_seg_scan
    griddep_wait();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    constexpr long long E = f32_per_seg(G);
    constexpr long long n_eb = E / 128;
    // The warp's element block.  The packed-z blocks, whose dense Z prefix
    // goes out in scattered 2-byte stores, take warp 0 of the first n_zb * BH
    // CTAs, one per CTA, so that no SM serialises several of them; the state
    // blocks fill the other warps in order (head-major).
    constexpr long long n_zb = state_rows(G) / 128, n_sb = n_eb - n_zb;
    const long long NZ = n_zb * BH, blk = blockIdx.x;
    const long long gidx = blk * kScanWarps + w;  // warp-uniform
    if (gidx >= n_eb * BH) return;
    long long bh, eb;
    if (w == 0 && blk < NZ) {
        bh = blk / n_zb;
        eb = n_sb + blk % n_zb;
    } else {
        const long long zb_before = blk + (w > 0 ? 1 : 0) < NZ ? blk + (w > 0 ? 1 : 0) : NZ;
        const long long s = gidx - zb_before;
        bh = s / n_sb;
        eb = s % n_sb;
    }
    const ScanLane<G> sl(eb * 128 + 4 * lane);
    const float *base = seg_state + bh * (long long)n_seg * E + sl.e0;
    __nv_bfloat16 *pbase = prefix ? prefix + bh * (long long)n_seg * bf16_per_seg(G) : nullptr;
    float4 v[RUN];
#pragma unroll
    for (int i = 0; i < RUN; ++i)
        v[i] = i < n_valid ? *reinterpret_cast<const float4 *>(base + (long long)i * E)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 run = sl.template init<RUN <= 4 ? 1 : RUN <= 8 ? 2 : 4>(bh, init_s, init_z, n_in, s_stride, z_stride, d);
    const int g_first = n_in > 0 ? 0 : 1;
#pragma unroll
    for (int i = 0; i < RUN; ++i) {
        if (prefix != nullptr && i >= g_first && i < n_seg)
            sl.write(pbase + (long long)i * bf16_per_seg(G), run, lane);
        run = f4add(run, v[i]);
    }
    if (total != nullptr) *reinterpret_cast<float4 *>(total + bh * E + sl.e0) = run;
    if (state_out != nullptr) sl.write_dense(state_out, z_out, bh, run, d);
}

// ---------------------------------------------------------------------------
// fp32 total (packed rows) -> dense state [D*D][D] and Z [D][D], for G = 2
// factors (KATA-Mg, D = 64), whose pairs across factors are not in the layout
// and export 0 (one factor, and heads of d <= 32 on the two-factor layout,
// export straight from the scan, every dense entry being a pair of the
// layout).  D < 64 would export the leading D x D part of heads computed as
// 64.  D is a template parameter so the index arithmetic divides by
// constants.
// ---------------------------------------------------------------------------
// A thread writes 4 consecutive outputs (one 16-byte store: the outputs are
// 16-byte aligned, and D, the packed row length and the per-head strides are
// multiples of 4).
template <int G, int D>
__global__ void __launch_bounds__(256)
tc_state_expand(const float *__restrict__ total, long long stride_bh, float *__restrict__ state_out,
                float *__restrict__ z_out, long long BH) {
    constexpr int d3 = D * D * D, per4 = (d3 + D * D) / 4;
    const long long idx = (long long)blockIdx.x * 256 + threadIdx.x;
    if (idx >= (long long)per4 * BH) return;
    const long long bh = idx / per4;
    const int x = 4 * (int)(idx % per4);
    const float *src = total + bh * stride_bh;
    if (x < d3) {
        // values e .. e + 3 of dense row (i, j): the packed row of the pair
        const int row = x / D, e = x % D;
        int i = row / D, j = row % D;
        if (i > j) { const int t = i; i = j; j = t; }
        const float4 v = same_factor(G, i, j)
                             ? *reinterpret_cast<const float4 *>(src + (long long)row_index_g(G, i, j) * kD + e)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(state_out + bh * d3 + x) = v;
    } else {
        // Z[i][j0 .. j0 + 3]
        const int xz = x - d3, i = xz / D, j0 = xz % D;
        float z[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int a = min(i, j0 + u), b = max(i, j0 + u);
            z[u] = same_factor(G, a, b) ? src[z_packed0(G) + row_index_g(G, a, b)] : 0.f;
        }
        *reinterpret_cast<float4 *>(z_out + bh * (D * D) + xz) = make_float4(z[0], z[1], z[2], z[3]);
    }
}

// ---------------------------------------------------------------------------
// Readout kernel (persistent: one CTA per SM walks a contiguous range of work
// items, so consecutive items of a segment reuse its state prefix and keys
// from L2).
//
// Work item = 256 queries (two 128-query tiles) of one segment.  Roles:
//   warps 0-3 / 4-7  phi(Q) generation, then squared-score masking and the
//                    epilogue, for tile 0 / tile 1 (thread = query row)
//   warp 8           TMA producer (Q into a double-buffered item slot; the
//                    Z prefix and the state-prefix stages through the prefix
//                    ring; key and value blocks through rings of their own)
//   warps 9, 10      MMA issuers.  In the inter phase they take alternate
//                    stages (so one issuer's wait overlaps the other's queued
//                    MMAs).  In the intra phase, which runs in steps (key
//                    block, tile) over three score buffers, warp 9 issues
//                    the scores Q K^T and warp 10 the weights times values
//                    P V, so the scores of later steps run while earlier
//                    steps are squared.
//   warp 11          writes the finished output tiles (staged by the
//                    epilogue in the item's Q slot) back with TMA stores.
// Every barrier phase runs on across items.  Accumulators are zeroed by
// tcgen05.st (at the start, then by each epilogue right after it reads them)
// and every MMA accumulates, so the order in which the two issuers' MMAs run
// is free.
// ---------------------------------------------------------------------------
constexpr int kQT = 128;                 // query tile (MMA M)
constexpr int kTiles = 2;                // query tiles per item
constexpr int kCtaQ = kQT * kTiles;      // 256 queries per item
// Keys per intra step (one key/value block, one score buffer): 128 for one
// factor (scores Q K^T with N = 128), 64 for two (both factors' scores side
// by side, N = 64 each).
KATA_HD constexpr int step_keys(int G) { return G == 1 ? 128 : 64; }
constexpr int kKVMax = 6;                // key (or value) ring slots, the most either form uses
constexpr int kSBufs = 3;                // score buffers, shared round-robin by the two tiles
constexpr int kRKs = 8;                  // 16-row K-steps per inter stage (128 state rows)
// inter stages (128 state rows each): 17 for one factor, 9 for two
KATA_HD constexpr int read_stages(int G) { return state_rows(G) / (16 * kRKs); }
constexpr int kRRing = 3;                // inter A ring depth (tensor memory)
constexpr int kRBRing = 4;               // inter B ring depth (state-prefix tiles, shared memory)
constexpr int kRStageBytes = kRKs * 16 * 128;   // bf16 state-prefix rows per stage
constexpr int kTmaWarp = 8;
constexpr int kIssuer0 = 9;
constexpr int kStoreWarp = 11;
constexpr int kReadThreads = 384;

// shared memory (from a 1024-byte aligned base)
constexpr int kItemBytes = kTiles * 16384;  // Q tiles [128 x 64] x 2
constexpr int kSmItem = 0;                       // 2 item slots (double buffer)
// ring of [128 x 64] state-prefix tiles; an item with a prefix takes 1 +
// read_stages(G) entries: its Z hi / lo ([64 x 64] each), then the stages
constexpr int kSmS = kSmItem + 2 * kItemBytes;
KATA_HD constexpr int kv_bytes(int G) { return step_keys(G) * kD * 2; }  // one key or value block
constexpr int kKVRingBytes = 49152;              // keys (or values) of the whole ring
// key (and value) blocks in flight: 3 of 128 keys, or 6 of 64
KATA_HD constexpr int kv_ring(int G) { return kKVRingBytes / kv_bytes(G); }
constexpr int kSmK = kSmS + kRBRing * kRStageBytes;  // ring of [step_keys x 64] key blocks
constexpr int kSmV = kSmK + kKVRingBytes;         // ring of [step_keys x 64] value blocks
constexpr int kSmBytes = kSmV + kKVRingBytes;
constexpr int kSmAlloc = kSmBytes + 1024;

// tensor memory columns (512 allocated)
constexpr uint32_t kTmO = 0;     // O[t]: 64 columns at 64 t
constexpr uint32_t kTmA = 128;   // inter A slot s: 128 columns at 128 + 128 s (tile t at + 64 t)
constexpr uint32_t kTmU = 384;   // U[t] = Q Z (before slot 2 is first written): 64 columns at 384 + 64 t
// Intra score buffer x: 128 columns at 128 + 128 x (the inter phase's columns,
// free once its MMAs are done).  The intra phase runs in steps (key block b,
// tile t), b-major, on a CTA-wide step count n; step n uses buffer n % 3.
// One factor: the 128 scores of the step, then its weights (bf16 pairs, 64
// columns) written over the first half once the squaring warps have read it.
// Two factors: the two factors' 64 scores side by side, the weights (32
// columns) over the first quarter.  The weights times values MMAs read them
// there; the buffer takes new scores once those MMAs are done.
constexpr uint32_t kTmBuf = 128;

struct ReadBars {
    // ostaged[b]: the output rows of the item in slot b are staged.  One per
    // slot: a slot is refilled only after the store warp has released it, so
    // neither barrier can complete twice ahead of the store warp's wait.
    uint64_t qfull[2], qempty[2], u, interdone, done, genin, ostaged[2];
    uint64_t bfull[kRBRing], bempty[kRBRing], afull[kRRing], aempty[kRRing];
    // key and value rings apart; the keys of a block free well before its
    // values.  No commit releases a slot (a commit costs its issuer ~100 cycles
    // and commits arrive ~200 apart): kempty is a plain arrival by the squaring
    // warps that saw the block's last scores land, vempty one by issuer 0 when
    // it has seen the block's last products done (before reusing that buffer).
    uint64_t kfull[kKVMax], kempty[kKVMax], vfull[kKVMax], vempty[kKVMax];
    // per score buffer: sfull, the step's scores formed; pfull, its weights
    // stored over them; bfree, its weights times values done (the buffer may
    // take the scores of step n + 3)
    uint64_t sfull[kSBufs], pfull[kSBufs], bfree[kSBufs];
    uint64_t drain[2];
};

// One work item of the readout.
struct ReadItem {
    int bh, t0, seg0, sidx, n_kv;
    bool inter;
};

// has_init: the forward starts from a given state, so segment 0 has a prefix too.
// n_kv: key/value blocks (step_keys(G) keys) from the segment start to the
// item's last query.
template <int G>
__device__ __forceinline__ ReadItem read_item(int i, int n_ct, int T, int L, int n_seg, bool has_init) {
    ReadItem it;
    it.bh = i / n_ct;
    it.t0 = (i % n_ct) * kCtaQ;
    const int g = it.t0 / L;
    it.seg0 = g * L;
    it.sidx = it.bh * n_seg + g;
    it.inter = g > 0 || has_init;
    const int tend = min(it.t0 + kCtaQ, T);
    it.n_kv = (tend - it.seg0 + step_keys(G) - 1) / step_keys(G);
    return it;
}

// Work items a CTA walks.  Several segments: a contiguous range of the natural
// order (head-major), so the items of a segment reuse its state prefix and keys
// from L2.  One segment (the quadratic form): the costliest items (latest
// queries) first, dealt round-robin to the CTAs, which balances work that grows
// with the query position.
struct ReadSched {
    int first, end, stride, n_ct, BH;
    bool longest_first;
    __device__ __forceinline__ int item(int x) const {  // natural item index of position x
        return longest_first ? (x % BH) * n_ct + (n_ct - 1 - x / BH) : x;
    }
};

__device__ __forceinline__ ReadSched read_sched(int n_items, int n_ct, int n_seg) {
    ReadSched s;
    s.n_ct = n_ct;
    s.BH = n_items / n_ct;
    s.longest_first = n_seg == 1;
    if (s.longest_first) {
        s.first = blockIdx.x;
        s.end = n_items;
        s.stride = gridDim.x;
    } else {
        s.first = (int)((long long)blockIdx.x * n_items / gridDim.x);
        s.end = (int)((long long)(blockIdx.x + 1) * n_items / gridDim.x);
        s.stride = 1;
    }
    return s;
}

// Key blocks of tile t: keys seg0 .. min(end of tile, T) - 1; none when the
// tile starts at or after T.  Tile 0 never has more blocks than tile 1 unless
// tile 1 has none.
template <int G>
__device__ __forceinline__ int read_tile_blocks(const ReadItem &it, int t, int T) {
    const int q0 = it.t0 + kQT * t;
    if (q0 >= T) return 0;
    return (min(q0 + kQT, T) - it.seg0 + step_keys(G) - 1) / step_keys(G);
}

// Steps of an item before its step (key block b, tile t): the steps run
// b-major over the tiles that have a block b.
__device__ __forceinline__ int step_before(int b, int t, int nb0, int nb1) {
    return min(b, nb0) + min(b, nb1) + (t == 1 && b < nb0 ? 1 : 0);
}

// q_x duplicated into both halves of a bf16 pair.
template <int X>
__device__ __forceinline__ uint32_t dup_q(const uint32_t (&q2)[32]) {
    return __byte_perm(q2[X / 2], 0, (X & 1) ? 0x3232 : 0x1010);
}

__host__ __device__ constexpr uint32_t bf16_small(int c) { return c == 2 ? 0x4000u : c == 1 ? 0x3F80u : 0u; }
__host__ __device__ constexpr int pair_weight(PairIJ p) { return p.i < p.j ? 2 : p.i == p.j ? 1 : 0; }

// Word of phi(q) holding state rows R and R + 1 (tensor-memory A layout: row
// pair (2p, 2p+1) in column p): c_ij q_i q_j for both rows, c = 2 for i < j,
// 1 for i = j, 0 for padding rows.  The layout makes the word q_i (q_j,
// q_j+1) or (q_i, q_i+1) q_j, one bf16x2 product; a common factor 2 is put on
// the duplicated operand (exact), other weights multiply the product (exact).
template <int G, int R>
__device__ __forceinline__ uint32_t gen_word(const uint32_t (&q2)[32]) {
    constexpr PairIJ a = row_ij_g(G, R), b = row_ij_g(G, R + 1);
    constexpr int c0 = pair_weight(a), c1 = pair_weight(b);
    static_assert((a.i == b.i && b.j == a.j + 1 && a.j % 2 == 0) ||
                      (a.j == b.j && b.i == a.i + 1 && a.i % 2 == 0),
                  "state rows of one word must share i or j");
    constexpr bool share_i = a.i == b.i;
    if constexpr (c0 == 0 && c1 == 0) {
        return 0u;
    } else {
        uint32_t dup = share_i ? dup_q<a.i>(q2) : dup_q<a.j>(q2);
        const uint32_t pr = share_i ? q2[a.j / 2] : q2[a.i / 2];
        if constexpr (c0 == 2 && c1 == 2) dup = mul_bf16x2(dup, 0x40004000u);
        uint32_t w = mul_bf16x2(dup, pr);
        if constexpr (!(c0 == 2 && c1 == 2) && !(c0 == 1 && c1 == 1))
            w = mul_bf16x2(w, bf16_small(c0) | (bf16_small(c1) << 16));
        return w;
    }
}

// The 8 words of K-step K (state rows 16 K .. 16 K + 15).
template <int G, int K>
__device__ __forceinline__ void gen_kstep(const uint32_t (&q2)[32], uint32_t *out) {
    out[0] = gen_word<G, 16 * K + 0>(q2);
    out[1] = gen_word<G, 16 * K + 2>(q2);
    out[2] = gen_word<G, 16 * K + 4>(q2);
    out[3] = gen_word<G, 16 * K + 6>(q2);
    out[4] = gen_word<G, 16 * K + 8>(q2);
    out[5] = gen_word<G, 16 * K + 10>(q2);
    out[6] = gen_word<G, 16 * K + 12>(q2);
    out[7] = gen_word<G, 16 * K + 14>(q2);
}

// First half (K-steps 0-3) of inter stage ST.
template <int G, int ST>
__device__ __forceinline__ void gen_stage_lo(const uint32_t (&q2)[32], uint32_t (&x)[32]) {
    gen_kstep<G, kRKs * ST + 0>(q2, x);
    gen_kstep<G, kRKs * ST + 1>(q2, x + 8);
    gen_kstep<G, kRKs * ST + 2>(q2, x + 16);
    gen_kstep<G, kRKs * ST + 3>(q2, x + 24);
}

// Generates the inter stages of one item into the A ring, software-pipelined:
// the first half of stage ST (`x`) was generated before its slot frees up;
// while the tensor-memory stores of stage ST are in flight, the first half of
// stage ST + 1 is generated.  `g0` is the number of stages generated before
// this item (ring slot and phase).
template <int G, int ST>
__device__ __forceinline__ bool gen_loop(const uint32_t (&q2)[32], ReadBars &bars, uint32_t ta_tile,
                                         int g0, volatile int *abort, const uint32_t (&x)[32]) {
    const int n = g0 + ST;
    const int s = n % kRRing;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars.aempty[s], ((n / kRRing) & 1) ^ 1, abort)))
        return false;
    tc_fence_after();
    tmem_st32(ta_tile + 128 * s, x);
    {
        uint32_t y[16];
        gen_kstep<G, kRKs * ST + 4>(q2, y);
        gen_kstep<G, kRKs * ST + 5>(q2, y + 8);
        tmem_st16(ta_tile + 128 * s + 32, y);
    }
    {
        uint32_t y[16];
        gen_kstep<G, kRKs * ST + 6>(q2, y);
        gen_kstep<G, kRKs * ST + 7>(q2, y + 8);
        tmem_st16(ta_tile + 128 * s + 48, y);
    }
    if constexpr (ST + 1 < read_stages(G)) {
        uint32_t xn[32];
        gen_stage_lo<G, ST + 1>(q2, xn);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars.afull[s]);
        return gen_loop<G, ST + 1>(q2, bars, ta_tile, g0, abort, xn);
    } else {
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars.afull[s]);
        return true;
    }
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    const uint32_t s = smem_u32(p);
    return p + ((1024u - (s & 1023u)) & 1023u);
}

__device__ __forceinline__ void set_timeout_status(int *status) {
    atomicCAS(status, 0, (int)KATA_ERR_TIMEOUT);
}

// Start address of a descriptor advanced by `bytes` (16-byte units in the low bits).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// ---------------------------------------------------------------------------
// State builder on tcgen05 (persistent: one CTA per SM loops over work items).
//
// Work item = (head, segment, c), c = 0..4; item c accumulates its state
// tiles (4 tiles for c < 4, the single tile 16 for c = 4; rows as laid out in
// tc_layout.cuh) over the segment's tokens:  D[m] += A[m] . [V | 1]  with
// A[m][(i, j)][token] = k_i k_j generated from the transposed keys into tensor
// memory by the thread owning the row's lane (from the key tile transposed in
// shared memory), and the MN-major B operand
// [V | 1] = the value tile (64 columns) followed by a constant block whose
// first column is one, so column 64 of D accumulates the packed normaliser
// z = sum k_i k_j (N = 80; an N = 64 MMA costs the same issue time).
// Roles: warps 0-3 / 4-7 generate the first / second 16-token step of every
// 32-token stage (software-pipelined: the next stage's products are formed
// while this stage's tensor-memory stores are in flight) and drain the
// accumulators into swizzled shared memory; warp 8 loads the key and value
// tiles by TMA and warp 12 transposes each key tile in place once it has
// landed (d x tokens, so a thread reads 16 consecutive tokens of one feature
// as one 32-byte run);
// warps 9 and 10 issue the MMAs of alternate stages; warp 11 writes the
// drained tiles back with TMA stores, so the next item's MMAs start as soon as
// the accumulators are read.  Barrier phases run on across items.
// Accumulators are zeroed by tcgen05.st and every MMA accumulates.
// ---------------------------------------------------------------------------
constexpr int kBTiles = 4;                // accumulator tiles (the most an item uses)
constexpr int kBN = 80;                   // MMA N: 64 values, the ones column, 15 zero columns
constexpr int kBTok = 64;                 // tokens per TMA tile (2 stages)
constexpr int kBTileRing = 5;
constexpr int kBTileBytes = 2 * 8192;     // key tile (transposed in place), value tile
constexpr int kBOnes = kBTileRing * kBTileBytes;   // ones block [64 x 64] bf16, swizzled
constexpr int kBStage = kBOnes + 8192;             // staging: tile m, half h at + (2 m + h) * 16 KB
constexpr int kBStageBox = 16384;                  // [128 rows x 32 fp32], 128-byte swizzle
constexpr int kBSmAlloc = kBStage + 2 * kBTiles * kBStageBox + 1024;
constexpr int kBARing = 3;                // A stages in tensor memory
constexpr int kBTmaWarp = 8;
constexpr int kBIssuer0 = 9;
constexpr int kBStoreWarp = 11;
constexpr int kBTransWarp = 12;
constexpr int kBuildThreads = 416;
constexpr uint32_t kBTmA = kBTiles * kBN; // 320: A slot s at 320 + 64 s, step kk at + 32 kk

struct BuildBars {
    // kraw: a tile's keys and values landed (the issuers need only the values);
    // tfull: its keys transposed (the generation warps read them); tempty: the
    // slot may be refilled
    uint64_t kraw[kBTileRing], tfull[kBTileRing], tempty[kBTileRing];
    uint64_t afull[kBARing], aempty[kBARing];
    uint64_t done, staged, sfree;
    uint64_t drain[2];
};

// In-place transpose of one [64 tokens x 64 features] bf16 key tile in the
// 128-byte swizzle (16-byte chunk c of row r at chunk c ^ (r % 8)) into
// [64 features x 64 tokens] in the same swizzle, by one warp.  The tile is a
// grid of 8 x 8 blocks of 8 x 8 elements; block (R, C) (tokens 8R.., features
// 8C..) becomes block (C, R) transposed.  Lane l + 8 q takes the blocks
// (l, (l + q) % 8) and (l, (l + q + 4) % 8): in every 8-lane phase of a
// 16-byte access the lanes touch 8 distinct chunk columns, on the loads
// (C ^ u) and on the stores (R ^ u), so neither conflicts.  Every lane reads
// both its blocks before any lane writes.
__device__ __forceinline__ void transpose_key_tile(uint8_t *tile, int lane) {
    const int R = lane & 7, q = lane >> 3;
    uint32_t a[2][8][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int C = (R + q + 4 * h) & 7;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint4 x = *reinterpret_cast<const uint4 *>(tile + (8 * R + u) * 128 + ((C ^ u) * 16));
            a[h][u][0] = x.x;
            a[h][u][1] = x.y;
            a[h][u][2] = x.z;
            a[h][u][3] = x.w;
        }
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int C = (R + q + 4 * h) & 7;
        // row v (feature 8C + v) of the transposed block: tokens 2w, 2w + 1 in word w
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const uint32_t sel = (v & 1) ? 0x7632u : 0x5410u;
            uint4 y;
            y.x = __byte_perm(a[h][0][v >> 1], a[h][1][v >> 1], sel);
            y.y = __byte_perm(a[h][2][v >> 1], a[h][3][v >> 1], sel);
            y.z = __byte_perm(a[h][4][v >> 1], a[h][5][v >> 1], sel);
            y.w = __byte_perm(a[h][6][v >> 1], a[h][7][v >> 1], sel);
            *reinterpret_cast<uint4 *>(tile + (8 * C + v) * 128 + ((R ^ v) * 16)) = y;
        }
    }
}

// Products k_i k_j of one 16-token step (this warpgroup's half of a 32-token
// stage) for the thread's NT rows: p[8 m + w] holds tokens 2 w, 2 w + 1.
template <int NT>
__device__ __forceinline__ void build_products(const uint8_t *kt, int half, int wg, int jcol,
                                               const int (&im)[kBTiles], uint32_t (&p)[8 * NT]) {
    const int c0 = 4 * half + 2 * wg, c1 = c0 + 1;  // 16-byte chunks of this warpgroup's 16 tokens
    uint32_t own[8];
    {
        const uint8_t *r = kt + jcol * 128;
        const uint4 x0 = *reinterpret_cast<const uint4 *>(r + ((c0 ^ (jcol & 7)) * 16));
        const uint4 x1 = *reinterpret_cast<const uint4 *>(r + ((c1 ^ (jcol & 7)) * 16));
        own[0] = x0.x; own[1] = x0.y; own[2] = x0.z; own[3] = x0.w;
        own[4] = x1.x; own[5] = x1.y; own[6] = x1.z; own[7] = x1.w;
    }
#pragma unroll
    for (int m = 0; m < NT; ++m) {
        const int i = im[m];
        const uint8_t *r = kt + i * 128;
        const uint4 x0 = *reinterpret_cast<const uint4 *>(r + ((c0 ^ (i & 7)) * 16));
        const uint4 x1 = *reinterpret_cast<const uint4 *>(r + ((c1 ^ (i & 7)) * 16));
        p[8 * m + 0] = mul_bf16x2(own[0], x0.x); p[8 * m + 1] = mul_bf16x2(own[1], x0.y);
        p[8 * m + 2] = mul_bf16x2(own[2], x0.z); p[8 * m + 3] = mul_bf16x2(own[3], x0.w);
        p[8 * m + 4] = mul_bf16x2(own[4], x1.x); p[8 * m + 5] = mul_bf16x2(own[5], x1.y);
        p[8 * m + 6] = mul_bf16x2(own[6], x1.z); p[8 * m + 7] = mul_bf16x2(own[7], x1.w);
    }
}

template <int NT>
__device__ __forceinline__ void build_store(uint32_t taddr, const uint32_t (&p)[8 * NT]) {
    if constexpr (NT == 4) tmem_st32(taddr, p);
    else tmem_st8(taddr, p);
}

// Generation side of one item: 2 stages per 64-token tile.  `tt` is the
// CTA's running tile counter (ring slot and phase), advanced past the item.
template <int NT>
__device__ __forceinline__ bool build_item_gen(BuildBars &bars, const uint8_t *sm, uint32_t ta, int wg,
                                               int jcol, const int (&im)[kBTiles], int &tt, int n_tt,
                                               volatile int *abort) {
    uint32_t pa[8 * NT], pb[8 * NT];
    {
        const int b = tt % kBTileRing;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.tfull[b], (tt / kBTileRing) & 1, abort))) return false;
        build_products<NT>(sm + b * kBTileBytes, 0, wg, jcol, im, pa);
    }
    for (int t = 0; t < n_tt; ++t, ++tt) {
        const int b = tt % kBTileRing;
        int G = 2 * tt, a = G % kBARing;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.aempty[a], ((G / kBARing) & 1) ^ 1, abort)))
            return false;
        tc_fence_after();
        build_store<NT>(ta + 64 * a, pa);
        build_products<NT>(sm + b * kBTileBytes, 1, wg, jcol, im, pb);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars.afull[a]);

        G = 2 * tt + 1;
        a = G % kBARing;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.aempty[a], ((G / kBARing) & 1) ^ 1, abort)))
            return false;
        tc_fence_after();
        build_store<NT>(ta + 64 * a, pb);
        if (t + 1 < n_tt) {
            const int bn = (tt + 1) % kBTileRing;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars.tfull[bn], ((tt + 1) / kBTileRing) & 1, abort)))
                return false;
            build_products<NT>(sm + bn * kBTileBytes, 0, wg, jcol, im, pa);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars.afull[a]);
    }
    return true;
}

template <int G>
__device__ __forceinline__ void build_item_geom(int item, int n_build, int T, int L, int &c, int &g, int &bh,
                                                int &s0, int &n_tt) {
    c = item % build_items(G);
    const int rest = item / build_items(G);
    g = rest % n_build;
    bh = rest / n_build;
    s0 = g * L;
    n_tt = (min(L, T - s0) + kBTok - 1) / kBTok;
}

template <int G>
__global__ void __launch_bounds__(kBuildThreads, 1)
tc_build(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
         const __grid_constant__ CUtensorMap tm_st, float *__restrict__ seg_state, int T, int L,
         int n_seg, int n_build, int n_items, int *status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ BuildBars bars;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    uint8_t *sm = align1024(smem_raw);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

    if (tid == 0) {
        abort_flag = 0;
        for (int x = 0; x < kBTileRing; ++x) {
            mbar_init(&bars.kraw[x], 1);
            mbar_init(&bars.tfull[x], 32);  // every lane of the transposing warp
            mbar_init(&bars.tempty[x], 2);
        }
        for (int x = 0; x < kBARing; ++x) {
            mbar_init(&bars.afull[x], 256);
            mbar_init(&bars.aempty[x], 1);
        }
        mbar_init(&bars.done, 2);
        mbar_init(&bars.staged, 256);
        mbar_init(&bars.sfree, 1);
        mbar_init(&bars.drain[0], 1);
        mbar_init(&bars.drain[1], 1);
        fence_mbarrier_init();
    }
    // constant ones block: logical column 0 of each of the 64 rows is 1.0
    for (int x = tid; x < 8192 / 4; x += kBuildThreads) {
        const int r = x / 32, w = x % 32;  // 32-bit word w of row r
        reinterpret_cast<uint32_t *>(sm + kBOnes)[x] = (w == 4 * (r & 7)) ? 0x3F80u : 0u;
    }
    fence_proxy_async_smem();
    if (warp == kBIssuer0) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    volatile int *abort = &abort_flag;
    griddep_launch_dependents();  // the scan may start launching (it waits for this grid to finish)

    if (warp == kBTmaWarp) {
        // ------------------------------------------------------------ producer
        // the key tile (row-major: zero rows past T) and the value tile of each
        // 64-token tile, on a CTA-wide tile counter across items
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int tt = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                int c, g, bh, s0, n_tt;
                build_item_geom<G>(item, n_build, T, L, c, g, bh, s0, n_tt);
                for (int t = 0; t < n_tt; ++t, ++tt) {
                    const int b = tt % kBTileRing;
                    ok = mbar_wait(&bars.tempty[b], ((tt / kBTileRing) & 1) ^ 1, abort);
                    if (!ok) break;
                    uint8_t *st = sm + b * kBTileBytes;
                    mbar_arrive_expect_tx(&bars.kraw[b], kBTileBytes);
                    tma_load_3d(st, &tm_k, &bars.kraw[b], 0, s0 + kBTok * t, bh);
                    tma_load_3d(st + 8192, &tm_v, &bars.kraw[b], 0, s0 + kBTok * t, bh);
                }
            }
            // every load issued must have landed before the CTA exits
            for (int t = (tt > kBTileRing ? tt - kBTileRing : 0); t < tt; ++t)
                mbar_wait_issued(&bars.kraw[t % kBTileRing], (t / kBTileRing) & 1);
        }
    } else if (warp == kBTransWarp) {
        // ------------------------------------------------------------ key transposer
        // each key tile, once landed, transposed in place for the generation warps
        int tt = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            int c, g, bh, s0, n_tt;
            build_item_geom<G>(item, n_build, T, L, c, g, bh, s0, n_tt);
            for (int t = 0; t < n_tt; ++t, ++tt) {
                const int b = tt % kBTileRing;
                ok = __all_sync(0xffffffffu, mbar_wait(&bars.kraw[b], (tt / kBTileRing) & 1, abort));
                if (!ok) break;
                transpose_key_tile(sm + b * kBTileBytes, lane);
                mbar_arrive(&bars.tfull[b]);
            }
        }
    } else if (warp == kBIssuer0 || warp == kBIssuer0 + 1) {
        // ------------------------------------------------------------ MMA issuers
        if (lane == 0) {
            const int me = warp - kBIssuer0;
            const uint32_t idesc = idesc_bf16(128, kBN, 0, 1);
            const uint32_t sbase = smem_u32(sm);
            int tt = 0;  // global tile counter
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                int c, g, bh, s0, n_tt;
                build_item_geom<G>(item, n_build, T, L, c, g, bh, s0, n_tt);
                const int nt = build_item_tiles(G, c);
                for (int t = 0; t < n_tt && ok; ++t, ++tt) {
                    const int gs = 2 * tt + me;  // global stage: this issuer takes one half of each tile
                    const int b = tt % kBTileRing, a = gs % kBARing;
                    ok = mbar_wait(&bars.kraw[b], (tt / kBTileRing) & 1, abort) &&
                         mbar_wait(&bars.afull[a], (gs / kBARing) & 1, abort);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t vaddr = sbase + b * kBTileBytes + 8192 + 4096 * me;
                    const uint32_t oaddr = sbase + kBOnes + 4096 * me;
                    const uint64_t dv = desc_sw128(vaddr, oaddr - vaddr, 1024);
                    const uint32_t ta = tm + kBTmA + 64 * a;
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
#pragma unroll
                        for (int m = 0; m < kBTiles; ++m)
                            if (m < nt)
                                mma_ts(tm + kBN * m, ta + 32 * kk + 8 * m, desc_add(dv, 2048 * kk), idesc, 1);
                    mma_commit(&bars.aempty[a]);
                    mma_commit(&bars.tempty[b]);
                }
                if (ok) mma_commit(&bars.done);  // this item's accumulation complete (with the other issuer)
            }
            // no MMA of this CTA may still read or write tensor memory when it is freed
            mma_commit(&bars.drain[me]);
            mbar_wait_issued(&bars.drain[me], 0);
        }
    } else if (warp == kBStoreWarp) {
        // ------------------------------------------------------------ write-back of drained tiles
        if (lane == 0) {
            tma_prefetch_desc(&tm_st);
            int j = 0;
            for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++j) {
                int c, g, bh, s0, n_tt;
                build_item_geom<G>(item, n_build, T, L, c, g, bh, s0, n_tt);
                if (!mbar_wait(&bars.staged, j & 1, abort)) break;
                for (int m = 0; m < build_item_tiles(G, c); ++m)
                    for (int h = 0; h < 2; ++h)
                        tma_store_3d(&tm_st, sm + kBStage + (2 * m + h) * kBStageBox, 32 * h,
                                     128 * build_item_tile(G, c, m), bh * n_seg + g);
                bulk_commit_group();
                bulk_wait_read_all();
                mbar_arrive(&bars.sfree);
            }
            bulk_wait_all();
        }
    } else {
        // ------------------------------------------------------------ generation / drain
        const int wg = warp / 4, qd = warp % 4;
        const int row = 32 * qd + lane;          // lane within the 128-row tile
        const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
        uint32_t zero[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) zero[x] = 0u;
        // zero this warpgroup's accumulators (tiles 2 wg, 2 wg + 1; 80 columns each)
        auto zero_acc = [&]() {
#pragma unroll
            for (int m = 2 * wg; m < 2 * wg + 2; ++m) {
                tmem_st32(tm + kBN * m + lane_base, zero);
                tmem_st32(tm + kBN * m + 32 + lane_base, zero);
                tmem_st16(tm + kBN * m + 64 + lane_base, zero);
            }
        };
        zero_acc();
        int tt = 0, j = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++j) {
            int c, g, bh, s0, n_tt;
            build_item_geom<G>(item, n_build, T, L, c, g, bh, s0, n_tt);
            const int nt = build_item_tiles(G, c);
            int im[kBTiles], jcol = 0;
#pragma unroll
            for (int m = 0; m < kBTiles; ++m) {
                const PairIJ pij = row_ij_g(G, 128 * build_item_tile(G, c, m < nt ? m : 0) + row);
                im[m] = pij.i;
                jcol = pij.j;  // the same for every tile of the item
            }
            const uint32_t ta = tm + kBTmA + 32 * wg + lane_base;
            ok = nt == kBTiles ? build_item_gen<kBTiles>(bars, sm, ta, wg, jcol, im, tt, n_tt, abort)
                               : build_item_gen<1>(bars, sm, ta, wg, jcol, im, tt, n_tt, abort);
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars.done, j & 1, abort));
            if (ok && j > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars.sfree, (j - 1) & 1, abort));
            if (!ok) break;
            // Drain: tile m's 128 rows go to shared memory as two [128 x 32] fp32
            // boxes in the 128-byte swizzle of the store's tensor map (16-byte
            // chunk c of row r at chunk c ^ (r % 8): conflict-free), its packed z
            // (column 64) straight to global memory.
            tc_fence_after();
            float *zbase = seg_state + ((long long)bh * n_seg + g) * f32_per_seg(G) + z_packed0(G);
            for (int m = 2 * wg; m < 2 * wg + 2 && m < nt; ++m) {
                uint32_t o[32];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    tmem_ld32(tm + kBN * m + 32 * h + lane_base, o);
                    tmem_ld_wait();
                    uint8_t *box = sm + kBStage + (2 * m + h) * kBStageBox + row * 128;
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        *reinterpret_cast<uint4 *>(box + ((x ^ (row & 7)) * 16)) =
                            make_uint4(o[4 * x], o[4 * x + 1], o[4 * x + 2], o[4 * x + 3]);
                }
                tmem_ld8(tm + kBN * m + 64 + lane_base, o);
                tmem_ld_wait();
                zbase[128 * build_item_tile(G, c, m) + row] = __uint_as_float(o[0]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars.staged);
            zero_acc();  // ordered before the next item's first MMA by the hand-off's tcgen05.st wait
        }
        tmem_st_wait();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBIssuer0) tmem_dealloc(tm, 512);
    if (tid == 0 && abort_flag) set_timeout_status(status);
}

// G: factors of the state layout (inter phase); GI: factors of the
// intra-segment weight (1: (q.k)^2 in 128-key steps; 2: the sum over the two
// factors in 64-key steps).  A single-factor head of d <= 32 runs G = 2,
// GI = 1: its state on the two-factor layout, its scores whole.
template <int G, int GI>
__global__ void __launch_bounds__(kReadThreads, 1)
tc_read(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_s,
        const __grid_constant__ CUtensorMap tm_o, int T, int L, int n_seg, int n_ct, int n_items,
        bool has_init, int qk_ks, int *status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ ReadBars bars;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    uint8_t *sm = align1024(smem_raw);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const ReadSched sched = read_sched(n_items, n_ct, n_seg);

    if (tid == 0) {
        abort_flag = 0;
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.qfull[b], 1);
            mbar_init(&bars.qempty[b], 3);  // both issuers' commits + the output store's read
            mbar_init(&bars.drain[b], 1);
        }
        for (int b = 0; b < kKVMax; ++b) {
            mbar_init(&bars.kfull[b], 1);
            mbar_init(&bars.kempty[b], 1);
            mbar_init(&bars.vfull[b], 1);
            mbar_init(&bars.vempty[b], 1);
        }
        mbar_init(&bars.u, 1);
        mbar_init(&bars.interdone, 2);
        mbar_init(&bars.done, 2);
        mbar_init(&bars.genin, 8);
        mbar_init(&bars.ostaged[0], 8);
        mbar_init(&bars.ostaged[1], 8);
        for (int s = 0; s < kRBRing; ++s) {
            mbar_init(&bars.bfull[s], 1);
            mbar_init(&bars.bempty[s], 1);
        }
        for (int s = 0; s < kRRing; ++s) {
            mbar_init(&bars.afull[s], 8 * 32);
            mbar_init(&bars.aempty[s], 1);
        }
        for (int x = 0; x < kSBufs; ++x) {
            mbar_init(&bars.sfull[x], 1);
            mbar_init(&bars.pfull[x], 4);  // one arrival per squaring warp of the step's tile
            mbar_init(&bars.bfree[x], 1);
        }
        fence_mbarrier_init();
    }
    if (warp == kIssuer0) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    volatile int *abort = &abort_flag;

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_s);
            int n_q = 0, n_bs = 0, n_kv = 0, n_v = 0;  // loads issued into each ring (n_kv: keys)
            bool ok = true, scanned = false;
            for (int x = sched.first; x < sched.end && ok; x += sched.stride) {
                const ReadItem it = read_item<GI>(sched.item(x), n_ct, T, L, n_seg, has_init);
                // Launched as the scan's programmatic dependent (small problems),
                // this kernel may run while the scan does: the prefixes (the one
                // input the scan writes) are loaded only after griddepcontrol.wait,
                // while queries, keys and values, and the items without an inter
                // phase, go ahead.  Other threads read no global memory before
                // this thread's loads land.
                if (it.inter && !scanned) {
                    griddep_wait();
                    scanned = true;
                }
                {
                    const int qb = n_q & 1;
                    uint8_t *slot = sm + kSmItem + qb * kItemBytes;
                    ok = mbar_wait(&bars.qempty[qb], ((n_q >> 1) & 1) ^ 1, abort);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&bars.qfull[qb], kTiles * 16384);
                    for (int t = 0; t < kTiles; ++t)
                        tma_load_3d(slot + t * 16384, &tm_q, &bars.qfull[qb], 0, it.t0 + t * kQT, it.bh);
                    ++n_q;
                }
                // entry -1: Z hi / lo (the 128 prefix rows from zhi_row0); then the stages
                for (int st = -1; it.inter && st < read_stages(G) && ok; ++st) {
                    const int s = n_bs % kRBRing;
                    ok = mbar_wait(&bars.bempty[s], ((n_bs / kRBRing) & 1) ^ 1, abort);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&bars.bfull[s], kRStageBytes);
                    const int row0 = st < 0 ? zhi_row0(G) : 16 * kRKs * st;
                    for (int bx = 0; bx < kRStageBytes / 4096; ++bx)
                        tma_load_3d(sm + kSmS + s * kRStageBytes + 4096 * bx, &tm_s, &bars.bfull[s], 0,
                                    row0 + 32 * bx, it.sidx);
                    ++n_bs;
                }
                for (int kb = 0; kb < it.n_kv && ok; ++kb) {
                    const int s = n_kv % kv_ring(GI);
                    const uint32_t par = ((n_kv / kv_ring(GI)) & 1) ^ 1;
                    ok = mbar_wait(&bars.kempty[s], par, abort);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&bars.kfull[s], kv_bytes(GI));
                    tma_load_3d(sm + kSmK + s * kv_bytes(GI), &tm_k, &bars.kfull[s], 0,
                                it.seg0 + kb * step_keys(GI), it.bh);
                    ok = mbar_wait(&bars.vempty[s], par, abort);
                    if (!ok) {
                        ++n_kv;  // its keys are in flight: waited for below
                        break;
                    }
                    mbar_arrive_expect_tx(&bars.vfull[s], kv_bytes(GI));
                    tma_load_3d(sm + kSmV + s * kv_bytes(GI), &tm_v, &bars.vfull[s], 0,
                                it.seg0 + kb * step_keys(GI), it.bh);
                    ++n_kv;
                    ++n_v;
                }
            }
            // no CTA finishes before the scan (a CTA whose items have no inter
            // phase waits here)
            if (!scanned) griddep_wait();
            // every load issued must have landed before the CTA exits
            for (int x = (n_q > 2 ? n_q - 2 : 0); x < n_q; ++x)
                mbar_wait_issued(&bars.qfull[x & 1], (x >> 1) & 1);
            for (int x = (n_bs > kRBRing ? n_bs - kRBRing : 0); x < n_bs; ++x)
                mbar_wait_issued(&bars.bfull[x % kRBRing], (x / kRBRing) & 1);
            for (int x = (n_kv > kv_ring(GI) ? n_kv - kv_ring(GI) : 0); x < n_kv; ++x)
                mbar_wait_issued(&bars.kfull[x % kv_ring(GI)], (x / kv_ring(GI)) & 1);
            for (int x = (n_v > kv_ring(GI) ? n_v - kv_ring(GI) : 0); x < n_v; ++x)
                mbar_wait_issued(&bars.vfull[x % kv_ring(GI)], (x / kv_ring(GI)) & 1);
        }
    } else if (warp == kIssuer0 || warp == kIssuer0 + 1) {
        // ------------------------------------------------------------ MMA issuers
        if (lane == 0) {
            const int me = warp - kIssuer0;
            const uint32_t id_n64 = idesc_bf16(kQT, 64, 0, 1);  // B MN-major, N = 64
            // scores: B = keys, K-major; N = 128 keys (one factor) or 64 per factor
            const uint32_t id_qk = idesc_bf16(kQT, GI == 1 ? 128 : 64, 0, 0);
            const uint64_t dS = desc_sw128(smem_u32(sm + kSmS), 8192, 1024);
            const uint64_t dK = desc_sw128(smem_u32(sm + kSmK), 16, 1024);
            const uint64_t dV = desc_sw128(smem_u32(sm + kSmV), 8192, 1024);
            int n_inter = 0, g_kv = 0, ns = 0, j = 0;  // ns: the CTA's intra step count
            // issuer 0, per score buffer (4 bits each): the key/value slot + 1 whose
            // values the buffer's current step finishes reading, or 0
            uint32_t vrel = 0;
            bool ok = true;
            for (int x = sched.first; x < sched.end && ok; x += sched.stride, ++j) {
                const ReadItem it = read_item<GI>(sched.item(x), n_ct, T, L, n_seg, has_init);
                const int qb = j & 1;
                const uint32_t slot = smem_u32(sm + kSmItem + qb * kItemBytes);
                ok = mbar_wait(&bars.qfull[qb], (j >> 1) & 1, abort);
                if (!ok) break;
                tc_fence_after();
                if (it.inter) {
                    if (me == 0) {
                        // U = Q (Z hi + Z lo) into columns that held the previous item's weights
                        if (j > 0) {
                            ok = mbar_wait(&bars.done, (j - 1) & 1, abort);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        // Z hi / lo: the item's first state-prefix ring entry
                        const int ze = n_inter * (read_stages(G) + 1), zs = ze % kRBRing;
                        ok = mbar_wait(&bars.bfull[zs], (ze / kRBRing) & 1, abort);
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t dZ = desc_add(dS, kRStageBytes * zs);
                        for (int u = 0; u < kTiles; ++u) {
                            const uint64_t dq = desc_sw128(slot + u * 16384, 16, 1024);
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_ss(tm + kTmU + 64 * u, desc_add(dq, 32 * ks), desc_add(dZ, 2048 * ks),
                                       id_n64, ks > 0);
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_ss(tm + kTmU + 64 * u, desc_add(dq, 32 * ks),
                                       desc_add(dZ, 8192 + 2048 * ks), id_n64, 1);
                        }
                        mma_commit(&bars.u);
                        mma_commit(&bars.bempty[zs]);
                    }
                    for (int st = me; st < read_stages(G) && ok; st += 2) {
                        // gs: the CTA's inter stage count (A ring); be: its prefix ring entry
                        const int gs = n_inter * read_stages(G) + st, be = n_inter * (read_stages(G) + 1) + 1 + st;
                        const int s = gs % kRRing, sb = be % kRBRing;
                        // the A stage first: the generation warps start after U, so the
                        // ring entry before this one (perhaps Z, the other issuer's) is done
                        ok = mbar_wait(&bars.afull[s], (gs / kRRing) & 1, abort) &&
                             mbar_wait(&bars.bfull[sb], (be / kRBRing) & 1, abort);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t ta = tm + kTmA + 128 * s;
                        const uint64_t db = desc_add(dS, kRStageBytes * sb);
#pragma unroll
                        for (int ks = 0; ks < kRKs; ++ks) {
                            mma_ts(tm + kTmO, ta + 8 * ks, desc_add(db, 2048 * ks), id_n64, 1);
                            mma_ts(tm + kTmO + 64, ta + 64 + 8 * ks, desc_add(db, 2048 * ks), id_n64, 1);
                        }
                        mma_commit(&bars.bempty[sb]);
                        mma_commit(&bars.aempty[s]);
                    }
                    if (!ok) break;
                    mma_commit(&bars.interdone);
                    // the scores reuse the A ring's columns: every inter MMA must be done
                    ok = mbar_wait(&bars.interdone, n_inter & 1, abort);
                    if (!ok) break;
                    tc_fence_after();
                    ++n_inter;
                }
                // Intra phase, step by step (key block b, tile t; b-major).  Issuer 0
                // forms the scores of step n in buffer n % 3 once the weights times
                // values of step n - 3 have freed it; issuer 1 multiplies the step's
                // weights, stored over its scores, by the values.  Each issuer
                // releases key/value block b after its last step of the block.
                const int nb[kTiles] = {read_tile_blocks<GI>(it, 0, T), read_tile_blocks<GI>(it, 1, T)};
                const int nbm = max(nb[0], nb[1]);
                for (int b = 0; b < nbm && ok; ++b) {
                    const int kvb = g_kv + b, kvs = kvb % kv_ring(GI);
                    // issuer 0 reads the block's keys; issuer 1 its values, which the
                    // squaring warps have seen land before they hand over the weights
                    if (me == 0) ok = mbar_wait(&bars.kfull[kvs], (kvb / kv_ring(GI)) & 1, abort);
                    for (int t = 0; t < kTiles && ok; ++t) {
                        if (b >= nb[t]) continue;
                        const int x = ns % kSBufs;
                        const uint32_t buf = tm + kTmBuf + 128 * x;
                        if (me == 0) {
                            if (ns >= kSBufs) {
                                ok = mbar_wait(&bars.bfree[x], ((ns - kSBufs) / kSBufs) & 1, abort);
                                if (!ok) break;
                                // step ns - 3 was the last of its block: that block's values are read
                                const uint32_t code = (vrel >> (4 * x)) & 15u;
                                if (code) mbar_arrive(&bars.vempty[code - 1]);
                            }
                            // this step's block slot + 1 if it is the block's last step
                            // (tile 1's, or tile 0's when tile 1 has no block b), else 0
                            const bool last = t == 1 || b >= nb[1];
                            vrel = (vrel & ~(15u << (4 * x))) | ((last ? kvs + 1u : 0u) << (4 * x));
                            tc_fence_after();
                            const uint64_t dk = desc_add(dK, kv_bytes(GI) * kvs);
                            const uint64_t dQt = desc_sw128(slot + t * 16384, 16, 1024);
                            if constexpr (GI == 1) {
                                // K-steps of the head's own coordinates only (qk_ks = d / 16:
                                // the columns past d are zeros)
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)
                                    if (ks < qk_ks)
                                        mma_ss(buf, desc_add(dQt, 32 * ks), desc_add(dk, 32 * ks), id_qk, ks > 0);
                            } else {
                                // one score per factor: coordinates 0-31 (K-steps 0, 1) into
                                // columns 0-63 of the buffer, 32-63 (K-steps 2, 3) into 64-127
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)
                                    mma_ss(buf + 64 * (ks / 2), desc_add(dQt, 32 * ks), desc_add(dk, 32 * ks),
                                           id_qk, (ks & 1) != 0);
                            }
                            mma_commit(&bars.sfull[x]);
                        } else {
                            ok = mbar_wait(&bars.pfull[x], (ns / kSBufs) & 1, abort);
                            if (!ok) break;
                            tc_fence_after();
                            const uint64_t dv = desc_add(dV, kv_bytes(GI) * kvs);
#pragma unroll
                            for (int ks = 0; ks < step_keys(GI) / 16; ++ks)
                                mma_ts(tm + kTmO + 64 * t, buf + 8 * ks, desc_add(dv, 2048 * ks), id_n64, 1);
                            mma_commit(&bars.bfree[x]);
                        }
                        ++ns;
                    }
                    if (!ok) break;
                }
                if (!ok) break;
                g_kv += it.n_kv;
                // every generation warp has entered this item, so `done` cannot run a phase ahead of it
                ok = mbar_wait(&bars.genin, j & 1, abort);
                if (!ok) break;
                mma_commit(&bars.done);
                mma_commit(&bars.qempty[qb]);
            }
            // no MMA of this CTA may still read or write tensor memory when it is freed
            mma_commit(&bars.drain[me]);
            mbar_wait_issued(&bars.drain[me], 0);
        }
    } else if (warp == kStoreWarp) {
        // ------------------------------------------------------------ output write-back
        if (lane == 0) {
            tma_prefetch_desc(&tm_o);
            int j = 0;
            for (int x = sched.first; x < sched.end; x += sched.stride, ++j) {
                const ReadItem it = read_item<GI>(sched.item(x), n_ct, T, L, n_seg, has_init);
                const int qb = j & 1;
                if (!mbar_wait(&bars.ostaged[qb], (j >> 1) & 1, abort)) break;
                for (int t = 0; t < kTiles; ++t)
                    if (it.t0 + kQT * t < T)
                        tma_store_3d(&tm_o, sm + kSmItem + qb * kItemBytes + t * 16384, 0, it.t0 + kQT * t, it.bh);
                bulk_commit_group();
                bulk_wait_read_all();
                mbar_arrive(&bars.qempty[qb]);  // the slot may be refilled
            }
            bulk_wait_all();
        }
    } else {
        // ------------------------------------------------------------ generation / scores / epilogue
        const int t = warp / 4, qd = warp % 4;
        const int row = 32 * qd + lane;
        const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
        const uint32_t tO = tm + kTmO + 64 * t + lane_base;
        const uint32_t tU = tm + kTmU + 64 * t + lane_base;
        const uint32_t tA = tm + kTmA + 64 * t + lane_base;
        uint32_t zero[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) zero[x] = 0u;
        // zero this thread's accumulator row; every MMA accumulates
        tmem_st32(tO, zero);
        tmem_st32(tO + 32, zero);
        tmem_st_wait();
        int n_inter = 0, ns = 0, g_kv = 0, j = 0;  // ns: the CTA's intra step count
        bool ok = true;
        for (int x = sched.first; x < sched.end && ok; x += sched.stride, ++j) {
            const ReadItem it = read_item<GI>(sched.item(x), n_ct, T, L, n_seg, has_init);
            const int qb = j & 1;
            if (lane == 0) mbar_arrive(&bars.genin);
            ok = __all_sync(0xffffffffu, mbar_wait(&bars.qfull[qb], (j >> 1) & 1, abort));
            if (!ok) break;
            uint32_t q2[32];
            {
                const uint8_t *qrow = sm + kSmItem + qb * kItemBytes + t * 16384 + row * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(qrow + ((c ^ (row & 7)) * 16));
                    q2[4 * c + 0] = x.x;
                    q2[4 * c + 1] = x.y;
                    q2[4 * c + 2] = x.z;
                    q2[4 * c + 3] = x.w;
                }
            }
            const int tq0 = it.t0 + kQT * t, tq = tq0 + row;
            float den_inter = 0.f;
            if (it.inter) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bars.u, n_inter & 1, abort));
                if (!ok) break;
                tc_fence_after();
                uint32_t u[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(tU + 32 * half, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const uint32_t w = q2[16 * half + x];
                        den_inter = fmaf(__uint_as_float(w << 16), __uint_as_float(u[2 * x]), den_inter);
                        den_inter = fmaf(__uint_as_float(w & 0xFFFF0000u), __uint_as_float(u[2 * x + 1]),
                                         den_inter);
                    }
                }
                uint32_t x0[32];
                gen_stage_lo<G, 0>(q2, x0);
                ok = gen_loop<G, 0>(q2, bars, tA, n_inter * read_stages(G), abort, x0);
                if (!ok) break;
                ++n_inter;
            }
            float l = 0.f;
            const int nb0 = read_tile_blocks<GI>(it, 0, T), nb1 = read_tile_blocks<GI>(it, 1, T);
            const int n_b = t == 0 ? nb0 : nb1;
            for (int b = 0; b < n_b && ok; ++b) {
                const int n = ns + step_before(b, t, nb0, nb1), x = n % kSBufs;
                const uint32_t tB = tm + kTmBuf + 128 * x + lane_base;
                ok = __all_sync(0xffffffffu, mbar_wait(&bars.sfull[x], (n / kSBufs) & 1, abort));
                if (!ok) break;
                // the block's last scores have landed: its keys are read
                if (qd == 0 && lane == 0 && (t == 1 || b >= nb1))
                    mbar_arrive(&bars.kempty[(g_kv + b) % kv_ring(GI)]);
                tc_fence_after();
                const int kbs = it.seg0 + step_keys(GI) * b;
                // every key of the block precedes every query of the tile
                const bool full = kbs + step_keys(GI) - 1 <= tq0;
                const int lim = tq - kbs;  // otherwise keys kbs + c with c <= lim are visible
                // weights w (packed fp32 pairs), four partial row sums
                uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
                if constexpr (GI == 1) {
                    // w = s^2, 64 keys at a time; each half's weights (bf16 pairs, 32
                    // columns) go over the scores of keys 0-63, already read
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t r[64], p[32];
                        tmem_ld32(tB + 64 * h, r);
                        tmem_ld32(tB + 64 * h + 32, r + 32);
                        tmem_ld_wait();
                        if (full) {
#pragma unroll
                            for (int y = 0; y < 32; ++y) {
                                const uint64_t s2 = f32x2_pack(r[2 * y], r[2 * y + 1]);
                                const uint64_t w2 = f32x2_mul(s2, s2);
                                acc[y & 3] = f32x2_add(acc[y & 3], w2);
                                p[y] = f32x2_to_bf16x2(w2);
                            }
                        } else {
#pragma unroll
                            for (int y = 0; y < 32; ++y) {
                                const int c = 64 * h + 2 * y;
                                const uint32_t m0 = c <= lim ? r[2 * y] : 0u;
                                const uint32_t m1 = c + 1 <= lim ? r[2 * y + 1] : 0u;
                                const uint64_t s2 = f32x2_pack(m0, m1);
                                const uint64_t w2 = f32x2_mul(s2, s2);
                                acc[y & 3] = f32x2_add(acc[y & 3], w2);
                                p[y] = f32x2_to_bf16x2(w2);
                            }
                        }
                        tmem_st32(tB + 32 * h, p);
                    }
                } else {
                    // w = a^2 + b^2, a and b the two factors' scores (columns 0-63 and
                    // 64-127), 32 keys at a time; each half's weights (16 columns) go
                    // over factor-a scores already read
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t ra[32], rb[32], p[16];
                        tmem_ld32(tB + 32 * h, ra);
                        tmem_ld32(tB + 64 + 32 * h, rb);
                        tmem_ld_wait();
#pragma unroll
                        for (int y = 0; y < 16; ++y) {
                            const int c = 32 * h + 2 * y;
                            const bool v0 = full || c <= lim, v1 = full || c + 1 <= lim;
                            const uint64_t a2 = f32x2_pack(v0 ? ra[2 * y] : 0u, v1 ? ra[2 * y + 1] : 0u);
                            const uint64_t b2 = f32x2_pack(v0 ? rb[2 * y] : 0u, v1 ? rb[2 * y + 1] : 0u);
                            const uint64_t w2 = f32x2_fma(b2, b2, f32x2_mul(a2, a2));
                            acc[y & 3] = f32x2_add(acc[y & 3], w2);
                            p[y] = f32x2_to_bf16x2(w2);
                        }
                        tmem_st16(tB + 16 * h, p);
                    }
                }
                {
                    const uint64_t a01 = f32x2_add(acc[0], acc[1]), a23 = f32x2_add(acc[2], acc[3]);
                    const uint64_t a = f32x2_add(a01, a23);
                    l += f32x2_lo(a) + f32x2_hi(a);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    // the block's values have landed (issuer 1, which reads them, learns
                    // it from pfull: a wait of its own would stall behind its MMAs)
                    const int kvb = g_kv + b;
                    ok = mbar_wait(&bars.vfull[kvb % kv_ring(GI)], (kvb / kv_ring(GI)) & 1, abort);
                    if (ok) mbar_arrive(&bars.pfull[x]);  // the step's weights are in place
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
            }
            if (!ok) break;
            ns += nb0 + nb1;
            g_kv += it.n_kv;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars.done, j & 1, abort));
            if (!ok) break;
            tc_fence_after();
            tmem_st_wait();
            uint32_t o[64];
            tmem_ld32(tO, o);
            tmem_ld32(tO + 32, o + 32);
            tmem_ld_wait();
            // zero the accumulator for the next item (ordered before its first MMA by the
            // tcgen05.st wait that precedes every hand-off to the issuers)
            tmem_st32(tO, zero);
            tmem_st32(tO + 32, zero);
            const float den = l + den_inter;
            const float inv = den == 0.f ? 0.f : 1.f / den;
            // the output row replaces this thread's own query row in the item slot (same
            // swizzled layout); warp 11 stores both tiles with TMA once all rows are in
            {
                uint8_t *orow = sm + kSmItem + qb * kItemBytes + t * 16384 + row * 128;
                const uint64_t inv2 = f32x2_pack(__float_as_uint(inv), __float_as_uint(inv));
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 v;
                    v.x = f32x2_to_bf16x2(f32x2_mul(f32x2_pack(o[8 * c + 0], o[8 * c + 1]), inv2));
                    v.y = f32x2_to_bf16x2(f32x2_mul(f32x2_pack(o[8 * c + 2], o[8 * c + 3]), inv2));
                    v.z = f32x2_to_bf16x2(f32x2_mul(f32x2_pack(o[8 * c + 4], o[8 * c + 5]), inv2));
                    v.w = f32x2_to_bf16x2(f32x2_mul(f32x2_pack(o[8 * c + 6], o[8 * c + 7]), inv2));
                    *reinterpret_cast<uint4 *>(orow + ((c ^ (row & 7)) * 16)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.ostaged[qb]);
            }
        }
        tmem_st_wait();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kIssuer0) tmem_dealloc(tm, 512);
    if (tid == 0 && abort_flag) set_timeout_status(status);
}

template <int G, int GI>
bool make_maps(const Plan &p, const void *q, const void *k, const void *v, const void *prefix, void *out,
               CUtensorMap *mq, CUtensorMap *mk, CUtensorMap *mv, CUtensorMap *ms, CUtensorMap *mo) {
    // inner extent d (the boxes stay 64 wide: columns past d read as zeros, and
    // the output store writes only the first d)
    const uint64_t dqkv[3] = {(uint64_t)p.dk, (uint64_t)p.T, (uint64_t)p.BH};
    const uint64_t sqkv[2] = {(uint64_t)p.dk * 2, (uint64_t)p.T * p.dk * 2};
    const uint32_t bqkv[3] = {64, 128, 1};
    const uint64_t ds[3] = {(uint64_t)kD, (uint64_t)bf16_rows(G), (uint64_t)(p.BH * p.n_seg)};
    const uint64_t ss[2] = {(uint64_t)kD * 2, (uint64_t)bf16_rows(G) * kD * 2};
    const uint32_t bs[3] = {64, 32, 1};
    const uint32_t bkv[3] = {64, (uint32_t)step_keys(GI), 1};
    return make_tmap_bf16(mq, q, 3, dqkv, sqkv, bqkv) && make_tmap_bf16(mk, k, 3, dqkv, sqkv, bkv) &&
           make_tmap_bf16(mv, v, 3, dqkv, sqkv, bkv) &&
           make_tmap_bf16(ms, prefix ? prefix : q, 3, ds, ss, bs) && make_tmap_bf16(mo, out, 3, dqkv, sqkv, bqkv);
}

// The dense export of two factors (d = 64).
cudaError_t launch_expand_m2(const float *src, long long stride, float *state_out, float *z_out, long long BH,
                             int d_out, cudaStream_t st) {
    if (d_out != kD) return cudaErrorInvalidValue;
    const long long n = ((long long)kD * kD * kD + (long long)kD * kD) / 4 * BH;
    const unsigned grid = (unsigned)((n + 255) / 256);
    ProfScope ps("tc_state_expand_m2", st);
    tc_state_expand<2, kD><<<grid, 256, 0, st>>>(src, stride, state_out, z_out, BH);
    return cudaSuccess;
}

// Launches `kern` on `st`, as the programmatic dependent of the stream's
// previous kernel when `pdl`: its CTAs may then start (and run their
// prologue) while that kernel finishes, and wait in griddep_wait before they
// read what it wrote.
template <typename... Exp, typename... Act>
cudaError_t launch_k(bool pdl, void (*kern)(Exp...), unsigned grid, unsigned block, size_t smem,
                     cudaStream_t st, Act &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Act &&>(args)...);
}

// The readout of a forward on the G-factor layout with GI-factor weights.
template <int G, int GI>
cudaError_t launch_read(const Plan &p, const void *q, const void *k, const void *v, const void *prefix,
                        void *out, bool has_init, int *status, cudaStream_t st, bool pdl) {
    CUtensorMap mq, mk, mv, ms, mo;
    if (!make_maps<G, GI>(p, q, k, v, prefix, out, &mq, &mk, &mv, &ms, &mo)) return cudaErrorInvalidValue;
    cudaError_t e = smem_opt_in_once<tc_read<G, GI>>(kSmAlloc);
    if (e != cudaSuccess) return e;
    const int n_ct = (p.T + kCtaQ - 1) / kCtaQ;
    const long long n_items = (long long)n_ct * p.BH;
    if (n_items >= 0x7fffffffLL - 4096) return cudaErrorInvalidValue;
    const int grid = (int)(n_items < num_sms() ? n_items : num_sms());
    // score K-steps: one per 16 coordinates of the head (two factors: all four)
    const int qk_ks = GI == 1 ? (p.dk + 15) / 16 : 4;
    ProfScope ps(GI == 1 ? "tc_read" : "tc_read_m2", st);
    return launch_k(pdl, tc_read<G, GI>, (unsigned)grid, kReadThreads, kSmAlloc, st, mq, mk, mv, ms, mo, p.T,
                    p.L, p.n_seg, n_ct, (int)n_items, has_init, qk_ks, status);
}

// The forward with G factors (1: KATA-M1; 2: KATA-Mg with two factors).
template <int G>
cudaError_t launch_tc_forward_g(const Plan &p, const void *q, const void *k, const void *v, void *out,
                                float *state_out, float *z_out, const InitState &init, void *ws,
                                cudaStream_t st, bool reuse_seg) {
    // heads of d < 64 are read as 64 by every tensor map (TMA zero-fills the
    // columns past d; with G = 2 the second factor is then zero) and exported
    // at their own size
    const int d_out = p.dk;
    // no workspace (the quadratic plan): no state is built, scanned or read
    char *w = static_cast<char *>(ws);
    float *seg = w ? reinterpret_cast<float *>(w + p.ws_seg_state) : nullptr;
    float *total = w ? reinterpret_cast<float *>(w + p.ws_total) : nullptr;
    __nv_bfloat16 *prefix = w ? reinterpret_cast<__nv_bfloat16 *>(w + p.ws_extra) : nullptr;
    const bool readout = out != nullptr;
    const bool want_state = state_out != nullptr;
    const bool has_init = init.n > 0;
    // the last segment's increment is needed only for the total; with reuse_seg
    // every segment's increment is in the workspace already
    const int n_build = reuse_seg ? 0 : want_state ? p.n_seg : p.n_seg - 1;
    const int n_valid = reuse_seg ? p.n_seg : n_build;
    // the scan writes the exported state when every dense entry is a pair of
    // the layout (one factor, or heads of d <= 32 on the two-factor layout),
    // so it runs whenever a state is wanted (with one segment and no initial
    // state it only copies)
    const bool dense_from_scan = want_state && (G == 1 || d_out <= kD / 2);
    const bool scan = p.n_seg > 1 || has_init || dense_from_scan;
    const long long BH = p.BH;
    int *status = device_status_ptr();
    if (!status) return cudaErrorUnknown;
    if ((has_init || n_build > 0 || want_state || reuse_seg) && !w) return cudaErrorInvalidValue;
    if (want_state && (d_out < 1 || d_out > kD)) return cudaErrorInvalidValue;
    // Small problems (the builder's and the readout's work items at most one
    // per SM) chain their kernels as programmatic dependents, so that a
    // kernel's launch and prologue overlap its predecessor's tail; larger ones
    // launch plainly (early dependents would take SMs from the previous
    // kernel's last waves).
    const long long read_items = (long long)((p.T + kCtaQ - 1) / kCtaQ) * BH;
    const bool small = (long long)build_items(G) * n_build * BH <= num_sms() && read_items <= num_sms();

    if (n_build > 0) {
        CUtensorMap mkb, mvb, mst;
        const uint64_t dqkv[3] = {(uint64_t)p.dk, (uint64_t)p.T, (uint64_t)BH};
        const uint64_t sqkv[2] = {(uint64_t)p.dk * 2, (uint64_t)p.T * p.dk * 2};
        const uint32_t b64[3] = {64, 64, 1};
        const uint64_t dst[3] = {(uint64_t)kD, (uint64_t)state_rows(G), (uint64_t)(BH * p.n_seg)};
        const uint64_t sst[2] = {(uint64_t)kD * 4, (uint64_t)f32_per_seg(G) * 4};
        const uint32_t bst[3] = {32, 128, 1};
        if (!make_tmap_bf16(&mkb, k, 3, dqkv, sqkv, b64) || !make_tmap_bf16(&mvb, v, 3, dqkv, sqkv, b64) ||
            !make_tmap(&mst, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, seg, 3, dst, sst, bst))
            return cudaErrorInvalidValue;
        cudaError_t e = smem_opt_in_once<tc_build<G>>(kBSmAlloc);
        if (e != cudaSuccess) return e;
        const long long n_items = (long long)build_items(G) * n_build * BH;
        const int grid = (int)(n_items < num_sms() ? n_items : num_sms());
        ProfScope ps(G == 1 ? "tc_build" : "tc_build_m2", st);
        tc_build<G><<<(unsigned)grid, kBuildThreads, kBSmAlloc, st>>>(mkb, mvb, mst, seg, p.T, p.L, p.n_seg,
                                                                       n_build, (int)n_items, status);
    }
    if (scan) {
        ProfScope ps(G == 1 ? "tc_seg_scan" : "tc_seg_scan_m2", st);
        __nv_bfloat16 *pre = readout ? prefix : nullptr;
        float *tot = want_state && !dense_from_scan ? total : nullptr;
        float *s_out = dense_from_scan ? state_out : nullptr;
        float *z_dense = dense_from_scan ? z_out : nullptr;
        if (p.n_seg <= 16) {
            // few segments: one warp per element block (no cross-warp scan)
            const long long grid = ((f32_per_seg(G) / 128) * BH + kScanWarps - 1) / kScanWarps;
            auto kern = p.n_seg <= 4 ? tc_seg_scan_short<G, 4>
                        : p.n_seg <= 8 ? tc_seg_scan_short<G, 8> : tc_seg_scan_short<G, 16>;
            const cudaError_t e = launch_k(small && n_build > 0, kern, (unsigned)grid, 256u, 0, st, seg, pre,
                                           tot, p.n_seg, n_valid, BH, init.s, init.z, init.n, init.s_stride,
                                           init.z_stride, d_out, s_out, z_dense);
            if (e != cudaSuccess) return e;
        } else {
            const long long grid = (f32_per_seg(G) / 128) * BH;
            auto kern = p.n_seg <= 4 * kScanWarps ? tc_seg_scan<G, 4>
                        : p.n_seg <= 8 * kScanWarps ? tc_seg_scan<G, 8>
                                                    : tc_seg_scan<G, 16>;
            const cudaError_t e = launch_k(small && n_build > 0, kern, (unsigned)grid, 256u, 0, st, seg, pre,
                                           tot, p.n_seg, n_valid, init.s, init.z, init.n, init.s_stride,
                                           init.z_stride, d_out, s_out, z_dense);
            if (e != cudaSuccess) return e;
        }
    }
    if (readout) {
        // a single-factor head on the two-factor layout (d <= 32): whole scores
        const bool pdl = small && scan;  // the dependent of this call's scan
        const cudaError_t e = G == 2 && p.g == 1
                                  ? launch_read<G, 1>(p, q, k, v, prefix, out, has_init, status, st, pdl)
                                  : launch_read<G, G>(p, q, k, v, prefix, out, has_init, status, st, pdl);
        if (e != cudaSuccess) return e;
    }
    if (want_state && !dense_from_scan) {
        const float *src = scan ? total : seg;
        const long long stride = scan ? f32_per_seg(G) : f32_per_seg(G) * p.n_seg;
        const cudaError_t e = launch_expand_m2(src, stride, state_out, z_out, BH, d_out, st);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace

// Streaming multiprocessors of the current device (persistent grids).
int num_sms() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lk(mu);
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Workspace of the tensor-core path (bytes; 256-aligned parts), R = 2176 state
// rows for one factor, 1152 for two (tc_layout.cuh):
//   fp32 segment states  BH * n_seg * R * 65 * 4   (state rows, then packed z)
//   fp32 total           BH * R * 65 * 4
//   bf16 prefixes        BH * n_seg * (R + 128) * 64 * 2
void plan_tc_workspace(Plan &p) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const int G = p.tc_g;
    const size_t seg = (size_t)p.BH * p.n_seg * f32_per_seg(G) * 4;
    const size_t tot = (size_t)p.BH * f32_per_seg(G) * 4;
    const size_t pre = (size_t)p.BH * p.n_seg * bf16_per_seg(G) * 2;
    p.ws_seg_state = 0;
    p.ws_total = up(seg);
    p.ws_extra = p.ws_total + up(tot);
    p.ws_aux = 0;
    p.ws_bytes = p.ws_extra + up(pre);
}

cudaError_t launch_tc_forward(const Plan &p, const void *q, const void *k, const void *v, void *out,
                              float *state_out, float *z_out, const InitState &init, void *ws,
                              cudaStream_t st, bool reuse_seg) {
    switch (p.tc_g) {
        case 1: return launch_tc_forward_g<1>(p, q, k, v, out, state_out, z_out, init, ws, st, reuse_seg);
        case 2: return launch_tc_forward_g<2>(p, q, k, v, out, state_out, z_out, init, ws, st, reuse_seg);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tc
}  // namespace kata
