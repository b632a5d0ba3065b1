// KATA causal forward, fp32 CUDA-core path (every head size, fp32 or bf16 input).
//
// Exact chunked-state form (gist.science summary of "Kernelized Linear
// Attention: Breaking the Capacity Wall with Symmetric Cones", Technical
// summary 2.3; arXiv abstract, "exact O(T) chunked-state form"):
//
//   1. seg_state_build  per segment g of L tokens, the state increment
//                       dS_g[r, e] = sum_{s in g} k_si k_sj v_se and
//                       dz_g[r]    = sum_{s in g} k_si k_sj   on packed rows r=(i<=j)
//   2. seg_scan         exclusive prefix over segments (the associative scan of
//                       summary 2.3), in place, plus the total for export
//   3. seg_read         per 64-query tile: phi(q)^T S_prev + (q^T Z_prev q) from
//                       the prefix, plus the causal quadratic term over the
//                       tile's own segment, then the division (summary 2.1)
//   4. state_expand     packed total -> dense [dk*dk, dv] state and [dk, dk] Z
//
// All arithmetic is fp32.  G factors (KATA-Mg, gist.science summary 2.3
// "Variantes"): each factor is its own block of dk / G coordinates, only pairs
// inside a factor carry state, and the intra weight is the sum over factors of
// the squared block inner products.  G = 1 is the single-factor form.
#include "kata_internal.cuh"

namespace kata {
namespace {

constexpr int kTok = 64;    // token tile
constexpr int kRowB = 32;   // state rows per inter step in seg_read

// ---------------------------------------------------------------------------
// 1. Per-segment state increments.
// grid.x = row-block + nrb * (segment + n_build * bh); block 256 = 32 rows x 8 e-groups
// ---------------------------------------------------------------------------
template <int DK, int DV, int G, typename TIn>
__global__ void __launch_bounds__(256)
seg_state_build(const TIn *__restrict__ k, const TIn *__restrict__ v, float *__restrict__ seg_state,
                int T, int L, int n_seg, int n_build) {
    constexpr int R = packed_rows_g(DK, G);
    constexpr long long E = (long long)R * (DV + 1);
    constexpr int EG = DV / 8;
    constexpr int NRB = (R + 31) / 32;
    __shared__ float sk[kTok][DK + 1];
    __shared__ float sv[kTok][DV];

    const int tid = threadIdx.x;
    const int lr = tid & 31, eg = tid >> 5;
    long long blk = blockIdx.x;
    const int rb = (int)(blk % NRB);
    blk /= NRB;
    const int g = (int)(blk % n_build);
    const long long bh = blk / n_build;
    const int r = rb * 32 + lr;
    const bool live = r < R;
    int i = 0, j = 0;
    if (live) packed_row_ij_g(DK, G, r, i, j);

    float acc[EG];
#pragma unroll
    for (int u = 0; u < EG; ++u) acc[u] = 0.f;
    float accz = 0.f;

    const int s0 = g * L, s1 = min(T, s0 + L);
    for (int t0 = s0; t0 < s1; t0 += kTok) {
        __syncthreads();
        for (int x = tid; x < kTok * DK; x += 256) {
            const int s = x / DK, c = x % DK, ts = t0 + s;
            sk[s][c] = ts < s1 ? load_f32(k, (bh * T + ts) * DK + c) : 0.f;
        }
        for (int x = tid; x < kTok * DV; x += 256) {
            const int s = x / DV, c = x % DV, ts = t0 + s;
            sv[s][c] = ts < s1 ? load_f32(v, (bh * T + ts) * DV + c) : 0.f;
        }
        __syncthreads();
        const int n = min(kTok, s1 - t0);
        for (int s = 0; s < n; ++s) {
            const float f = sk[s][i] * sk[s][j];
            accz += f;
#pragma unroll
            for (int u = 0; u < EG; ++u) acc[u] = fmaf(f, sv[s][eg * EG + u], acc[u]);
        }
    }
    if (live) {
        float *dst = seg_state + (bh * n_seg + g) * E;
#pragma unroll
        for (int u = 0; u < EG; ++u) dst[(long long)r * DV + eg * EG + u] = acc[u];
        if (eg == 0) dst[(long long)R * DV + r] = accz;
    }
}

// ---------------------------------------------------------------------------
// 2. Exclusive prefix over segments, per element, log-depth per 32 segments.
//
// A block owns 32 consecutive elements of every segment of one head.  Tiles
// of 32 segments x 32 elements are staged through shared memory (coalesced
// loads and stores along elements), each warp then scans element columns
// across 32 segments with a Kogge-Stone shuffle scan (5 steps) and carries
// the column total into the next tile.  An initial state (the sum of n_in
// dense states) seeds the carries, so every prefix, segment 0's included,
// and the total contain it.
// grid.x = element-tile + n_et * bh; block (32, 8)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
seg_scan(float *__restrict__ seg_state, float *__restrict__ total, long long E, int n_seg,
         int n_valid, int dk, int dv, int g, const float *__restrict__ init_s,
         const float *__restrict__ init_z, int n_in, long long s_stride, long long z_stride) {
    __shared__ float tile[32][33];
    const int lane = threadIdx.x, w = threadIdx.y;
    const long long n_et = (E + 31) / 32;
    const long long et = blockIdx.x % n_et;
    const long long bh = blockIdx.x / n_et;
    const long long e_base = et * 32;
    float *base = seg_state + bh * (long long)n_seg * E;
    float carry[4] = {0.f, 0.f, 0.f, 0.f};
    const long long R = E / (dv + 1);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {  // packed element e = row (i, j): dense row i * dk + j
        const long long e = e_base + threadIdx.y + 8 * cc;
        if (e >= E) continue;
        const bool z_part = e >= R * dv;
        int i, j;
        packed_row_ij_g(dk, g, (int)(z_part ? e - R * dv : e / dv), i, j);
        for (int n = 0; n < n_in; ++n)
            carry[cc] += z_part ? init_z[n * z_stride + (bh * dk + i) * dk + j]
                                : init_s[n * s_stride + ((bh * dk + i) * dk + j) * dv + e % dv];
    }

    for (int g0 = 0; g0 < n_seg; g0 += 32) {
        // load 32 segments x 32 elements
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            const int gs = w + 8 * rr, g = g0 + gs;
            const long long e = e_base + lane;
            tile[gs][lane] = (g < n_valid && e < E) ? base[(long long)g * E + e] : 0.f;
        }
        __syncthreads();
        // scan 4 element columns per warp across the 32 segments (lane = segment)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const int c = w + 8 * cc;
            const float x = tile[lane][c];
            float inc = x;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, inc, off);
                if (lane >= off) inc += y;
            }
            tile[lane][c] = carry[cc] + (inc - x);
            carry[cc] += __shfl_sync(0xffffffffu, inc, 31);
        }
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            const int gs = w + 8 * rr, g = g0 + gs;
            const long long e = e_base + lane;
            if (g < n_seg && e < E) base[(long long)g * E + e] = tile[gs][lane];
        }
        __syncthreads();
    }
    if (total != nullptr && lane == 0) {
        // carries are warp-uniform; lane 0 of warp w owns columns w + 8 cc
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const long long e = e_base + w + 8 * cc;
            if (e < E) total[bh * E + e] = carry[cc];
        }
    }
}

// ---------------------------------------------------------------------------
// 3. Readout per 64-query tile.
// grid.x = query-tile + n_qt * bh; block 256: thread = 4 queries x DV/16 values
// ---------------------------------------------------------------------------
template <int DK, int DV>
struct ReadSmem {
    static constexpr int kQ = kTok * (DK + 1);
    static constexpr int kK = kTok * (DK + 1);
    static constexpr int kV = kTok * DV;
    static constexpr int kP = kTok * (kTok + 1);
    static constexpr int kS = kRowB * (DV + 1);
    static constexpr int kFloats = kQ + kK + kV + kP + kS;
    static constexpr size_t kBytes = kFloats * sizeof(float) + packed_rows(DK) * sizeof(unsigned short);
};

template <int DK, int DV, int G, typename TIn>
__global__ void __launch_bounds__(256)
seg_read(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
         TIn *__restrict__ out, const float *__restrict__ seg_state, int T, int L, int n_seg,
         bool has_init) {
    constexpr int R = packed_rows_g(DK, G);
    constexpr long long E = (long long)R * (DV + 1);
    constexpr int TE = DV / 16;
    using SM = ReadSmem<DK, DV>;
    extern __shared__ float smem[];
    float *sq = smem;
    float *sk = sq + SM::kQ;
    float *sv = sk + SM::kK;
    float *sp = sv + SM::kV;
    float *ss = sp + SM::kP;
    unsigned short *sij = reinterpret_cast<unsigned short *>(ss + SM::kS);

    const int tid = threadIdx.x;
    const int tq = tid >> 4, te = tid & 15;
    // One segment (the quadratic form): the latest query tiles, whose work is
    // largest, are scheduled first, across all heads.
    const int n_qt = (T + kTok - 1) / kTok;
    long long bh;
    int t0;
    if (n_seg == 1) {
        const long long BH = gridDim.x / n_qt;
        bh = blockIdx.x % BH;
        t0 = (n_qt - 1 - (int)(blockIdx.x / BH)) * kTok;
    } else {
        bh = blockIdx.x / n_qt;
        t0 = (int)(blockIdx.x % n_qt) * kTok;
    }
    const int g = t0 / L;
    const int seg0 = g * L;

    for (int x = tid; x < kTok * DK; x += 256) {
        const int s = x / DK, c = x % DK, t = t0 + s;
        sq[s * (DK + 1) + c] = t < T ? load_f32(q, (bh * T + t) * DK + c) : 0.f;
    }
    for (int r = tid; r < R; r += 256) {
        int i, j;
        packed_row_ij_g(DK, G, r, i, j);
        sij[r] = (unsigned short)(i | (j << 8));
    }
    float num[4][TE], den[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        den[a] = 0.f;
#pragma unroll
        for (int u = 0; u < TE; ++u) num[a][u] = 0.f;
    }
    __syncthreads();

    // inter-segment term: phi(q)^T S_prev and q^T Z_prev q, from the packed prefix
    // (segment 0 has one when the forward starts from a given state)
    if (g > 0 || has_init) {
        const float *Sg = seg_state + (bh * n_seg + g) * E;
        for (int r0 = 0; r0 < R; r0 += kRowB) {
            for (int x = tid; x < kRowB * DV; x += 256) {
                const int rr = x / DV, e = x % DV;
                ss[rr * (DV + 1) + e] = (r0 + rr < R) ? Sg[(long long)(r0 + rr) * DV + e] : 0.f;
            }
            for (int x = tid; x < kRowB; x += 256)
                ss[x * (DV + 1) + DV] = (r0 + x < R) ? Sg[(long long)R * DV + r0 + x] : 0.f;
            for (int x = tid; x < kTok * kRowB; x += 256) {
                const int qq = x / kRowB, rr = x % kRowB, r = r0 + rr;
                float w = 0.f;
                if (r < R) {
                    const int ij = sij[r], i = ij & 255, j = ij >> 8;
                    w = sq[qq * (DK + 1) + i] * sq[qq * (DK + 1) + j];
                    if (i != j) w *= 2.f;
                }
                sp[qq * (kTok + 1) + rr] = w;
            }
            __syncthreads();
#pragma unroll 4
            for (int rr = 0; rr < kRowB; ++rr) {
                float sr[TE];
#pragma unroll
                for (int u = 0; u < TE; ++u) sr[u] = ss[rr * (DV + 1) + te * TE + u];
                const float zr = ss[rr * (DV + 1) + DV];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float w = sp[(tq * 4 + a) * (kTok + 1) + rr];
                    den[a] = fmaf(w, zr, den[a]);
#pragma unroll
                    for (int u = 0; u < TE; ++u) num[a][u] = fmaf(w, sr[u], num[a][u]);
                }
            }
            __syncthreads();
        }
    }

    // intra-segment term: keys from the segment start up to the tile end, causal
    const int kend = min(T, t0 + kTok);
    for (int k0 = seg0; k0 < kend; k0 += kTok) {
        for (int x = tid; x < kTok * DK; x += 256) {
            const int s = x / DK, c = x % DK, ts = k0 + s;
            sk[s * (DK + 1) + c] = ts < kend ? load_f32(k, (bh * T + ts) * DK + c) : 0.f;
        }
        for (int x = tid; x < kTok * DV; x += 256) {
            const int s = x / DV, c = x % DV, ts = k0 + s;
            sv[s * DV + c] = ts < kend ? load_f32(v, (bh * T + ts) * DV + c) : 0.f;
        }
        __syncthreads();
        for (int x = tid; x < kTok * kTok; x += 256) {
            const int qq = x / kTok, s = x % kTok;
            float w = 0.f;
#pragma unroll
            for (int f = 0; f < G; ++f) {  // one squared inner product per factor
                float dot = 0.f;
#pragma unroll
                for (int c = f * (DK / G); c < (f + 1) * (DK / G); ++c)
                    dot = fmaf(sq[qq * (DK + 1) + c], sk[s * (DK + 1) + c], dot);
                w = fmaf(dot, dot, w);
            }
            if (k0 + s > t0 + qq || k0 + s >= kend) w = 0.f;
            sp[qq * (kTok + 1) + s] = w;
        }
        __syncthreads();
#pragma unroll 4
        for (int s = 0; s < kTok; ++s) {
            float vr[TE];
#pragma unroll
            for (int u = 0; u < TE; ++u) vr[u] = sv[s * DV + te * TE + u];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float w = sp[(tq * 4 + a) * (kTok + 1) + s];
                den[a] += w;
#pragma unroll
                for (int u = 0; u < TE; ++u) num[a][u] = fmaf(w, vr[u], num[a][u]);
            }
        }
        __syncthreads();
    }

#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int t = t0 + tq * 4 + a;
        if (t >= T) continue;
#pragma unroll
        for (int u = 0; u < TE; ++u) {
            const float y = den[a] == 0.f ? 0.f : num[a][u] / den[a];
            store_out(out, (bh * T + t) * DV + te * TE + u, y);
        }
    }
}

// ---------------------------------------------------------------------------
// 4. Packed total -> dense state [dk*dk, dv] and Z [dk, dk].
// ---------------------------------------------------------------------------
template <int DK, int DV, int G>
__global__ void __launch_bounds__(256)
state_expand(const float *__restrict__ total, long long stride_bh, float *__restrict__ state_out,
             float *__restrict__ z_out, long long BH) {
    constexpr int R = packed_rows_g(DK, G), P = DK / G;
    const long long per = (long long)DK * DK * DV + DK * DK;
    const long long idx = (long long)blockIdx.x * 256 + threadIdx.x;
    if (idx >= per * BH) return;
    const long long bh = idx / per;
    long long x = idx % per;
    const float *src = total + bh * stride_bh;
    if (x < (long long)DK * DK * DV) {
        const int row = (int)(x / DV), e = (int)(x % DV);
        int i = row / DK, j = row % DK;
        if (i > j) { const int t = i; i = j; j = t; }
        // pairs across factors carry no state
        state_out[bh * DK * DK * DV + x] =
            i / P == j / P ? src[(long long)packed_row_index_g(DK, G, i, j) * DV + e] : 0.f;
    } else {
        x -= (long long)DK * DK * DV;
        int i = (int)(x / DK), j = (int)(x % DK);
        if (i > j) { const int t = i; i = j; j = t; }
        z_out[bh * DK * DK + x] =
            i / P == j / P ? src[(long long)R * DV + packed_row_index_g(DK, G, i, j)] : 0.f;
    }
}

template <int DK, int DV, int G, typename TIn>
cudaError_t run(const Plan &p, const TIn *q, const TIn *k, const TIn *v, TIn *out,
                float *state_out, float *z_out, const InitState &init, void *ws, cudaStream_t st) {
    constexpr int R = packed_rows_g(DK, G);
    constexpr long long E = (long long)R * (DV + 1);
    const long long BH = p.BH;
    // no workspace (the quadratic plan): no state is built, scanned or read
    char *w = static_cast<char *>(ws);
    float *seg = w ? reinterpret_cast<float *>(w + p.ws_seg_state) : nullptr;
    float *total = w ? reinterpret_cast<float *>(w + p.ws_total) : nullptr;
    const bool readout = out != nullptr;
    const bool want_state = state_out != nullptr;
    const bool has_init = init.n > 0;
    // the last segment's increment is needed only for the total
    const int n_build = want_state ? p.n_seg : p.n_seg - 1;
    const bool scan = p.n_seg > 1 || has_init;
    if ((has_init || n_build > 0 || want_state) && !w) return cudaErrorInvalidValue;

    if (n_build > 0) {
        const long long grid = (long long)((R + 31) / 32) * n_build * BH;
        ProfScope ps("simt_seg_state_build", st);
        seg_state_build<DK, DV, G, TIn><<<(unsigned)grid, 256, 0, st>>>(k, v, seg, p.T, p.L,
                                                                        p.n_seg, n_build);
    }
    if (scan) {
        const long long grid = ((E + 31) / 32) * BH;
        ProfScope ps("seg_scan", st);
        seg_scan<<<(unsigned)grid, dim3(32, 8), 0, st>>>(seg, want_state ? total : nullptr, E,
                                                         p.n_seg, n_build, DK, DV, G, init.s, init.z,
                                                         init.n, init.s_stride, init.z_stride);
    }
    if (readout) {
        using SM = ReadSmem<DK, DV>;
        cudaError_t e = smem_opt_in_once<seg_read<DK, DV, G, TIn>>((int)SM::kBytes);
        if (e != cudaSuccess) return e;
        const long long grid = (long long)((p.T + kTok - 1) / kTok) * BH;
        ProfScope ps("simt_seg_read", st);
        seg_read<DK, DV, G, TIn><<<(unsigned)grid, 256, SM::kBytes, st>>>(q, k, v, out, seg, p.T,
                                                                           p.L, p.n_seg, has_init);
    }
    if (want_state) {
        const float *src = scan ? total : seg;
        const long long stride = scan ? E : E * p.n_seg;
        const long long n = ((long long)DK * DK * DV + DK * DK) * BH;
        ProfScope ps("state_expand", st);
        state_expand<DK, DV, G><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(src, stride, state_out,
                                                                             z_out, BH);
    }
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t dispatch(const Plan &p, const void *q, const void *k, const void *v, void *out,
                     float *so, float *zo, const InitState &init, void *ws, cudaStream_t st) {
    const TIn *Q = static_cast<const TIn *>(q);
    const TIn *K = static_cast<const TIn *>(k);
    const TIn *V = static_cast<const TIn *>(v);
    TIn *O = static_cast<TIn *>(out);
    const int key = p.dk * 4 + p.g;
    switch (key) {
        case 16 * 4 + 1: return run<16, 16, 1, TIn>(p, Q, K, V, O, so, zo, init, ws, st);
        case 32 * 4 + 1: return run<32, 32, 1, TIn>(p, Q, K, V, O, so, zo, init, ws, st);
        case 64 * 4 + 1: return run<64, 64, 1, TIn>(p, Q, K, V, O, so, zo, init, ws, st);
        case 16 * 4 + 2: return run<16, 16, 2, TIn>(p, Q, K, V, O, so, zo, init, ws, st);
        case 32 * 4 + 2: return run<32, 32, 2, TIn>(p, Q, K, V, O, so, zo, init, ws, st);
        case 64 * 4 + 2: return run<64, 64, 2, TIn>(p, Q, K, V, O, so, zo, init, ws, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_simt_forward(const Plan &p, const void *q, const void *k, const void *v,
                                void *out, float *state_out, float *z_out, const InitState &init,
                                void *ws, cudaStream_t st) {
    if (p.dtype == KATA_BF16)
        return dispatch<__nv_bfloat16>(p, q, k, v, out, state_out, z_out, init, ws, st);
    return dispatch<float>(p, q, k, v, out, state_out, z_out, init, ws, st);
}

}  // namespace kata
