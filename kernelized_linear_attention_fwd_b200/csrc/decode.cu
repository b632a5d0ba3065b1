// KATA recurrent decode step (arXiv abstract of "Kernelized Linear Attention:
// Breaking the Capacity Wall with Symmetric Cones", "constant-time recurrent
// inference"; gist.science summary, Technical summary 1: a fixed-size state
// replaces the key-value cache).  Per head, in place:
//
//   S[i,j,:] += k_i k_j v,   Z[i,j] += k_i k_j,
//   y = sum_{ij} q_i q_j S[i,j,:] / sum_{ij} q_i q_j Z[i,j]   (0 if the sum is 0)
//
// The step is bound by HBM bandwidth: every byte of the fp32 state is read
// once and written once.  A CTA streams a slice of one head's state with
// 128-bit coalesced loads and stores, several rows in flight per thread, and
// reduces its part of the readout across its threads through shared memory.
// With few heads, each head is split over a thread-block cluster of P CTAs
// (so the whole GPU streams the state) and the P partial readouts are summed
// through distributed shared memory: no global scratch, no atomics.
//
// Two state layouts: dense (d^2 rows i * d + j, the layout the forward
// exports) and packed (the d(d+1)/2 rows i <= j, i outer, weighted c_ij = 2
// off the diagonal and 1 on it at readout), which holds the same information
// in half the bytes, so the step moves half the data.  Pack and unpack
// kernels convert between them.
//
// KATA-Mg with G factors (gist.science summary 2.3, "Variantes"), on the dense
// layout: only rows (i, j) with i and j in one factor of dk / G coordinates
// carry state; the others hold zeros and are neither read nor written, so
// the step streams 1 / G of the bytes.  G = 1 is the single factor.
#include <cooperative_groups.h>

#include "kata_internal.cuh"

namespace kata {
namespace {

constexpr int kThreads = 512;
constexpr int kMaxParts = 8;  // portable cluster size
// State rows a thread has in flight: 4, or 8 when a single-factor head is
// split over a full cluster (few heads, one or two CTAs per SM: the step is
// then bound by the latency of each CTA's passes, not by the bytes in flight
// per SM).
template <int P, int G>
constexpr int unroll_of() { return P == kMaxParts && G == 1 ? 8 : 4; }

// Rows of the d^2-row state that one pass of the block covers.
template <int DV>
constexpr int rows_per_pass() { return kThreads / (DV / 4); }

template <int DK, bool PACKED>
constexpr int state_rows() { return PACKED ? DK * (DK + 1) / 2 : DK * DK; }

// Largest split of a head's rows into P parts (a power of two, at most
// kMaxParts) that still gives every CTA at least one full pass.
template <int DK, int DV, bool PACKED>
constexpr int max_parts() {
    int p = 1;
    while (2 * p <= kMaxParts && state_rows<DK, PACKED>() / (2 * p) >= rows_per_pass<DV>()) p *= 2;
    return p;
}

// (i, j), i <= j, of packed row r: the largest i with start(i) <= r, start(i) =
// i d - i (i - 1) / 2; the square-root estimate is corrected to the exact i.
template <int DK>
__device__ __forceinline__ void packed_ij(int r, int &i, int &j) {
    constexpr float b = 2.f * DK + 1.f;
    int a = (int)((b - sqrtf(b * b - 8.f * (float)r)) * 0.5f);
    a = a < 0 ? 0 : (a > DK - 1 ? DK - 1 : a);
    while (a > 0 && a * DK - a * (a - 1) / 2 > r) --a;
    while (a < DK - 1 && (a + 1) * DK - (a + 1) * a / 2 <= r) ++a;
    i = a;
    j = a + (r - (a * DK - a * (a - 1) / 2));
}

// CTAs per SM the register budget must allow (loads in flight per SM): 4 fit
// the dense single-CTA kernel without spills, 3 the others, 2 the full-cluster
// split with its deeper unroll.
template <int P, bool PACKED, int G = 1>
constexpr int min_ctas_per_sm() {
    return unroll_of<P, G>() == 8 ? 2 : !PACKED && P == 1 && G == 1 ? 4 : 3;
}

template <int DK, int DV, int P, bool PACKED, typename TIn, int G = 1>
__global__ void __launch_bounds__(kThreads, min_ctas_per_sm<P, PACKED, G>())
decode_step_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                   TIn *__restrict__ out, float *__restrict__ S, float *__restrict__ Z) {
    static_assert(G == 1 || !PACKED, "factors only on the dense layout");
    constexpr int FW = DK / G;  // coordinates per factor
    constexpr int ROWS = state_rows<DK, PACKED>();
    constexpr int V4 = DV / 4;               // float4 slots per state row
    constexpr int RPI = kThreads / V4;       // rows covered per pass
    constexpr int UNR = (ROWS / P / RPI) < unroll_of<P, G>() ? (ROWS / P / RPI) : unroll_of<P, G>();
    static_assert(UNR >= 1, "every CTA covers at least one pass");
    __shared__ float sq[DK], sk[DK], sv[DV];
    __shared__ float red[RPI][DV + 1];
    __shared__ float redz[kThreads / 32];
    __shared__ float part_num[DV], part_den;
    // packed layout: (i, j) of each row of this CTA's slice, i | j << 8
    __shared__ uint16_t sij[PACKED ? (ROWS + P - 1) / P + 1 : 1];

    const int tid = threadIdx.x;
    const long long bh = blockIdx.x / P;
    const int part = blockIdx.x % P;         // = the block's rank in its cluster
    const int row_base = part * ROWS / P;    // this CTA's slice [row_base, row_end)
    const int row_end = (part + 1) * ROWS / P;
    if (tid < DK) {
        sq[tid] = load_f32(q, bh * DK + tid);
        sk[tid] = load_f32(k, bh * DK + tid);
    }
    if (tid < DV) sv[tid] = load_f32(v, bh * DV + tid);
    if constexpr (PACKED) {
        for (int r = row_base + tid; r < row_end; r += kThreads) {
            int i, j;
            packed_ij<DK>(r, i, j);
            sij[r - row_base] = (uint16_t)(i | (j << 8));
        }
    }
    __syncthreads();

    const int c4 = tid % V4, rg = tid / V4;
    const float4 vv = make_float4(sv[4 * c4], sv[4 * c4 + 1], sv[4 * c4 + 2], sv[4 * c4 + 3]);
    float4 *Sh = reinterpret_cast<float4 *>(S + bh * (long long)ROWS * DV);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;

    for (int row0 = row_base + rg; row0 < row_end; row0 += RPI * UNR) {
        float4 s[UNR];
        if constexpr (G == 1) {
#pragma unroll
            for (int u = 0; u < UNR; ++u)
                if (row0 + u * RPI < row_end) s[u] = Sh[(long long)(row0 + u * RPI) * V4 + c4];
        } else {
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int row = row0 + u * RPI;
                // rows across factors hold zeros and stay so: not read
                const bool held = row < row_end && (row / DK) / FW == (row % DK) / FW;
                s[u] = held ? Sh[(long long)row * V4 + c4] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int row = row0 + u * RPI;
            if (row >= row_end) continue;
            int i, j;
            if constexpr (PACKED) {
                const int ij = sij[row - row_base];
                i = ij & 255;
                j = ij >> 8;
            } else {
                i = row / DK;
                j = row % DK;
            }
            // a row across factors stays zero: no update, so no readout share
            float f = sk[i] * sk[j];
            if constexpr (G > 1) f = i / FW == j / FW ? f : 0.f;
            const float w = (PACKED && i != j ? 2.f : 1.f) * (sq[i] * sq[j]);
            s[u].x = fmaf(f, vv.x, s[u].x);
            s[u].y = fmaf(f, vv.y, s[u].y);
            s[u].z = fmaf(f, vv.z, s[u].z);
            s[u].w = fmaf(f, vv.w, s[u].w);
            a0 = fmaf(w, s[u].x, a0);
            a1 = fmaf(w, s[u].y, a1);
            a2 = fmaf(w, s[u].z, a2);
            a3 = fmaf(w, s[u].w, a3);
        }
        if constexpr (G == 1) {
#pragma unroll
            for (int u = 0; u < UNR; ++u)
                if (row0 + u * RPI < row_end) Sh[(long long)(row0 + u * RPI) * V4 + c4] = s[u];
        } else {
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int row = row0 + u * RPI;
                if (row < row_end && (row / DK) / FW == (row % DK) / FW)
                    Sh[(long long)row * V4 + c4] = s[u];
            }
        }
    }

    // normaliser: Z += k k^T, den = q^T Z q (this CTA's slice of the d^2 entries)
    float dz = 0.f;
    float *Zh = Z + bh * (long long)ROWS;
    for (int x = row_base + tid; x < row_end; x += kThreads) {
        int i, j;
        if constexpr (PACKED) {
            const int ij = sij[x - row_base];
            i = ij & 255;
            j = ij >> 8;
        } else {
            i = x / DK;
            j = x % DK;
            if (G > 1 && i / FW != j / FW) continue;
        }
        const float z = Zh[x] + sk[i] * sk[j];
        Zh[x] = z;
        dz = fmaf((PACKED && i != j ? 2.f : 1.f) * (sq[i] * sq[j]), z, dz);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dz += __shfl_xor_sync(0xffffffffu, dz, off);
    if ((tid & 31) == 0) redz[tid >> 5] = dz;
    red[rg][4 * c4 + 0] = a0;
    red[rg][4 * c4 + 1] = a1;
    red[rg][4 * c4 + 2] = a2;
    red[rg][4 * c4 + 3] = a3;
    __syncthreads();
    if (tid < DV) {
        float num = 0.f;
        for (int r = 0; r < RPI; ++r) num += red[r][tid];
        float den = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) den += redz[w];
        if constexpr (P == 1) {
            store_out(out, bh * DV + tid, den == 0.f ? 0.f : num / den);
        } else {
            part_num[tid] = num;
            if (tid == 0) part_den = den;
        }
    }
    if constexpr (P > 1) {
        // sum the P partial readouts of the cluster in its first CTA
        cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
        cluster.sync();
        if (part == 0 && tid < DV) {
            float num = 0.f, den = 0.f;
#pragma unroll
            for (int r = 0; r < P; ++r) {
                num += cluster.map_shared_rank(part_num, r)[tid];
                den += *cluster.map_shared_rank(&part_den, r);
            }
            store_out(out, bh * DV + tid, den == 0.f ? 0.f : num / den);
        }
        cluster.sync();  // the other CTAs' shared memory stays valid until the sums are read
    }
}

template <int DK, int DV, int P, bool PACKED, typename TIn, int G>
cudaError_t launch_parts(int BH, const void *q, const void *k, const void *v, void *out, float *S,
                         float *Z, cudaStream_t st) {
    auto kern = decode_step_kernel<DK, DV, P, PACKED, TIn, G>;
    const TIn *qq = static_cast<const TIn *>(q), *kk = static_cast<const TIn *>(k),
              *vv = static_cast<const TIn *>(v);
    TIn *oo = static_cast<TIn *>(out);
    if constexpr (P == 1) {
        kern<<<BH, kThreads, 0, st>>>(qq, kk, vv, oo, S, Z);
        return cudaGetLastError();
    } else {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(BH * P));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = P;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kern, qq, kk, vv, oo, S, Z);
    }
}

template <int DK, int DV, bool PACKED, typename TIn, int G = 1>
cudaError_t run(int BH, const void *q, const void *k, const void *v, void *out, float *S,
                float *Z, cudaStream_t st) {
    // split heads over clusters while a CTA per head would leave SMs idle
    constexpr int MP = max_parts<DK, DV, PACKED>();
    int parts = 1;
    const int sms = tc::num_sms();
    while (parts < MP && (long long)BH * parts < sms) parts *= 2;
    ProfScope ps(PACKED ? "decode_step_packed" : G == 1 ? "decode_step" : "decode_step_mg", st);
    switch (parts) {
        case 1: return launch_parts<DK, DV, 1, PACKED, TIn, G>(BH, q, k, v, out, S, Z, st);
        case 2: return launch_parts<DK, DV, (MP >= 2 ? 2 : 1), PACKED, TIn, G>(BH, q, k, v, out, S, Z, st);
        case 4: return launch_parts<DK, DV, (MP >= 4 ? 4 : 1), PACKED, TIn, G>(BH, q, k, v, out, S, Z, st);
        default: return launch_parts<DK, DV, (MP >= 8 ? 8 : 1), PACKED, TIn, G>(BH, q, k, v, out, S, Z, st);
    }
}

template <bool PACKED, typename TIn, int G = 1>
cudaError_t dispatch(int BH, int dk, const void *q, const void *k, const void *v, void *out,
                     float *S, float *Z, cudaStream_t st) {
    switch (dk) {
        case 16: return run<16, 16, PACKED, TIn, G>(BH, q, k, v, out, S, Z, st);
        case 32: return run<32, 32, PACKED, TIn, G>(BH, q, k, v, out, S, Z, st);
        case 64: return run<64, 64, PACKED, TIn, G>(BH, q, k, v, out, S, Z, st);
        default: return cudaErrorInvalidValue;
    }
}

// Dense [BH, d*d, dv] + [BH, d*d]  ->  packed [BH, R, dv] + [BH, R]: row r = (i, j),
// i <= j, takes dense row i * d + j.  One thread per packed float4 / z entry.
template <int DK, int DV>
__global__ void __launch_bounds__(256)
state_pack(const float *__restrict__ S, const float *__restrict__ Z, float *__restrict__ Sp,
           float *__restrict__ Zp, long long BH) {
    constexpr int R = DK * (DK + 1) / 2, V4 = DV / 4;
    constexpr long long per = (long long)R * V4 + R;
    const long long idx = (long long)blockIdx.x * 256 + threadIdx.x;
    if (idx >= per * BH) return;
    const long long bh = idx / per;
    const long long x = idx % per;
    int i, j;
    if (x < (long long)R * V4) {
        const int r = (int)(x / V4), c = (int)(x % V4);
        packed_ij<DK>(r, i, j);
        reinterpret_cast<float4 *>(Sp)[(bh * R + r) * V4 + c] =
            reinterpret_cast<const float4 *>(S)[(bh * DK * DK + i * DK + j) * V4 + c];
    } else {
        const int r = (int)(x - (long long)R * V4);
        packed_ij<DK>(r, i, j);
        Zp[bh * R + r] = Z[bh * DK * DK + i * DK + j];
    }
}

// Packed -> dense: dense row a * d + b (either order) takes packed row
// (min(a, b), max(a, b)), so the result is symmetric.  One thread per dense
// float4 / z entry.
template <int DK, int DV>
__global__ void __launch_bounds__(256)
state_unpack(const float *__restrict__ Sp, const float *__restrict__ Zp, float *__restrict__ S,
             float *__restrict__ Z, long long BH) {
    constexpr int R = DK * (DK + 1) / 2, V4 = DV / 4;
    constexpr long long per = (long long)DK * DK * V4 + DK * DK;
    const long long idx = (long long)blockIdx.x * 256 + threadIdx.x;
    if (idx >= per * BH) return;
    const long long bh = idx / per;
    const long long x = idx % per;
    const bool z_part = x >= (long long)DK * DK * V4;
    const int dr = z_part ? (int)(x - (long long)DK * DK * V4) : (int)(x / V4);
    const int a = dr / DK, b = dr % DK;
    const int i = a < b ? a : b, j = a < b ? b : a;
    const int r = i * DK - i * (i - 1) / 2 + (j - i);
    if (z_part)
        Z[bh * DK * DK + dr] = Zp[bh * R + r];
    else
        reinterpret_cast<float4 *>(S)[(bh * DK * DK + dr) * V4 + x % V4] =
            reinterpret_cast<const float4 *>(Sp)[(bh * R + r) * V4 + x % V4];
}

template <int DK, int DV>
cudaError_t convert(bool pack, long long BH, const float *src_s, const float *src_z, float *dst_s,
                    float *dst_z, cudaStream_t st) {
    constexpr long long R = DK * (DK + 1) / 2;
    const long long per = pack ? R * (DV / 4) + R : (long long)DK * DK * (DV / 4) + DK * DK;
    const unsigned grid = (unsigned)((per * BH + 255) / 256);
    ProfScope ps(pack ? "state_pack" : "state_unpack", st);
    if (pack)
        state_pack<DK, DV><<<grid, 256, 0, st>>>(src_s, src_z, dst_s, dst_z, BH);
    else
        state_unpack<DK, DV><<<grid, 256, 0, st>>>(src_s, src_z, dst_s, dst_z, BH);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(int B, int H, int dk, int dv, kata_dtype dtype, const void *q,
                          const void *k, const void *v, void *out, float *state, float *z,
                          bool packed, cudaStream_t st) {
    (void)dv;
    const int BH = B * H;
    if (packed)
        return dtype == KATA_BF16
                   ? dispatch<true, __nv_bfloat16>(BH, dk, q, k, v, out, state, z, st)
                   : dispatch<true, float>(BH, dk, q, k, v, out, state, z, st);
    return dtype == KATA_BF16 ? dispatch<false, __nv_bfloat16>(BH, dk, q, k, v, out, state, z, st)
                              : dispatch<false, float>(BH, dk, q, k, v, out, state, z, st);
}

cudaError_t launch_decode_mg(int B, int H, int dk, int g, kata_dtype dtype, const void *q,
                             const void *k, const void *v, void *out, float *state, float *z,
                             cudaStream_t st) {
    const int BH = B * H;
    if (g == 1) return launch_decode(B, H, dk, dk, dtype, q, k, v, out, state, z, false, st);
    if (g != 2) return cudaErrorInvalidValue;
    return dtype == KATA_BF16 ? dispatch<false, __nv_bfloat16, 2>(BH, dk, q, k, v, out, state, z, st)
                              : dispatch<false, float, 2>(BH, dk, q, k, v, out, state, z, st);
}

cudaError_t launch_state_convert(bool pack, int B, int H, int dk, const float *src_s,
                                 const float *src_z, float *dst_s, float *dst_z, cudaStream_t st) {
    const long long BH = (long long)B * H;
    switch (dk) {
        case 16: return convert<16, 16>(pack, BH, src_s, src_z, dst_s, dst_z, st);
        case 32: return convert<32, 32>(pack, BH, src_s, src_z, dst_s, dst_z, st);
        case 64: return convert<64, 64>(pack, BH, src_s, src_z, dst_s, dst_z, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kata
