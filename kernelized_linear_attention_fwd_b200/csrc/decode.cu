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
#include <cooperative_groups.h>

#include "kata_internal.cuh"

namespace kata {
namespace {

constexpr int kThreads = 512;
constexpr int kUnroll = 4;
constexpr int kMaxParts = 8;  // portable cluster size

// Rows of the d^2-row state that one pass of the block covers.
template <int DV>
constexpr int rows_per_pass() { return kThreads / (DV / 4); }

// Largest split of a head's DK * DK rows into P parts (a power of two, at most
// kMaxParts) that still gives every CTA whole passes.
template <int DK, int DV>
constexpr int max_parts() {
    int p = 1;
    while (2 * p <= kMaxParts && (DK * DK) / (2 * p) >= rows_per_pass<DV>()) p *= 2;
    return p;
}

template <int DK, int DV, int P, typename TIn>
__global__ void __launch_bounds__(kThreads)
decode_step_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                   TIn *__restrict__ out, float *__restrict__ S, float *__restrict__ Z) {
    constexpr int ROWS = DK * DK;
    constexpr int PROWS = ROWS / P;          // rows of this CTA's slice
    constexpr int V4 = DV / 4;               // float4 slots per state row
    constexpr int RPI = kThreads / V4;       // rows covered per pass
    constexpr int UNR = (PROWS / RPI) < kUnroll ? (PROWS / RPI) : kUnroll;
    static_assert(PROWS % (RPI * UNR) == 0, "rows must tile the passes");
    __shared__ float sq[DK], sk[DK], sv[DV];
    __shared__ float red[RPI][DV + 1];
    __shared__ float redz[kThreads / 32];
    __shared__ float part_num[DV], part_den;

    const int tid = threadIdx.x;
    const long long bh = blockIdx.x / P;
    const int part = blockIdx.x % P;         // = the block's rank in its cluster
    const int row_base = part * PROWS;
    if (tid < DK) {
        sq[tid] = load_f32(q, bh * DK + tid);
        sk[tid] = load_f32(k, bh * DK + tid);
    }
    if (tid < DV) sv[tid] = load_f32(v, bh * DV + tid);
    __syncthreads();

    const int c4 = tid % V4, rg = tid / V4;
    const float4 vv = make_float4(sv[4 * c4], sv[4 * c4 + 1], sv[4 * c4 + 2], sv[4 * c4 + 3]);
    float4 *Sh = reinterpret_cast<float4 *>(S + bh * (long long)ROWS * DV);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;

    for (int row0 = row_base + rg; row0 < row_base + PROWS; row0 += RPI * UNR) {
        float4 s[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) s[u] = Sh[(long long)(row0 + u * RPI) * V4 + c4];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int row = row0 + u * RPI, i = row / DK, j = row % DK;
            const float f = sk[i] * sk[j];
            const float w = sq[i] * sq[j];
            s[u].x = fmaf(f, vv.x, s[u].x);
            s[u].y = fmaf(f, vv.y, s[u].y);
            s[u].z = fmaf(f, vv.z, s[u].z);
            s[u].w = fmaf(f, vv.w, s[u].w);
            a0 = fmaf(w, s[u].x, a0);
            a1 = fmaf(w, s[u].y, a1);
            a2 = fmaf(w, s[u].z, a2);
            a3 = fmaf(w, s[u].w, a3);
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) Sh[(long long)(row0 + u * RPI) * V4 + c4] = s[u];
    }

    // normaliser: Z += k k^T, den = q^T Z q (this CTA's slice of the d^2 entries)
    float dz = 0.f;
    float *Zh = Z + bh * (long long)ROWS;
    for (int x = row_base + tid; x < row_base + PROWS; x += kThreads) {
        const int i = x / DK, j = x % DK;
        const float z = Zh[x] + sk[i] * sk[j];
        Zh[x] = z;
        dz = fmaf(sq[i] * sq[j], z, dz);
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

template <int DK, int DV, int P, typename TIn>
cudaError_t launch_parts(int BH, const void *q, const void *k, const void *v, void *out, float *S,
                         float *Z, cudaStream_t st) {
    auto kern = decode_step_kernel<DK, DV, P, TIn>;
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

template <int DK, int DV, typename TIn>
cudaError_t run(int BH, const void *q, const void *k, const void *v, void *out, float *S,
                float *Z, cudaStream_t st) {
    // split heads over clusters while a CTA per head would leave SMs idle
    int parts = 1;
    const int sms = tc::num_sms();
    while (parts < max_parts<DK, DV>() && (long long)BH * parts < sms) parts *= 2;
    ProfScope ps("decode_step", st);
    switch (parts) {
        case 1: return launch_parts<DK, DV, 1, TIn>(BH, q, k, v, out, S, Z, st);
        case 2: return launch_parts<DK, DV, (max_parts<DK, DV>() >= 2 ? 2 : 1), TIn>(BH, q, k, v, out, S, Z, st);
        case 4: return launch_parts<DK, DV, (max_parts<DK, DV>() >= 4 ? 4 : 1), TIn>(BH, q, k, v, out, S, Z, st);
        default: return launch_parts<DK, DV, (max_parts<DK, DV>() >= 8 ? 8 : 1), TIn>(BH, q, k, v, out, S, Z, st);
    }
}

template <typename TIn>
cudaError_t dispatch(int BH, int dk, const void *q, const void *k, const void *v, void *out,
                     float *S, float *Z, cudaStream_t st) {
    switch (dk) {
        case 16: return run<16, 16, TIn>(BH, q, k, v, out, S, Z, st);
        case 32: return run<32, 32, TIn>(BH, q, k, v, out, S, Z, st);
        case 64: return run<64, 64, TIn>(BH, q, k, v, out, S, Z, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode(int B, int H, int dk, int dv, kata_dtype dtype, const void *q,
                          const void *k, const void *v, void *out, float *state, float *z,
                          cudaStream_t st) {
    (void)dv;
    const int BH = B * H;
    if (dtype == KATA_BF16) return dispatch<__nv_bfloat16>(BH, dk, q, k, v, out, state, z, st);
    return dispatch<float>(BH, dk, q, k, v, out, state, z, st);
}

}  // namespace kata
