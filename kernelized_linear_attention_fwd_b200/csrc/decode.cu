// KATA recurrent decode step (arXiv abstract of "Kernelized Linear Attention:
// Breaking the Capacity Wall with Symmetric Cones", "constant-time recurrent
// inference"; gist.science summary, Technical summary 1: a fixed-size state
// replaces the key-value cache).  Per head, in place:
//
//   S[i,j,:] += k_i k_j v,   Z[i,j] += k_i k_j,
//   y = sum_{ij} q_i q_j S[i,j,:] / sum_{ij} q_i q_j Z[i,j]   (0 if the sum is 0)
//
// The step is bound by HBM bandwidth: every byte of the fp32 state is read
// once and written once.  One CTA streams one head's state with 128-bit
// coalesced loads and stores, several rows in flight per thread, and reduces
// the readout across its threads through shared memory (no atomics).
#include "kata_internal.cuh"

namespace kata {
namespace {

constexpr int kThreads = 512;
constexpr int kUnroll = 4;

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(kThreads)
decode_step_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                   TIn *__restrict__ out, float *__restrict__ S, float *__restrict__ Z) {
    constexpr int ROWS = DK * DK;
    constexpr int V4 = DV / 4;              // float4 slots per state row
    constexpr int RPI = kThreads / V4;      // rows covered per pass
    constexpr int UNR = (ROWS / RPI) < kUnroll ? (ROWS / RPI) : kUnroll;
    static_assert(ROWS % (RPI * UNR) == 0, "rows must tile the passes");
    __shared__ float sq[DK], sk[DK], sv[DV];
    __shared__ float red[RPI][DV + 1];
    __shared__ float redz[kThreads / 32];

    const int tid = threadIdx.x;
    const long long bh = blockIdx.x;
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

    for (int row0 = rg; row0 < ROWS; row0 += RPI * UNR) {
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

    // normaliser: Z += k k^T, den = q^T Z q
    float dz = 0.f;
    float *Zh = Z + bh * (long long)ROWS;
    for (int x = tid; x < ROWS; x += kThreads) {
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
        store_out(out, bh * DV + tid, den == 0.f ? 0.f : num / den);
    }
}

template <int DK, int DV, typename TIn>
cudaError_t run(int BH, const void *q, const void *k, const void *v, void *out, float *S,
                float *Z, cudaStream_t st) {
    ProfScope ps("decode_step", st);
    decode_step_kernel<DK, DV, TIn><<<BH, kThreads, 0, st>>>(
        static_cast<const TIn *>(q), static_cast<const TIn *>(k), static_cast<const TIn *>(v),
        static_cast<TIn *>(out), S, Z);
    return cudaGetLastError();
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
