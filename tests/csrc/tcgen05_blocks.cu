// Test-only kernels that check the sm_100a building blocks of libkata
// (kernelized_linear_attention_fwd_b200/csrc/sm100.cuh) against CPU results:
//   blocks_tma_raw   TMA 2D load with the 128-byte swizzle, raw bytes out
//   blocks_mma_ss    D = A B^T, A K-major [128 x 64], B K-major [N x 64] or
//                    MN-major [64 x N]; both through TMA
//   blocks_mma_ts    D = A B with A written to tensor memory by tcgen05.st
//                    (row m in lane m, K pairs packed per 32-bit column) and
//                    B MN-major [K x 64] through TMA
//   blocks_wait_timeout  the bounded-wait failure path: two warps wait on
//                    mbarriers that nothing completes; the first wait gives up
//                    after the library's cycle budget and raises the CTA's
//                    abort flag, the other sees the flag and leaves too
// Every wait is bounded; a time-out sets *status and the kernel returns.
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../kernelized_linear_attention_fwd_b200/csrc/sm100.cuh"
#include "../../kernelized_linear_attention_fwd_b200/csrc/tmap.cuh"

using namespace kata::sm100;

namespace {

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    const uint32_t s = smem_u32(p);
    return p + ((1024u - (s & 1023u)) & 1023u);
}

__global__ void k_tma_raw(const __grid_constant__ CUtensorMap map, uint16_t *dst, int rows,
                          int *status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    uint8_t *tile = align1024(smem_raw);
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar, rows * 128);
        tma_load_2d(tile, &map, &bar, 0, 0);
    }
    if (!mbar_wait(&bar, 0, &abort_flag)) {
        if (threadIdx.x == 0) atomicExch(status, 3);
        return;
    }
    const uint16_t *s = reinterpret_cast<const uint16_t *>(tile);
    for (int i = threadIdx.x; i < rows * 64; i += blockDim.x) dst[i] = s[i];
}

// 128 threads.  A tile 16 KB at 0, B tile at 16 KB.
__global__ void k_mma_ss(const __grid_constant__ CUtensorMap mapA,
                         const __grid_constant__ CUtensorMap mapB, float *D, int N, int b_mn,
                         uint32_t tmem_cols, int *status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_tma, bar_mma;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    uint8_t *sA = align1024(smem_raw);
    uint8_t *sB = sA + 16384;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar_tma, 1);
        mbar_init(&bar_mma, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tD = tmem_base;
    bool ok = true;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar_tma, 16384 + N * 128);
        tma_load_2d(sA, &mapA, &bar_tma, 0, 0);
        if (b_mn) {
            // [64 K rows][N] in 64-column blocks of 64 rows x 128 B
            for (int nb = 0; nb < N / 64; ++nb) tma_load_2d(sB + nb * 8192, &mapB, &bar_tma, nb * 64, 0);
        } else {
            tma_load_2d(sB, &mapB, &bar_tma, 0, 0);
        }
        ok = mbar_wait(&bar_tma, 0, &abort_flag);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, N, 0, b_mn);
            for (int k = 0; k < 4; ++k) {
                const uint64_t da = desc_sw128(smem_u32(sA) + 32 * k, 16, 1024);
                const uint64_t db = b_mn ? desc_sw128(smem_u32(sB) + 2048 * k, 8192, 1024)
                                         : desc_sw128(smem_u32(sB) + 32 * k, 16, 1024);
                mma_ss(tD, da, db, idesc, k > 0 ? 1u : 0u);
            }
            mma_commit(&bar_mma);
        }
    }
    __syncthreads();
    if (abort_flag) ok = false;
    if (ok && mbar_wait(&bar_mma, 0, &abort_flag)) {
        tc_fence_after();
        const int row = warp * 32 + lane;
        for (int c = 0; c < N; c += 16) {
            uint32_t r[16];
            tmem_ld16(tD + (static_cast<uint32_t>(warp * 32) << 16) + c, r);
            tmem_ld_wait();
            for (int j = 0; j < 16; ++j) D[row * N + c + j] = __uint_as_float(r[j]);
        }
    } else if (threadIdx.x == 0) {
        atomicExch(status, 3);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tD, tmem_cols);
}

// 128 threads.  A [128 x KK] bf16 from global into tensor memory; B [KK x 64]
// MN-major through TMA; D [128 x 64].
__global__ void k_mma_ts(const __nv_bfloat16 *A, int KK, const __grid_constant__ CUtensorMap mapB,
                         float *D, int *status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_tma, bar_mma;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    uint8_t *sB = align1024(smem_raw);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar_tma, 1);
        mbar_init(&bar_mma, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tD = tmem_base, tA = tmem_base + 64;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar_tma, KK * 128);
        tma_load_2d(sB, &mapB, &bar_tma, 0, 0);
    }
    // A row m -> lane m, columns: pair (2c, 2c+1) of K in column c
    const int row = warp * 32 + lane;
    const uint32_t *arow = reinterpret_cast<const uint32_t *>(A + row * KK);
    for (int ks = 0; ks < KK / 16; ++ks) {
        uint32_t r[8];
        for (int c = 0; c < 8; ++c) r[c] = arow[ks * 8 + c];
        tmem_st8(tA + (static_cast<uint32_t>(warp * 32) << 16) + ks * 8, r);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    bool ok = true;
    if (threadIdx.x == 0) {
        tc_fence_after();
        ok = mbar_wait(&bar_tma, 0, &abort_flag);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, 64, 0, 1);
            for (int ks = 0; ks < KK / 16; ++ks) {
                const uint64_t db = desc_sw128(smem_u32(sB) + 2048 * ks, 8192, 1024);
                mma_ts(tD, tA + ks * 8, db, idesc, ks > 0 ? 1u : 0u);
            }
            mma_commit(&bar_mma);
        }
    }
    __syncthreads();
    if (abort_flag) ok = false;
    if (ok && mbar_wait(&bar_mma, 0, &abort_flag)) {
        tc_fence_after();
        for (int c = 0; c < 64; c += 16) {
            uint32_t r[16];
            tmem_ld16(tD + (static_cast<uint32_t>(warp * 32) << 16) + c, r);
            tmem_ld_wait();
            for (int j = 0; j < 16; ++j) D[row * 64 + c + j] = __uint_as_float(r[j]);
        }
    } else if (threadIdx.x == 0) {
        atomicExch(status, 3);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tD, 256);
}

// Lane 0 of warps 0 and 1 each wait on a barrier whose phase never completes
// (nothing arrives).  out[w] = 1 if warp w's wait returned true, out[2 + w] =
// the cycles it waited; *status = 5 (the library's time-out code) when the
// abort flag was raised.
__global__ void k_wait_timeout(long long *out, int *status) {
    __shared__ uint64_t bar[2];
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    const int warp = threadIdx.x / 32;
    if (threadIdx.x % 32 == 0 && warp < 2) {
        const long long t0 = clock64();
        const bool ok = mbar_wait(&bar[warp], 0, &abort_flag);
        out[2 + warp] = clock64() - t0;
        out[warp] = ok ? 1 : 0;
    }
    __syncthreads();
    if (threadIdx.x == 0 && abort_flag) atomicExch(status, 5);
}

bool tmap2d(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_in,
            uint32_t box_out) {
    const uint64_t dims[2] = {inner, outer};
    const uint64_t strides[1] = {inner * 2};
    const uint32_t box[2] = {box_in, box_out};
    return kata::make_tmap_bf16(m, base, 2, dims, strides, box);
}

int finish(int *d_status) {
    if (cudaGetLastError() != cudaSuccess) return 2;
    if (cudaDeviceSynchronize() != cudaSuccess) return 2;
    int s = 0;
    cudaMemcpy(&s, d_status, sizeof(int), cudaMemcpyDeviceToHost);
    return s;
}

}  // namespace

extern "C" {

// src [rows x 64] bf16 (rows <= 256); dst gets the raw shared-memory image.
int blocks_tma_raw(const void *src, void *dst, int rows, int *d_status) {
    CUtensorMap m;
    if (rows < 8 || rows > 256 || !tmap2d(&m, src, 64, rows, 64, rows)) return 1;
    k_tma_raw<<<1, 128, rows * 128 + 1024>>>(m, static_cast<uint16_t *>(dst), rows, d_status);
    return finish(d_status);
}

// A [128 x 64]; B K-major [N x 64] (b_mn = 0) or MN-major [64 x N] (b_mn = 1,
// N a multiple of 64); D [128 x N] fp32.
int blocks_mma_ss(const void *A, const void *B, float *D, int N, int b_mn, int *d_status) {
    CUtensorMap ma, mb;
    if (N < 16 || N > 256 || N % 16) return 1;
    if (!tmap2d(&ma, A, 64, 128, 64, 128)) return 1;
    if (b_mn) {
        if (N % 64) return 1;
        if (!tmap2d(&mb, B, N, 64, 64, 64)) return 1;
    } else if (!tmap2d(&mb, B, 64, N, 64, N)) {
        return 1;
    }
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(N)) cols *= 2;
    const int smem = 16384 + 256 * 128 + 1024;
    cudaFuncSetAttribute(k_mma_ss, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    k_mma_ss<<<1, 128, smem>>>(ma, mb, D, N, b_mn, cols, d_status);
    return finish(d_status);
}

// A [128 x KK] bf16 row-major (KK multiple of 16, <= 256); B [KK x 64]; D [128 x 64].
int blocks_mma_ts(const void *A, const void *B, float *D, int KK, int *d_status) {
    CUtensorMap mb;
    if (KK < 16 || KK > 256 || KK % 16) return 1;
    if (!tmap2d(&mb, B, 64, KK, 64, KK)) return 1;
    const int smem = KK * 128 + 1024;
    cudaFuncSetAttribute(k_mma_ts, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    k_mma_ts<<<1, 128, smem>>>(static_cast<const __nv_bfloat16 *>(A), KK, mb, D, d_status);
    return finish(d_status);
}

// out: 4 int64 (see k_wait_timeout).  Returns the status the kernel set.
int blocks_wait_timeout(long long *out, int *d_status) {
    k_wait_timeout<<<1, 64>>>(out, d_status);
    return finish(d_status);
}

}  // extern "C"
