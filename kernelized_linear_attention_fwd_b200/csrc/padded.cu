// The forward of bf16 heads of d = 16 or 32 on the tensor-core kernels.
// Padding q, k and v with zeros to d = 64 changes nothing in the method:
// (q.k)^2 and every sum of products gain only zero terms, the value columns
// past d stay zero, and the leading d x d x d part of the state is the state
// of the unpadded heads.  So the heads are padded into the workspace, run
// through the d = 64 tensor-core forward, and the first d output columns (and
// the leading part of the state) are kept.  The padding costs four times the
// state arithmetic of d = 32, still far below the fp32 CUDA-core path.
#include <cuda_bf16.h>
#include <stdint.h>

#include "kata_internal.cuh"

namespace kata {
namespace {

constexpr int kPadD = 64;
constexpr int kChunk = 8;  // bf16 per 16-byte vector

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// dst [rows][64] = src [rows][d] followed by zeros; one thread per 16 bytes of dst.
__global__ void __launch_bounds__(256)
pad_rows(const uint4 *__restrict__ src, uint4 *__restrict__ dst, long long rows, int d) {
    const long long x = (long long)blockIdx.x * 256 + threadIdx.x;
    if (x >= rows * (kPadD / kChunk)) return;
    const long long r = x / (kPadD / kChunk);
    const int c = (int)(x % (kPadD / kChunk)), nc = d / kChunk;
    dst[x] = c < nc ? src[r * nc + c] : make_uint4(0u, 0u, 0u, 0u);
}

// dst [rows][d] = the first d columns of src [rows][64]; one thread per 16 bytes of dst.
__global__ void __launch_bounds__(256)
unpad_rows(const uint4 *__restrict__ src, uint4 *__restrict__ dst, long long rows, int d) {
    const int nc = d / kChunk;
    const long long x = (long long)blockIdx.x * 256 + threadIdx.x;
    if (x >= rows * nc) return;
    dst[x] = src[(x / nc) * (kPadD / kChunk) + x % nc];
}

unsigned blocks_for(long long threads) { return (unsigned)((threads + 255) / 256); }

}  // namespace

cudaError_t launch_padded_forward(const Plan &p, const void *q, const void *k, const void *v,
                                  void *out, float *state_out, float *z_out, void *ws,
                                  cudaStream_t st) {
    if (p.dtype != KATA_BF16 || p.dk != p.dv || p.dk % kChunk != 0 || p.dk >= kPadD || !ws)
        return cudaErrorInvalidValue;
    Plan p64;
    if (make_plan(p.B, p.H, p.T, kPadD, kPadD, p.C, KATA_BF16, p64) != KATA_OK ||
        p64.path != Path::kTensorCore)
        return cudaErrorInvalidValue;
    const long long rows = p.BH * p.T;
    const size_t slab = up256((size_t)rows * kPadD * 2);
    char *w = static_cast<char *>(ws);
    uint4 *q64 = reinterpret_cast<uint4 *>(w), *k64 = reinterpret_cast<uint4 *>(w + slab),
          *v64 = reinterpret_cast<uint4 *>(w + 2 * slab), *o64 = reinterpret_cast<uint4 *>(w + 3 * slab);
    {
        ProfScope ps("pad_rows", st);
        const unsigned g = blocks_for(rows * (kPadD / kChunk));
        pad_rows<<<g, 256, 0, st>>>(static_cast<const uint4 *>(q), q64, rows, p.dk);
        pad_rows<<<g, 256, 0, st>>>(static_cast<const uint4 *>(k), k64, rows, p.dk);
        pad_rows<<<g, 256, 0, st>>>(static_cast<const uint4 *>(v), v64, rows, p.dv);
    }
    cudaError_t e = tc::launch_tc_forward(p64, q64, k64, v64, o64, state_out, z_out, InitState{},
                                          w + p.ws_aux, st, false, p.dk);
    if (e != cudaSuccess) return e;
    {
        ProfScope ps("unpad_rows", st);
        unpad_rows<<<blocks_for(rows * (p.dv / kChunk)), 256, 0, st>>>(o64, static_cast<uint4 *>(out),
                                                                       rows, p.dv);
    }
    return cudaGetLastError();
}

}  // namespace kata
