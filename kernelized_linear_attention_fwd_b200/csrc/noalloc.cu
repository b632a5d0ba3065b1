// kata_chunked_forward_noalloc: the chunked forward with its scratch in a
// statically sized device array instead of a caller-provided workspace, for
// callers that cannot allocate device memory (see include/kata.h).
#include <mutex>

#include "kata_internal.cuh"

namespace kata {
namespace {

constexpr size_t kScratchBytes = KATA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Device scratch shared by every kata_chunked_forward_noalloc call on a device.
// In host code this name is only a host-side handle: its device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
kata_status scratch_on_current_device(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return KATA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return KATA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) return KATA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KATA_OK;
}

}  // namespace
}  // namespace kata

extern "C" kata_status kata_chunked_forward_noalloc(const void *q, const void *k, const void *v,
                                                    void *out, int B, int H, int T, int dk,
                                                    int dv, int C, kata_dtype dtype,
                                                    float *state_out, float *z_out,
                                                    kata_stream_t stream) {
    kata::Plan p;
    const kata_status ps = kata::make_plan(B, H, T, dk, dv, C, dtype, p);
    if (ps != KATA_OK) return ps;
    if (p.ws_bytes > kata::kScratchBytes) return KATA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const kata_status ss = kata::scratch_on_current_device(&scratch);
    if (ss != KATA_OK) return ss;
    return kata_chunked_forward(q, k, v, out, B, H, T, dk, dv, C, dtype, state_out, z_out,
                                scratch, kata::kScratchBytes, stream);
}
