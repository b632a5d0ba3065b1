// kata_chunked_forward_host: the chunked forward on q, k, v and out held in
// pinned host memory.  The heads are independent, so they are processed in
// groups, and three streams overlap the transfers with the compute: while
// group g runs on the caller's stream, group g+1's inputs cross PCIe to the
// device on a copy stream and group g-1's outputs cross back on another.
// Each group runs through kata_chunked_forward itself (same kernels, same
// checks).  Two device slots, each holding one group's q, k, v and out,
// alternate between groups; events order the reuse of a slot after the copy
// that last read it.  The two copy streams and the events come from a
// per-device pool: a call takes a set (creating one the first time), enqueues
// its work and returns the set, so repeated calls create nothing, and calls
// from several host threads each hold a set of their own while they enqueue.
// Reusing a set is safe as soon as the call that held it has returned: a
// stream wait captures an event's state when the wait is enqueued, so
// recording the event again later changes no wait already queued.
#include <stdint.h>

#include <mutex>
#include <vector>

#include "kata_internal.cuh"

namespace kata {
namespace {

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

struct HostPlan {
    long long BH;
    int G;                 // heads per group
    int n_groups;
    size_t q_head, v_head;  // bytes of one head's q (= k) and v (= out) rows
    size_t slot_bytes;     // q, k, v, out of G heads
    size_t ws_offset, ws_bytes;
    size_t total;
};

constexpr int kSlots = 2;

// Copy streams and events of one call.
struct PipeSet {
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t e_start = nullptr, e_in[kSlots] = {}, e_comp[kSlots] = {}, e_out[kSlots] = {};
};

constexpr int kMaxDevices = 64;
std::mutex g_pool_mu;
std::vector<PipeSet *> g_pool[kMaxDevices];

PipeSet *create_set() {
    PipeSet *ps = new PipeSet;
    bool ok = cudaStreamCreateWithFlags(&ps->s_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&ps->s_out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&ps->e_start, cudaEventDisableTiming) == cudaSuccess;
    for (int s = 0; s < kSlots && ok; ++s)
        ok = cudaEventCreateWithFlags(&ps->e_in[s], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&ps->e_comp[s], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&ps->e_out[s], cudaEventDisableTiming) == cudaSuccess;
    if (ok) return ps;
    if (ps->s_in) cudaStreamDestroy(ps->s_in);
    if (ps->s_out) cudaStreamDestroy(ps->s_out);
    if (ps->e_start) cudaEventDestroy(ps->e_start);
    for (int s = 0; s < kSlots; ++s) {
        if (ps->e_in[s]) cudaEventDestroy(ps->e_in[s]);
        if (ps->e_comp[s]) cudaEventDestroy(ps->e_comp[s]);
        if (ps->e_out[s]) cudaEventDestroy(ps->e_out[s]);
    }
    delete ps;
    return nullptr;
}

// A set of the current device, from the pool or new; nullptr on failure.
PipeSet *acquire_set(int dev) {
    {
        std::lock_guard<std::mutex> lk(g_pool_mu);
        if (!g_pool[dev].empty()) {
            PipeSet *ps = g_pool[dev].back();
            g_pool[dev].pop_back();
            return ps;
        }
    }
    return create_set();
}

void release_set(int dev, PipeSet *ps) {
    std::lock_guard<std::mutex> lk(g_pool_mu);
    g_pool[dev].push_back(ps);
}

kata_status host_plan(int B, int H, int T, int dk, int dv, int C, kata_dtype dtype,
                      int heads_per_group, HostPlan &hp) {
    Plan p;
    const kata_status ps = make_plan(B, H, T, dk, dv, C, dtype, p);
    if (ps != KATA_OK) return ps;
    hp.BH = p.BH;
    long long G = heads_per_group > 0 ? heads_per_group : (p.BH + 7) / 8;  // about 8 groups
    if (G > p.BH) G = p.BH;
    if (G > 0x7fffffffLL) return KATA_ERR_UNSUPPORTED;
    hp.G = (int)G;
    hp.n_groups = (int)((p.BH + G - 1) / G);
    const size_t es = dtype == KATA_BF16 ? 2 : 4;
    hp.q_head = (size_t)T * dk * es;
    hp.v_head = (size_t)T * dv * es;
    hp.slot_bytes = 2 * up256(G * hp.q_head) + 2 * up256(G * hp.v_head);
    Plan pg;
    if (make_plan(1, hp.G, T, dk, dv, C, dtype, pg) != KATA_OK) return KATA_ERR_UNSUPPORTED;
    hp.ws_offset = kSlots * hp.slot_bytes;
    hp.ws_bytes = pg.ws_bytes;
    hp.total = hp.ws_offset + up256(hp.ws_bytes);
    return KATA_OK;
}

}  // namespace
}  // namespace kata

extern "C" {

size_t kata_chunked_forward_host_buffer_bytes(int B, int H, int T, int dk, int dv, int C,
                                              kata_dtype dtype, int heads_per_group) {
    kata::HostPlan hp;
    if (kata::host_plan(B, H, T, dk, dv, C, dtype, heads_per_group, hp) != KATA_OK) return 0;
    return hp.total;
}

kata_status kata_chunked_forward_host(const void *q, const void *k, const void *v, void *out,
                                      int B, int H, int T, int dk, int dv, int C,
                                      kata_dtype dtype, float *state_out, float *z_out,
                                      void *device_buffer, size_t device_buffer_bytes,
                                      int heads_per_group, kata_stream_t stream) {
    kata::HostPlan hp;
    const kata_status ps = kata::host_plan(B, H, T, dk, dv, C, dtype, heads_per_group, hp);
    if (ps != KATA_OK) return ps;
    if (!q || !k || !v || !out) return KATA_ERR_INVALID_ARG;
    if ((state_out == nullptr) != (z_out == nullptr)) return KATA_ERR_INVALID_ARG;
    if (!device_buffer || device_buffer_bytes < hp.total ||
        (reinterpret_cast<uintptr_t>(device_buffer) & 255u) != 0)
        return KATA_ERR_WORKSPACE;

    if (!kata::device_ptrs_ok({device_buffer, state_out, z_out})) return KATA_ERR_INVALID_ARG;
    int device = -1;
    if (cudaGetDevice(&device) != cudaSuccess) return KATA_ERR_CUDA;
    if (device < 0 || device >= kata::kMaxDevices) return KATA_ERR_UNSUPPORTED;
    kata::PipeSet *set = kata::acquire_set(device);
    if (!set) return KATA_ERR_CUDA;
    cudaStream_t user = reinterpret_cast<cudaStream_t>(stream);
    cudaStream_t s_in = set->s_in, s_out = set->s_out;
    cudaEvent_t e_start = set->e_start, *e_in = set->e_in, *e_comp = set->e_comp,
                *e_out = set->e_out;
    // the copies start after the work already queued on the caller's stream; a
    // slot's first use waits on nothing of this call's, so its events are
    // first recorded right after that start point
    bool ok = cudaEventRecord(e_start, user) == cudaSuccess &&
              cudaStreamWaitEvent(s_in, e_start, 0) == cudaSuccess &&
              cudaStreamWaitEvent(s_out, e_start, 0) == cudaSuccess;
    for (int s = 0; s < kata::kSlots && ok; ++s)
        ok = cudaEventRecord(e_comp[s], user) == cudaSuccess &&
             cudaEventRecord(e_out[s], s_out) == cudaSuccess &&
             cudaEventRecord(e_in[s], s_in) == cudaSuccess;

    kata_status status = ok ? KATA_OK : KATA_ERR_CUDA;
    const char *qh = static_cast<const char *>(q), *kh = static_cast<const char *>(k),
               *vh = static_cast<const char *>(v);
    char *oh = static_cast<char *>(out);
    char *dev = static_cast<char *>(device_buffer);
    const size_t es_q = hp.q_head, es_v = hp.v_head;
    for (int g = 0; g < hp.n_groups && status == KATA_OK; ++g) {
        const int s = g % kata::kSlots;
        const long long h0 = (long long)g * hp.G;
        const int gh = (int)(hp.BH - h0 < hp.G ? hp.BH - h0 : hp.G);
        char *slot = dev + s * hp.slot_bytes;
        char *dq = slot, *dk_ = dq + kata::up256(hp.G * es_q), *dv_ = dk_ + kata::up256(hp.G * es_q),
             *dout = dv_ + kata::up256(hp.G * es_v);
        // inputs: once the compute of the group that last used this slot is done
        ok = cudaStreamWaitEvent(s_in, e_comp[s], 0) == cudaSuccess &&
             cudaMemcpyAsync(dq, qh + h0 * es_q, gh * es_q, cudaMemcpyHostToDevice, s_in) ==
                 cudaSuccess &&
             cudaMemcpyAsync(dk_, kh + h0 * es_q, gh * es_q, cudaMemcpyHostToDevice, s_in) ==
                 cudaSuccess &&
             cudaMemcpyAsync(dv_, vh + h0 * es_v, gh * es_v, cudaMemcpyHostToDevice, s_in) ==
                 cudaSuccess &&
             cudaEventRecord(e_in[s], s_in) == cudaSuccess;
        // compute: once the inputs are in and the slot's previous output has left
        ok = ok && cudaStreamWaitEvent(user, e_in[s], 0) == cudaSuccess &&
             cudaStreamWaitEvent(user, e_out[s], 0) == cudaSuccess;
        if (!ok) {
            status = KATA_ERR_CUDA;
            break;
        }
        const long long so = h0 * (long long)dk * dk * dv, zo = h0 * (long long)dk * dk;
        status = kata_chunked_forward(dq, dk_, dv_, dout, 1, gh, T, dk, dv, C, dtype,
                                      state_out ? state_out + so : nullptr,
                                      z_out ? z_out + zo : nullptr, dev + hp.ws_offset,
                                      hp.ws_bytes, stream);
        if (status != KATA_OK) break;
        // output: once computed
        ok = cudaEventRecord(e_comp[s], user) == cudaSuccess &&
             cudaStreamWaitEvent(s_out, e_comp[s], 0) == cudaSuccess &&
             cudaMemcpyAsync(oh + h0 * es_v, dout, gh * es_v, cudaMemcpyDeviceToHost, s_out) ==
                 cudaSuccess &&
             cudaEventRecord(e_out[s], s_out) == cudaSuccess;
        if (!ok) status = KATA_ERR_CUDA;
    }
    // the caller's stream completes after every copy this call queued
    for (int s = 0; s < kata::kSlots; ++s) {
        cudaEventRecord(e_out[s], s_out);
        cudaEventRecord(e_in[s], s_in);
        cudaStreamWaitEvent(user, e_out[s], 0);
        cudaStreamWaitEvent(user, e_in[s], 0);
    }
    kata::release_set(device, set);
    return status;
}

}  // extern "C"
