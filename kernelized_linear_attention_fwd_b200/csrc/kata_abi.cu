// C ABI of libkata: argument checks, the forward plan, and kernel dispatch.
// Declarations and the contract of every entry point: include/kata.h.
#include <stdint.h>

#include <initializer_list>
#include <mutex>

#include "kata_internal.cuh"

namespace kata {

namespace {

__device__ int g_device_status = 0;


constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_chunk(int C) {
    return C == 16 || C == 32 || C == 64 || C == 128 || C == 256 || C == 512 || C == 1024 ||
           C == 2048 || C == 4096;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// Segment length: states are stored every L tokens.  Inside a segment the
// exact causal quadratic form is used, so L trades state traffic (~1/L)
// against quadratic work (~L).  Chunks of C <= 256 tokens are merged into
// segments of a length fixed per head size (a multiple of C), so every such C
// runs the same schedule; C >= 512 sets the segment itself (L = C).  L is a
// multiple of 256, as the tensor-core readout's 256-query work items need.
int segment_length(int dk, int C) {
    if (C >= 512) return C;
    return dk >= 64 ? 1024 : (dk >= 32 ? 512 : 256);
}

}  // namespace

int *device_status_ptr() {
    static std::mutex mu;
    static int *ptrs[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int *>(p);
    }
    return ptrs[dev];
}

bool device_ptrs_ok(std::initializer_list<const void *> ptrs) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    for (const void *p : ptrs) {
        if (p == nullptr) continue;
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
            cudaGetLastError();  // clear the error this query left, so it reaches no later call
            return false;
        }
        if (a.type == cudaMemoryTypeManaged) continue;
        if (a.type != cudaMemoryTypeDevice || a.device != dev) return false;
    }
    return true;
}

kata_status make_plan(int B, int H, int T, int dk, int dv, int C, kata_dtype dtype, Plan &p,
                      bool small_tc) {
    if (B < 1 || H < 1 || T < 1 || dk < 1 || dv < 1) return KATA_ERR_INVALID_ARG;
    if (!valid_chunk(C)) return KATA_ERR_INVALID_ARG;
    if (dtype != KATA_F32 && dtype != KATA_BF16) return KATA_ERR_UNSUPPORTED;
    if (dk != dv || (dk != 16 && dk != 32 && dk != 64)) return KATA_ERR_UNSUPPORTED;
    const long long BH = (long long)B * H;
    if (BH * (long long)T > (1LL << 40)) return KATA_ERR_UNSUPPORTED;
    p.B = B;
    p.H = H;
    p.T = T;
    p.dk = dk;
    p.dv = dv;
    p.C = C;
    p.dtype = dtype;
    p.BH = BH;
    p.path = (dtype == KATA_BF16 && (dk == 64 || small_tc)) ? Path::kTensorCore : Path::kSimt;
    if (p.path == Path::kTensorCore) {
        // the tensor-core kernels compute every head as d = 64; a head of d <= 32
        // as a two-factor head whose second factor (coordinates 32-63) is zero
        p.tc_g = dk <= 32 ? 2 : 1;
        p.R = packed_rows_g(64, p.tc_g);
        p.L = segment_length(64, C);
        p.n_seg = (T + p.L - 1) / p.L;
        tc::plan_tc_workspace(p);
        return KATA_OK;
    }
    p.R = packed_rows(dk);
    p.L = segment_length(dk, C);
    p.n_seg = (T + p.L - 1) / p.L;
    const size_t E = (size_t)p.R * (dv + 1);
    const size_t seg_bytes = (size_t)BH * p.n_seg * E * sizeof(float);
    const size_t total_bytes = (size_t)BH * E * sizeof(float);  // also for one segment + initial state
    p.ws_seg_state = 0;
    p.ws_total = align_up(seg_bytes);
    p.ws_extra = p.ws_total + align_up(total_bytes);
    p.ws_aux = 0;
    p.ws_bytes = p.ws_extra;
    return KATA_OK;
}

// KATA-Mg with g factors: g = 1 is the plain plan.  g = 2: bf16 heads of
// d = 64 take the tensor-core path (its two-factor layout); every other head
// size and dtype takes the fp32 CUDA-core path (the tensor-core kernels'
// d = 64 view of a smaller head would put the factor boundary at 32, not d/2).  Other g: unsupported.
kata_status make_plan_mg(int B, int H, int T, int dk, int dv, int C, int g, kata_dtype dtype,
                         Plan &p) {
    if (g == 1) return make_plan(B, H, T, dk, dv, C, dtype, p);
    if (g < 1) return KATA_ERR_INVALID_ARG;
    const kata_status s = make_plan(B, H, T, dk, dv, C, dtype, p, false);
    if (s != KATA_OK) return s;
    if (g != 2 || dk % g != 0) return KATA_ERR_UNSUPPORTED;
    p.g = g;
    p.R = packed_rows_g(dk, g);
    if (p.path == Path::kTensorCore) {
        p.tc_g = g;
        tc::plan_tc_workspace(p);
        return KATA_OK;
    }
    const size_t E = (size_t)p.R * (dv + 1);
    p.ws_seg_state = 0;
    p.ws_total = align_up((size_t)p.BH * p.n_seg * E * sizeof(float));
    p.ws_extra = p.ws_total + align_up((size_t)p.BH * E * sizeof(float));
    p.ws_aux = 0;
    p.ws_bytes = p.ws_extra;
    return KATA_OK;
}

// The quadratic form is the chunked plan with one segment spanning the whole
// sequence: no state is built, scanned or stored, so no workspace is used.
kata_status make_quadratic_plan(int B, int H, int T, int dk, int dv, kata_dtype dtype, Plan &p) {
    const kata_status s = make_plan(B, H, T, dk, dv, 256, dtype, p);
    if (s != KATA_OK) return s;
    p.tc_g = 1;  // no state: the one-factor readout, whose intra steps are 128 keys
    p.L = T;
    p.n_seg = 1;
    p.ws_seg_state = p.ws_total = p.ws_extra = p.ws_aux = p.ws_bytes = 0;
    return KATA_OK;
}

namespace {

// Checks shared by both forward entry points: q, k, v, out present, 16-byte
// aligned, and out disjoint from the inputs.
kata_status check_forward_io(const Plan &p, const void *q, const void *k, const void *v,
                             const void *out) {
    if (!q || !k || !v || !out) return KATA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return KATA_ERR_INVALID_ARG;
    const size_t es = p.dtype == KATA_BF16 ? 2 : 4;
    const size_t nq = (size_t)p.BH * p.T * p.dk * es, nv = (size_t)p.BH * p.T * p.dv * es;
    if (overlaps(out, nv, q, nq) || overlaps(out, nv, k, nq) || overlaps(out, nv, v, nv))
        return KATA_ERR_INVALID_ARG;
    return KATA_OK;
}

// reuse_seg: the workspace holds the segment states a state-only launch wrote
// for the same inputs and sizes.  The tensor-core path then skips building
// them; the fp32 path's state-only scan leaves prefixes, not the states, in
// place, so it rebuilds them (same result).
cudaError_t launch_forward(const Plan &p, const void *q, const void *k, const void *v, void *out,
                           float *state_out, float *z_out, const InitState &init, void *ws,
                           cudaStream_t st, bool reuse_seg = false) {
    return p.path == Path::kTensorCore
               ? tc::launch_tc_forward(p, q, k, v, out, state_out, z_out, init, ws, st, reuse_seg)
               : launch_simt_forward(p, q, k, v, out, state_out, z_out, init, ws, st);
}

// Workspace present, large enough and 256-byte aligned when the plan needs one.
kata_status check_workspace(const Plan &p, const void *workspace, size_t workspace_bytes) {
    if (p.ws_bytes == 0) return KATA_OK;
    if (!workspace || workspace_bytes < p.ws_bytes) return KATA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KATA_ERR_WORKSPACE;
    return KATA_OK;
}

// state_out and z_out: both or neither, 16-byte aligned, disjoint from each
// other and from the inputs.
kata_status check_state_out(const Plan &p, const float *state_out, const float *z_out,
                            const void *q, const void *k, const void *v, bool required) {
    if ((state_out == nullptr) != (z_out == nullptr)) return KATA_ERR_INVALID_ARG;
    if (!state_out) return required ? KATA_ERR_INVALID_ARG : KATA_OK;
    if (!aligned16(state_out) || !aligned16(z_out)) return KATA_ERR_INVALID_ARG;
    const size_t es = p.dtype == KATA_BF16 ? 2 : 4;
    const size_t ns = (size_t)p.BH * p.dk * p.dk * p.dv * 4, nz = (size_t)p.BH * p.dk * p.dk * 4;
    const size_t nq = (size_t)p.BH * p.T * p.dk * es, nv = (size_t)p.BH * p.T * p.dv * es;
    if (overlaps(state_out, ns, z_out, nz)) return KATA_ERR_INVALID_ARG;
    for (const float *o : {state_out, z_out}) {
        const size_t n = o == state_out ? ns : nz;
        if ((q && overlaps(o, n, q, nq)) || overlaps(o, n, k, nq) || overlaps(o, n, v, nv))
            return KATA_ERR_INVALID_ARG;
    }
    return KATA_OK;
}

// The decode step on either state layout; g factors (KATA-Mg) on the dense one.
kata_status decode_step(const void *q, const void *k, const void *v, void *out, float *state,
                        float *z, int B, int H, int dk, int dv, kata_dtype dtype, bool packed,
                        kata_stream_t stream, int g = 1) {
    if (B < 1 || H < 1 || dk < 1 || dv < 1 || g < 1) return KATA_ERR_INVALID_ARG;
    if (g > 2 || (packed && g != 1)) return KATA_ERR_UNSUPPORTED;
    if (dtype != KATA_F32 && dtype != KATA_BF16) return KATA_ERR_UNSUPPORTED;
    if (dk != dv || (dk != 16 && dk != 32 && dk != 64)) return KATA_ERR_UNSUPPORTED;
    if ((long long)B * H > 0x7fffffffLL / 8) return KATA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !out || !state || !z) return KATA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state) ||
        !aligned16(z))
        return KATA_ERR_INVALID_ARG;
    const size_t es = dtype == KATA_BF16 ? 2 : 4;
    const size_t BH = (size_t)B * H;
    const size_t rows = packed ? (size_t)packed_rows(dk) : (size_t)dk * dk;
    const size_t ns = BH * rows * dv * 4, nz = BH * rows * 4, no = BH * dv * es;
    if (overlaps(state, ns, z, nz) || overlaps(out, no, state, ns) || overlaps(out, no, z, nz))
        return KATA_ERR_INVALID_ARG;
    if (!device_ptrs_ok({q, k, v, out, state, z})) return KATA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = g == 1 ? launch_decode(B, H, dk, dv, dtype, q, k, v, out, state, z, packed, st)
                                 : launch_decode_mg(B, H, dk, g, dtype, q, k, v, out, state, z, st);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
}

kata_status state_convert(bool pack, const float *src_s, const float *src_z, float *dst_s,
                          float *dst_z, int B, int H, int dk, int dv, kata_stream_t stream) {
    if (B < 1 || H < 1 || dk < 1 || dv < 1) return KATA_ERR_INVALID_ARG;
    if (dk != dv || (dk != 16 && dk != 32 && dk != 64)) return KATA_ERR_UNSUPPORTED;
    if (!src_s || !src_z || !dst_s || !dst_z) return KATA_ERR_INVALID_ARG;
    if (!aligned16(src_s) || !aligned16(src_z) || !aligned16(dst_s) || !aligned16(dst_z))
        return KATA_ERR_INVALID_ARG;
    const size_t BH = (size_t)B * H;
    const size_t dense_s = BH * dk * dk * dv * 4, dense_z = BH * dk * dk * 4;
    const size_t pk_s = BH * packed_rows(dk) * dv * 4, pk_z = BH * packed_rows(dk) * 4;
    const size_t ss = pack ? dense_s : pk_s, sz = pack ? dense_z : pk_z;
    const size_t ds = pack ? pk_s : dense_s, dz = pack ? pk_z : dense_z;
    for (const void *d : {static_cast<const void *>(dst_s), static_cast<const void *>(dst_z)}) {
        const size_t n = d == dst_s ? ds : dz;
        if (overlaps(d, n, src_s, ss) || overlaps(d, n, src_z, sz)) return KATA_ERR_INVALID_ARG;
    }
    if (overlaps(dst_s, ds, dst_z, dz)) return KATA_ERR_INVALID_ARG;
    if (!device_ptrs_ok({src_s, src_z, dst_s, dst_z})) return KATA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = launch_state_convert(pack, B, H, dk, src_s, src_z, dst_s, dst_z, st);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
}

}  // namespace

}  // namespace kata

using kata::Plan;
using kata::aligned16;
using kata::overlaps;

extern "C" {

int kata_version(void) { return 100; }

const char *kata_status_string(kata_status s) {
    switch (s) {
        case KATA_OK: return "KATA_OK";
        case KATA_ERR_INVALID_ARG: return "KATA_ERR_INVALID_ARG";
        case KATA_ERR_UNSUPPORTED: return "KATA_ERR_UNSUPPORTED";
        case KATA_ERR_WORKSPACE: return "KATA_ERR_WORKSPACE";
        case KATA_ERR_CUDA: return "KATA_ERR_CUDA";
        case KATA_ERR_TIMEOUT: return "KATA_ERR_TIMEOUT";
    }
    return "KATA_ERR_UNKNOWN";
}

size_t kata_chunked_forward_workspace_bytes(int B, int H, int T, int dk, int dv, int C,
                                            kata_dtype dtype) {
    Plan p;
    if (kata::make_plan(B, H, T, dk, dv, C, dtype, p) != KATA_OK) return 0;
    return p.ws_bytes;
}

kata_status kata_chunked_forward(const void *q, const void *k, const void *v, void *out, int B,
                                 int H, int T, int dk, int dv, int C, kata_dtype dtype,
                                 float *state_out, float *z_out, void *workspace,
                                 size_t workspace_bytes, kata_stream_t stream) {
    Plan p;
    const kata_status ps = kata::make_plan(B, H, T, dk, dv, C, dtype, p);
    if (ps != KATA_OK) return ps;
    const kata_status io = kata::check_forward_io(p, q, k, v, out);
    if (io != KATA_OK) return io;
    const kata_status so = kata::check_state_out(p, state_out, z_out, q, k, v, false);
    if (so != KATA_OK) return so;
    const kata_status ws = kata::check_workspace(p, workspace, workspace_bytes);
    if (ws != KATA_OK) return ws;
    if (!kata::device_ptrs_ok({q, k, v, out, state_out, z_out, p.ws_bytes ? workspace : nullptr}))
        return KATA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e =
        kata::launch_forward(p, q, k, v, out, state_out, z_out, kata::InitState{}, workspace, st);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
}

size_t kata_mg_chunked_forward_workspace_bytes(int B, int H, int T, int dk, int dv, int C, int g,
                                               kata_dtype dtype) {
    Plan p;
    if (kata::make_plan_mg(B, H, T, dk, dv, C, g, dtype, p) != KATA_OK) return 0;
    return p.ws_bytes;
}

kata_status kata_mg_chunked_forward(const void *q, const void *k, const void *v, void *out, int B,
                                    int H, int T, int dk, int dv, int C, int g, kata_dtype dtype,
                                    float *state_out, float *z_out, void *workspace,
                                    size_t workspace_bytes, kata_stream_t stream) {
    Plan p;
    const kata_status ps = kata::make_plan_mg(B, H, T, dk, dv, C, g, dtype, p);
    if (ps != KATA_OK) return ps;
    const kata_status io = kata::check_forward_io(p, q, k, v, out);
    if (io != KATA_OK) return io;
    const kata_status so = kata::check_state_out(p, state_out, z_out, q, k, v, false);
    if (so != KATA_OK) return so;
    const kata_status ws = kata::check_workspace(p, workspace, workspace_bytes);
    if (ws != KATA_OK) return ws;
    if (!kata::device_ptrs_ok({q, k, v, out, state_out, z_out, p.ws_bytes ? workspace : nullptr}))
        return KATA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e =
        kata::launch_forward(p, q, k, v, out, state_out, z_out, kata::InitState{}, workspace, st);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
}

kata_status kata_chunked_state(const void *k, const void *v, int B, int H, int T, int dk, int dv,
                               int C, kata_dtype dtype, float *state_out, float *z_out,
                               void *workspace, size_t workspace_bytes, kata_stream_t stream) {
    Plan p;
    const kata_status ps = kata::make_plan(B, H, T, dk, dv, C, dtype, p);
    if (ps != KATA_OK) return ps;
    if (!k || !v || !aligned16(k) || !aligned16(v)) return KATA_ERR_INVALID_ARG;
    const kata_status so = kata::check_state_out(p, state_out, z_out, nullptr, k, v, true);
    if (so != KATA_OK) return so;
    const kata_status ws = kata::check_workspace(p, workspace, workspace_bytes);
    if (ws != KATA_OK) return ws;
    if (!kata::device_ptrs_ok({k, v, state_out, z_out, p.ws_bytes ? workspace : nullptr}))
        return KATA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = kata::launch_forward(p, nullptr, k, v, nullptr, state_out, z_out,
                                               kata::InitState{}, workspace, st);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
}

kata_status kata_chunked_forward_from_state(const void *q, const void *k, const void *v, void *out,
                                            int B, int H, int T, int dk, int dv, int C,
                                            kata_dtype dtype, const float *state_in,
                                            const float *z_in, int n_in, size_t s_stride,
                                            size_t z_stride, float *state_out, float *z_out,
                                            void *workspace, size_t workspace_bytes,
                                            unsigned flags, kata_stream_t stream) {
    Plan p;
    if (flags & ~KATA_REUSE_SEGMENT_STATES) return KATA_ERR_INVALID_ARG;
    const kata_status ps = kata::make_plan(B, H, T, dk, dv, C, dtype, p);
    if (ps != KATA_OK) return ps;
    const kata_status io = kata::check_forward_io(p, q, k, v, out);
    if (io != KATA_OK) return io;
    const kata_status so = kata::check_state_out(p, state_out, z_out, q, k, v, false);
    if (so != KATA_OK) return so;
    if (n_in < 0) return KATA_ERR_INVALID_ARG;
    kata::InitState init;
    if (n_in > 0) {
        if (!state_in || !z_in || !aligned16(state_in) || !aligned16(z_in))
            return KATA_ERR_INVALID_ARG;
        if (n_in > 1 && s_stride % 4 != 0) return KATA_ERR_INVALID_ARG;  // 16-byte rows
        const size_t ns = (size_t)p.BH * dk * dk * dv * 4, nz = (size_t)p.BH * dk * dk * 4;
        const size_t span_s = (size_t)(n_in - 1) * s_stride * 4 + ns;
        const size_t span_z = (size_t)(n_in - 1) * z_stride * 4 + nz;
        const size_t no = (size_t)p.BH * T * dv * (dtype == KATA_BF16 ? 2 : 4);
        if (overlaps(out, no, state_in, span_s) || overlaps(out, no, z_in, span_z))
            return KATA_ERR_INVALID_ARG;
        // every input is read before the state is written: state_out may be state_in
        // itself (one input, updated in place) but must not overlap the inputs otherwise
        const bool in_place = n_in == 1 && state_out == state_in && z_out == z_in;
        if (state_out && !in_place &&
            (overlaps(state_out, ns, state_in, span_s) || overlaps(state_out, ns, z_in, span_z) ||
             overlaps(z_out, nz, state_in, span_s) || overlaps(z_out, nz, z_in, span_z)))
            return KATA_ERR_INVALID_ARG;
        init.s = state_in;
        init.z = z_in;
        init.n = n_in;
        init.s_stride = (long long)s_stride;
        init.z_stride = (long long)z_stride;
    }
    const kata_status ws = kata::check_workspace(p, workspace, workspace_bytes);
    if (ws != KATA_OK) return ws;
    if (!kata::device_ptrs_ok({q, k, v, out, state_out, z_out, init.s, init.z,
                               p.ws_bytes ? workspace : nullptr}))
        return KATA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = kata::launch_forward(p, q, k, v, out, state_out, z_out, init, workspace,
                                               st, (flags & KATA_REUSE_SEGMENT_STATES) != 0);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
}

kata_status kata_quadratic_forward(const void *q, const void *k, const void *v, void *out, int B,
                                   int H, int T, int dk, int dv, kata_dtype dtype,
                                   kata_stream_t stream) {
    Plan p;
    const kata_status ps = kata::make_quadratic_plan(B, H, T, dk, dv, dtype, p);
    if (ps != KATA_OK) return ps;
    const kata_status io = kata::check_forward_io(p, q, k, v, out);
    if (io != KATA_OK) return io;
    if (p.BH * ((T + 255LL) / 256) >= 0x7fffffffLL) return KATA_ERR_UNSUPPORTED;
    if (!kata::device_ptrs_ok({q, k, v, out})) return KATA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e =
        kata::launch_forward(p, q, k, v, out, nullptr, nullptr, kata::InitState{}, nullptr, st);
    return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA;
}

kata_status kata_decode_step(const void *q, const void *k, const void *v, void *out,
                             float *state, float *z, int B, int H, int dk, int dv,
                             kata_dtype dtype, kata_stream_t stream) {
    return kata::decode_step(q, k, v, out, state, z, B, H, dk, dv, dtype, false, stream);
}

kata_status kata_mg_decode_step(const void *q, const void *k, const void *v, void *out,
                                float *state, float *z, int B, int H, int dk, int dv, int g,
                                kata_dtype dtype, kata_stream_t stream) {
    return kata::decode_step(q, k, v, out, state, z, B, H, dk, dv, dtype, false, stream, g);
}

kata_status kata_decode_step_packed(const void *q, const void *k, const void *v, void *out,
                                    float *state_p, float *z_p, int B, int H, int dk, int dv,
                                    kata_dtype dtype, kata_stream_t stream) {
    return kata::decode_step(q, k, v, out, state_p, z_p, B, H, dk, dv, dtype, true, stream);
}

kata_status kata_state_pack(const float *state, const float *z, float *state_p, float *z_p, int B,
                            int H, int dk, int dv, kata_stream_t stream) {
    return kata::state_convert(true, state, z, state_p, z_p, B, H, dk, dv, stream);
}

kata_status kata_state_unpack(const float *state_p, const float *z_p, float *state, float *z,
                              int B, int H, int dk, int dv, kata_stream_t stream) {
    return kata::state_convert(false, state_p, z_p, state, z, B, H, dk, dv, stream);
}

kata_status kata_get_device_status(kata_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return KATA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, kata::g_device_status, sizeof(int)) != cudaSuccess)
        return KATA_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(kata::g_device_status, &zero, sizeof(int)) != cudaSuccess)
            return KATA_ERR_CUDA;
    }
    return static_cast<kata_status>(word);
}

}  // extern "C"
