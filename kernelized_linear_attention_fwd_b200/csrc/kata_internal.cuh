// Internal declarations shared by the CUDA translation units of libkata.
// Not part of the public ABI (that is include/kata.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <initializer_list>
#include <mutex>

#include "../../include/kata.h"

namespace kata {

// ---------------------------------------------------------------------------
// Packed symmetric feature rows.
//
// phi(x) = vec(x x^T) has dk^2 entries but only dk(dk+1)/2 distinct ones:
// (q.k)^2 = sum_i q_i^2 k_i^2 + 2 sum_{i<j} q_i q_j k_i k_j.  The state is kept
// on the half triangle i <= j (row r enumerates (i, j) with i outer), storing
// the plain sums sum_s k_si k_sj v_s; the weight c_ij (1 on the diagonal, 2
// off it) is applied on the query side at readout.
// ---------------------------------------------------------------------------
__host__ __device__ constexpr int packed_rows(int d) { return d * (d + 1) / 2; }

__host__ __device__ inline int packed_row_start(int d, int i) { return i * d - (i * (i - 1)) / 2; }

__host__ __device__ inline void packed_row_ij(int d, int r, int &i, int &j) {
    int a = 0;
    while (r >= d - a) {
        r -= d - a;
        ++a;
    }
    i = a;
    j = a + r;
}

// KATA-Mg with G factors of P = DK / G coordinates each: only pairs (i, j)
// inside one factor carry state.  The packed rows are the G factors' own
// packed rows one after the other: row r = f * Rp + r', Rp = P (P + 1) / 2,
// is the pair (f P + i', f P + j') of the factor's row r' = (i', j').  G = 1
// is the layout above.
__host__ __device__ constexpr int packed_rows_g(int d, int G) { return G * packed_rows(d / G); }

__host__ __device__ inline void packed_row_ij_g(int d, int G, int r, int &i, int &j) {
    const int P = d / G, Rp = packed_rows(P), f = r / Rp;
    packed_row_ij(P, r - f * Rp, i, j);
    i += f * P;
    j += f * P;
}

// Packed row of the pair (i, j), i <= j, both in one factor.
__host__ __device__ inline int packed_row_index_g(int d, int G, int i, int j) {
    const int P = d / G, f = i / P;
    return f * packed_rows(P) + packed_row_start(P, i - f * P) + (j - i);
}

// ---------------------------------------------------------------------------
// Forward plan: segment length, number of segments, workspace layout.
// ---------------------------------------------------------------------------
// kTensorCore: bf16 heads of d = 64, and of d = 16 or 32 read as 64 by the
// tensor maps (TMA fills the columns past d with zeros, which add nothing to
// any product or sum; the output store writes only the first d columns) and
// run on the two-factor layout (Plan::tc_g).
enum class Path : int { kSimt = 0, kTensorCore = 1 };

struct Plan {
    int B, H, T, dk, dv, C;
    kata_dtype dtype;
    long long BH;
    int L;      // segment length (tokens), a multiple of C and of 128; T in the quadratic plan
    int n_seg;  // ceil(T / L)
    int R;      // packed feature rows (of d = 64 on the tensor-core path)
    int g = 1;  // rank-one PSD factors per head (KATA-Mg; 1 = the single factor)
    // Factors of the tensor-core layout the kernels run: g, except that a
    // single-factor head of d <= 32 runs the two-factor layout (its
    // coordinates 32-63, read as zeros, form a second factor that contributes
    // nothing), which holds its state in 1152 rows instead of 2176.
    int tc_g = 1;
    Path path;
    // workspace (bytes from the base, all 256-byte aligned)
    size_t ws_seg_state;  // fp32 per-segment states, exclusive prefix after the scan
    size_t ws_total;      // fp32 total state (packed), when needed
    size_t ws_extra;      // path-specific
    size_t ws_aux;        // path-specific (unused)
    size_t ws_bytes;
};

// Fills `p`; returns KATA_OK or the error the forward must return.  small_tc:
// bf16 heads of d < 64 run the tensor-core kernels (read as 64 by the tensor
// maps); without it (KATA-Mg, whose factors split the head at d / 2) they
// take the fp32 CUDA-core path.
kata_status make_plan(int B, int H, int T, int dk, int dv, int C, kata_dtype dtype, Plan &p,
                      bool small_tc = true);
// The plan of the quadratic form: one segment of T tokens, no workspace.
kata_status make_quadratic_plan(int B, int H, int T, int dk, int dv, kata_dtype dtype, Plan &p);

// Device address of the status word that kernels set when an on-device check
// fails (one per device; resolved on first use with that device current).
int *device_status_ptr();

// True when every non-null pointer is memory of the current device (or
// managed memory).  Host memory and another device's memory are rejected, so
// a call given them returns an error instead of launching kernels that would
// fault.  Checked after every other host-side check.
bool device_ptrs_ok(std::initializer_list<const void *> ptrs);

// Kernel timing (include/kata_profile.h): no-ops unless profiling is enabled.
int prof_begin(const char *name, cudaStream_t st);
void prof_end(int ev, cudaStream_t st);

struct ProfScope {
    int ev;
    cudaStream_t st;
    ProfScope(const char *name, cudaStream_t s) : ev(prof_begin(name, s)), st(s) {}
    ~ProfScope() { prof_end(ev, st); }
};

// Opt-in dynamic shared memory of a kernel, set once per device: the
// attribute lasts for the life of the context, and setting it on every launch
// costs host time that small launches cannot hide.
// The per-device record is guarded, so host threads may make first calls at
// the same time.
template <auto Kernel>
cudaError_t smem_opt_in_once(int bytes) {
    static std::mutex mu;
    static int set_bytes[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && set_bytes[dev] == bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < 64) set_bytes[dev] = bytes;
    return e;
}

// Element loads as fp32.
__device__ __forceinline__ float load_f32(const float *p, long long i) { return p[i]; }
__device__ __forceinline__ float load_f32(const __nv_bfloat16 *p, long long i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_out(float *p, long long i, float x) { p[i] = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, long long i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// Initial state of a forward: the sum of n dense states, S [B, H, d*d, d]
// and Z [B, H, d, d] fp32 (d = the plan's dk); input m starts s_stride
// (z_stride) floats after input m - 1.  n = 0: the forward starts from the
// empty state.
struct InitState {
    const float *s = nullptr;
    const float *z = nullptr;
    int n = 0;
    long long s_stride = 0, z_stride = 0;
};

// Launchers (return cudaSuccess or the launch error).  out == nullptr skips
// the readout (state only: state_out and z_out are then required).
cudaError_t launch_simt_forward(const Plan &p, const void *q, const void *k, const void *v,
                                void *out, float *state_out, float *z_out, const InitState &init,
                                void *ws, cudaStream_t st);
namespace tc {
// Tensor-core path (bf16, d = dv in {16, 32, 64}, computed as 64): workspace
// layout and launcher.
// reuse_seg: the workspace already holds every segment's state, written by a
// state-only launch for the same keys, values and sizes; skip building them.
void plan_tc_workspace(Plan &p);
cudaError_t launch_tc_forward(const Plan &p, const void *q, const void *k, const void *v,
                              void *out, float *state_out, float *z_out, const InitState &init,
                              void *ws, cudaStream_t st, bool reuse_seg = false);
// Streaming multiprocessors of the current device (cached).
int num_sms();
}  // namespace tc

// Decode step on the dense (d^2 rows) or packed (d(d+1)/2 rows) state layout.
cudaError_t launch_decode(int B, int H, int dk, int dv, kata_dtype dtype, const void *q,
                          const void *k, const void *v, void *out, float *state, float *z,
                          bool packed, cudaStream_t st);
// The decode step of KATA-Mg with g factors on the dense layout (g = 1: the
// dense step above).
cudaError_t launch_decode_mg(int B, int H, int dk, int g, kata_dtype dtype, const void *q,
                             const void *k, const void *v, void *out, float *state, float *z,
                             cudaStream_t st);
// Dense <-> packed state conversion (pack: dense -> packed).
cudaError_t launch_state_convert(bool pack, int B, int H, int dk, const float *src_s,
                                 const float *src_z, float *dst_s, float *dst_z, cudaStream_t st);

}  // namespace kata
