/*
 * kata.h — C ABI of the KATA causal forward on NVIDIA B200 (sm_100a).
 *
 * KATA ("Kernelized Linear Attention: Breaking the Capacity Wall with
 * Symmetric Cones") with the rank-one PSD feature phi(x) = vec(x x^T):
 * every attention weight is <q q^T, k k^T> = (q.k)^2 >= 0, and dividing by the
 * running sum of weights makes each output a convex combination of the values
 * seen so far.  Per head, for t = 0 .. T-1:
 *
 *     y_t = sum_{s<=t} (q_t.k_s)^2 v_s / sum_{s<=t} (q_t.k_s)^2     (y_t = 0 if 0)
 *
 * Sources (page title and section):
 *   - gist.science summary of the paper, Technical summary 2.2 "PSD cone
 *     (rank one)": psi(u) = u u^T squares the raw inner product.
 *   - same, 2.1 "output gating": the normalised denominator is a convex,
 *     parameter-free gate between the previous readout and the current value
 *     (so the current token is included, s <= t).
 *   - same, 2.3 "hardware-aligned implementation": chunked parallelism,
 *     tensor cores inside a chunk, an associative scan (parallel prefix sum)
 *     of chunk states across chunks, depth O(log N_C).
 *   - arXiv abstract of the paper: "exact O(T) chunked-state form",
 *     "constant-time recurrent inference".
 *
 * Readings where the pages are silent: no scale constant; no epsilon in the
 * denominator; a zero denominator gives y = 0; the state and normaliser are
 * kept in fp32; the output has the input's dtype.
 *
 * General contract of every entry point
 *   - All tensor pointers are DEVICE pointers (except the host buffers of
 *     kata_chunked_forward_host), owned by the caller, 16-byte aligned, dense
 *     row-major with the layout stated per argument, in the memory of the
 *     CURRENT device (or managed memory): the kernels run on the current
 *     device, and a pointer to host memory or to another device's memory is
 *     rejected with KATA_ERR_INVALID_ARG before anything is launched.  The
 *     library allocates no device memory and keeps no state between calls
 *     beyond per-device handles: the device addresses of its status word and
 *     of the kata_chunked_forward_noalloc scratch (looked up on first use),
 *     and the copy streams and events of kata_chunked_forward_host (created
 *     on first use, reused after).  Those handles belong to the device's
 *     context: do not use the library on a device after cudaDeviceReset() on
 *     it within the same process.
 *   - Work is enqueued on `stream` (NULL = legacy default stream) and the call
 *     returns without synchronising.  Errors found on the host (bad sizes,
 *     null or misaligned pointers, short workspace) return before anything is
 *     launched; a launch failure returns KATA_ERR_CUDA.  Errors raised while
 *     kernels run are recorded in a device status word that
 *     kata_get_device_status() reads.
 *   - Outputs must not alias inputs.
 *   - Supported head sizes: dk = dv in {16, 32, 64}; others return
 *     KATA_ERR_UNSUPPORTED.  T >= 1 (any value; the ragged tail is exact).
 *   - Calls on different streams may run concurrently if their buffers are
 *     disjoint.
 *   - A call's kernels run after the work queued on `stream` before it and
 *     end before the work queued after it starts.  On small problems (each
 *     kernel at most one work item per SM) the chunked calls (the forwards,
 *     the state-only call) start their scan, and the forwards their readout,
 *     as programmatic dependents of the call's previous
 *     kernel (CUDA programmatic dependent launch): they may begin while it
 *     finishes, but read nothing it writes until it has finished, and the
 *     call's last kernel ends after all of them.  Captured into a CUDA graph,
 *     those launches become programmatic edges.
 */
#ifndef KATA_H_
#define KATA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *kata_stream_t;

typedef enum {
    KATA_OK = 0,
    KATA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, non-positive size, bad chunk size */
    KATA_ERR_UNSUPPORTED = 2, /* a head size or dtype the kernels do not cover */
    KATA_ERR_WORKSPACE = 3,   /* workspace null or smaller than the size query returned */
    KATA_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
    KATA_ERR_TIMEOUT = 5      /* a bounded on-device wait gave up (device status only) */
} kata_status;

typedef enum {
    KATA_F32 = 0, /* float32 q, k, v and out */
    KATA_BF16 = 1 /* bfloat16 q, k, v and out; fp32 accumulation */
} kata_dtype;

/* Library version, major * 10000 + minor * 100 + patch. */
int kata_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *kata_status_string(kata_status status);

/*
 * Bytes of device workspace kata_chunked_forward needs for this problem.
 * Returns 0 for arguments the forward would reject.  The value depends only
 * on the arguments and may be 0 for short sequences (no state needs storing).
 */
size_t kata_chunked_forward_workspace_bytes(int B, int H, int T, int dk, int dv, int C,
                                            kata_dtype dtype);

/*
 * Causal KATA forward in the exact chunked-state form
 * (gist.science summary 2.3 and the arXiv abstract, "exact O(T)
 * chunked-state form"; the associative scan of chunk states of summary 2.3).
 *
 *   q, k   [B, H, T, dk]  dtype      queries, keys
 *   v      [B, H, T, dv]  dtype      values
 *   out    [B, H, T, dv]  dtype      y_t as defined above
 *   C      chunk size: 16, 32, 64, 128, 256, 512, 1024, 2048 or 4096.  The
 *          result does not depend on C (the form is exact for every C).  C
 *          sets where states are kept; between them the exact causal
 *          quadratic form is used:
 *            C <= 256: chunks are merged into segments of a fixed length,
 *              a multiple of C: L = 1024 tokens for bf16 (the tensor cores,
 *              every head size) and for fp32 dk = 64, 512 for fp32 dk = 32,
 *              256 for fp32 dk = 16.  Every such C runs the same kernels on
 *              the same schedule (on the tensor cores the intra-segment term
 *              is computed in 128-key steps with the diagonal block masked).
 *            C >= 512: states are kept every C tokens (L = C), which trades
 *              state traffic and scan depth (about 1/C) against intra-chunk
 *              work (about C).
 *          The scan over the ceil(T / L) segment states is the associative
 *          scan across chunks.
 *   state_out  nullable, [B, H, dk*dk, dv] fp32: S_T = sum_{s<T} phi(k_s) v_s^T,
 *          row index i*dk + j (symmetric in i, j), ready for kata_decode_step.
 *   z_out  nullable, [B, H, dk, dk] fp32: Z_T = sum_{s<T} k_s k_s^T.
 *          state_out and z_out must be both NULL or both non-NULL.
 *   workspace, workspace_bytes: device scratch of at least
 *          kata_chunked_forward_workspace_bytes(...) bytes (may be NULL when
 *          that is 0).  Its contents on entry do not matter.
 *
 * dtype KATA_BF16 runs the tensor-core (tcgen05) path: d = 64 directly,
 * d = 16 and 32 read as 64 by the kernels' tensor maps, which fill the
 * columns past d with zeros (exact: zeros add nothing to any product or sum;
 * the output store writes only the first d columns).  Heads of d = 16 and 32
 * run the kernels' two-factor state layout (the same as kata_mg_chunked_forward
 * with g = 2 at d = 64): coordinates 32-63 are zero, so (q.k)^2 = (q_a.k_a)^2
 * + (q_b.k_b)^2 with the second term 0, and the state needs 1152 packed rows
 * instead of 2176; the intra-segment scores are formed whole.  KATA_F32 runs
 * fp32 CUDA-core arithmetic end to end.
 */
kata_status kata_chunked_forward(const void *q, const void *k, const void *v, void *out, int B,
                                 int H, int T, int dk, int dv, int C, kata_dtype dtype,
                                 float *state_out, float *z_out, void *workspace,
                                 size_t workspace_bytes, kata_stream_t stream);

/*
 * The state after T tokens, without the outputs: S_T = sum_{s<T} phi(k_s) v_s^T
 * and Z_T = sum_{s<T} k_s k_s^T, from the chunk states and their scan
 * (gist.science summary 2.3; arXiv abstract, "exact O(T) chunked-state form"
 * and "constant-time recurrent inference": the state a prefill hands to the
 * recurrent decode).  It is also the first step of the sequence-sharded
 * forward: each block of a long sequence computes its own total, and a later
 * block starts from the sum of the earlier blocks' totals
 * (kata_chunked_forward_from_state), the chunk scan taken one level up.
 *
 *   k      [B, H, T, dk]  dtype;  v  [B, H, T, dv]  dtype
 *   state_out  [B, H, dk*dk, dv] fp32, required (layout as kata_chunked_forward)
 *   z_out      [B, H, dk, dk] fp32, required
 *   workspace  as kata_chunked_forward, of at least
 *              kata_chunked_forward_workspace_bytes(...) bytes
 *
 * The outputs must not overlap k, v or each other.
 */
kata_status kata_chunked_state(const void *k, const void *v, int B, int H, int T, int dk, int dv,
                               int C, kata_dtype dtype, float *state_out, float *z_out,
                               void *workspace, size_t workspace_bytes, kata_stream_t stream);

/*
 * kata_chunked_forward continuing from a given state: tokens 0 .. T-1 of the
 * call are preceded by a history whose state is S_0 = sum_m state_in[m],
 * Z_0 = sum_m z_in[m] (m = 0 .. n_in-1), so
 *
 *   y_t = (phi(q_t)^T S_0 + sum_{s<=t} (q_t.k_s)^2 v_s)
 *         / (q_t^T Z_0 q_t + sum_{s<=t} (q_t.k_s)^2)                (0 if 0)
 *
 * (the same chunked-state form with the initial state as the prefix of the
 * first chunk: gist.science summary 2.3; arXiv abstract).  Uses: a long
 * prompt processed in pieces, and the sequence-sharded forward, where block
 * r passes the all-gathered totals of all blocks with n_in = r.
 *
 *   q, k, v, out, B .. dtype, workspace: as kata_chunked_forward (same size
 *          query, same workspace).
 *   state_in   n_in fp32 states [B, H, dk*dk, dv] (symmetric in (i, j), as
 *              every state this library writes); state m starts at
 *              state_in + m * s_stride (floats; a multiple of 4 when n_in > 1).
 *   z_in       n_in fp32 [B, H, dk, dk]; z m starts at z_in + m * z_stride.
 *              Separately stacked inputs take s_stride = B*H*dk*dk*dv and
 *              z_stride = B*H*dk*dk; one gathered buffer of [S | Z] blocks
 *              takes the block size for both.
 *   n_in       number of inputs to sum, >= 0; 0 behaves as kata_chunked_forward
 *              (state_in and z_in may then be NULL).
 *   state_out, z_out  nullable (both or neither): S_0 + S_T and Z_0 + Z_T,
 *              the state after the call's last token.  With n_in = 1 they may
 *              be state_in and z_in themselves (updated in place); otherwise
 *              they must not overlap the inputs.
 *   flags      0, or KATA_REUSE_SEGMENT_STATES: the workspace holds what
 *              kata_chunked_state last wrote into it for the same k, v, B, H,
 *              T, dk, dv, C and dtype, and nothing has written it since (the
 *              sequence-sharded forward: the state pass before the all-gather,
 *              this call after it).  The tensor-core path then skips building
 *              the per-segment states again; the fp32 path rebuilds them.
 *              The result is the same either way; a workspace that does not
 *              hold those states gives wrong outputs, never a fault.  Other
 *              bits: KATA_ERR_INVALID_ARG.
 *
 * Accuracy (bf16): the term phi(q_t)^T S_0 is formed from bf16 products
 * q_i q_j and a bf16 copy of the state, so its rounding error scales with
 * sum_s (sum_i |q_t,i k_s,i|)^2 |v_s| over the history's tokens s, not with
 * the term itself (the products' signs cancel).  After a long history the
 * positive weights dominate; after a history of only a few tokens, a row
 * whose small total weight comes mostly from history keys nearly orthogonal
 * to its query can miss the bf16 tolerance of the plain forward.  fp32
 * inputs have the same structure at fp32 rounding.
 */
#define KATA_REUSE_SEGMENT_STATES 1u

kata_status kata_chunked_forward_from_state(const void *q, const void *k, const void *v, void *out,
                                            int B, int H, int T, int dk, int dv, int C,
                                            kata_dtype dtype, const float *state_in,
                                            const float *z_in, int n_in, size_t s_stride,
                                            size_t z_stride, float *state_out, float *z_out,
                                            void *workspace, size_t workspace_bytes,
                                            unsigned flags, kata_stream_t stream);

/*
 * kata_chunked_forward on q, k, v and out in HOST memory (pin it, e.g. with
 * cudaHostAlloc, for the copies to overlap; pageable memory works but
 * serialises them).  A deployment convenience, not a step of the method:
 * the heads are independent, so they run in groups of heads_per_group
 * (<= 0: the library picks about 8 groups), and while one group computes on
 * `stream` the next group's inputs are copied to the device and the previous
 * group's outputs back to the host, on two streams of the call's own.
 *
 *   q, k, v, out   host, [B, H, T, dk|dv] as kata_chunked_forward
 *   state_out, z_out  nullable DEVICE pointers, as kata_chunked_forward
 *   device_buffer  device scratch of at least
 *                  kata_chunked_forward_host_buffer_bytes(...) bytes,
 *                  256-byte aligned: two groups' staged q, k, v and out, and
 *                  one group's forward workspace
 *
 * Work is ordered after what is already queued on `stream`, and `stream`
 * completes only after every copy of the call (out holds the result once
 * `stream` has been synchronised).  The call's two copy streams and its
 * events come from a per-device pool (created by the first call, reused by
 * later ones; concurrent calls from several host threads each take their
 * own).  Same results as kata_chunked_forward on device copies of the inputs.
 */
size_t kata_chunked_forward_host_buffer_bytes(int B, int H, int T, int dk, int dv, int C,
                                              kata_dtype dtype, int heads_per_group);
kata_status kata_chunked_forward_host(const void *q, const void *k, const void *v, void *out,
                                      int B, int H, int T, int dk, int dv, int C,
                                      kata_dtype dtype, float *state_out, float *z_out,
                                      void *device_buffer, size_t device_buffer_bytes,
                                      int heads_per_group, kata_stream_t stream);

/*
 * kata_chunked_forward without a caller-provided workspace, for callers that
 * cannot allocate device memory themselves: code running inside a host
 * framework that owns all device memory through its own pool, or a
 * latency-critical loop whose memory is fixed before it starts.
 * The paper has no counterpart; this is a deployment convenience.
 *
 * The scratch lives in a statically sized device array inside libkata of
 * KATA_NOALLOC_SCRATCH_BYTES bytes.  Every GPU that loads the library keeps
 * that array for the life of the process.  The call allocates nothing and
 * frees nothing.  Arguments, layouts and results are those of
 * kata_chunked_forward (same kernels).
 *
 *   - A problem fits when kata_chunked_forward_workspace_bytes(...) <=
 *     KATA_NOALLOC_SCRATCH_BYTES; larger ones return KATA_ERR_WORKSPACE before
 *     anything is launched.
 *   - The scratch of the CURRENT device is used: make the device that owns
 *     the tensors current before the call.
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress) and caches it.  Make that first call before
 *     any stream capture on that device.  The cached address belongs to the
 *     device's context: after cudaDeviceReset() on that device it is stale,
 *     so do not call this entry point on it again in the same process.
 *   - All calls on a device share the one array, and the array keeps what the
 *     last call wrote.  Every scratch element a call reads was first written
 *     by that same call, so nothing needs clearing between calls.  Calls
 *     that can overlap on the GPU (different streams, or several host
 *     threads) race on the array: serialise them.
 */
#define KATA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

kata_status kata_chunked_forward_noalloc(const void *q, const void *k, const void *v, void *out,
                                         int B, int H, int T, int dk, int dv, int C,
                                         kata_dtype dtype, float *state_out, float *z_out,
                                         kata_stream_t stream);

/*
 * KATA-Mg: g rank-one PSD factors per head (gist.science summary 2.3,
 * "Variantes": several PSD factors, trading state size against packing
 * efficiency).  The pages print no formula; the reading implemented (2.1: the
 * admissible cones are products of Koecher-Vinberg factors; 2.2: a projection
 * dimension p per factor) is the product of g rank-one PSD cones, factor m
 * acting on the coordinates [m p, (m+1) p) of q and k, p = dk / g:
 *
 *     w_ts = sum_m (q_t^(m) . k_s^(m))^2,
 *     y_t  = sum_{s<=t} w_ts v_s / sum_{s<=t} w_ts                 (y_t = 0 if 0)
 *
 * The state is the g blocks of p*p x dv (dk^2 / g rows in all): 2 factors
 * halve the state of one.  g = 1 is kata_chunked_forward itself.
 *
 *   kata_mg_chunked_forward: as kata_chunked_forward (same arguments plus g,
 *       same workspace rules with its own size query).  g in {1, 2}: bf16
 *       heads of dk = 64 with g = 2 run the tensor-core path on a layout of the
 *       1056 pairs inside the factors; other head sizes and fp32 run fp32
 *       CUDA-core arithmetic.  Other g: KATA_ERR_UNSUPPORTED.
 *       state_out / z_out: the dense layouts of kata_chunked_forward, holding
 *       zeros at every pair (i, j) whose coordinates lie in different factors.
 *   kata_mg_decode_step: kata_decode_step for g factors on that dense layout:
 *       S[(i,j)] += k_i k_j v and Z[i,j] += k_i k_j only for i, j in one
 *       factor (the other rows stay zero and are neither read nor written),
 *       then y = phi(q)^T S / (q^T Z q).  g in {1, 2}.
 */
size_t kata_mg_chunked_forward_workspace_bytes(int B, int H, int T, int dk, int dv, int C, int g,
                                               kata_dtype dtype);
kata_status kata_mg_chunked_forward(const void *q, const void *k, const void *v, void *out, int B,
                                    int H, int T, int dk, int dv, int C, int g, kata_dtype dtype,
                                    float *state_out, float *z_out, void *workspace,
                                    size_t workspace_bytes, kata_stream_t stream);
kata_status kata_mg_decode_step(const void *q, const void *k, const void *v, void *out,
                                float *state, float *z, int B, int H, int dk, int dv, int g,
                                kata_dtype dtype, kata_stream_t stream);

/*
 * Causal KATA forward in its quadratic form: the flash-attention-style
 * operating point (gist.science summary 2.3, "two operating points", the
 * O(T^2) forward that never forms the state; arXiv abstract,
 * "flash-attention-style forward").
 *
 * Same y_t as kata_chunked_forward, computed from the T x T causal weights
 * (q_t.k_s)^2 in tiles that never leave the chip; no state is formed, so
 * nothing is exported and no workspace is needed.  Work grows as T^2: the
 * chunked form is the one to use for long sequences, this one for short
 * ones and as an independent check of the chunked form.
 *
 *   q, k   [B, H, T, dk]  dtype      queries, keys
 *   v      [B, H, T, dv]  dtype      values
 *   out    [B, H, T, dv]  dtype      y_t as defined at the top of this file
 *
 * dtype KATA_BF16 with dk = 64 runs the tensor-core (tcgen05) path; other
 * cases run fp32 CUDA-core arithmetic.  Errors as in the general contract;
 * B * H * ceil(T / 256) must stay below 2^31 (else KATA_ERR_UNSUPPORTED).
 */
kata_status kata_quadratic_forward(const void *q, const void *k, const void *v, void *out, int B,
                                   int H, int T, int dk, int dv, kata_dtype dtype,
                                   kata_stream_t stream);

/*
 * One recurrent decode step for every head, in place
 * (arXiv abstract, "constant-time recurrent inference"; gist.science summary
 * 1: a fixed-size state replaces the key-value cache):
 *
 *     S <- S + phi(k) v^T,   Z <- Z + k k^T,   y = phi(q)^T S / (q^T Z q)
 *
 * The readout includes the current token, so a forward over T tokens
 * followed by a decode step on token T gives row T of a forward over T + 1
 * tokens.
 *
 *   q, k   [B, H, dk]  dtype;  v, out  [B, H, dv]  dtype
 *   state  [B, H, dk*dk, dv] fp32, read and updated in place
 *   z      [B, H, dk, dk] fp32, read and updated in place
 *
 * The state must be symmetric in (i, j), as every state the forward writes
 * is; the update keeps it symmetric.
 */
kata_status kata_decode_step(const void *q, const void *k, const void *v, void *out,
                             float *state, float *z, int B, int H, int dk, int dv,
                             kata_dtype dtype, kata_stream_t stream);

/*
 * Packed state layout for decode.  The state is symmetric in (i, j), so the
 * rows i <= j hold all of it: R = dk(dk+1)/2 rows, i outer, row
 * r(i, j) = i*dk - i(i-1)/2 + (j - i), each the plain sum over tokens of
 * k_i k_j v (state) or k_i k_j (normaliser); the readout weighs row (i, j) by
 * 2 q_i q_j off the diagonal and q_i^2 on it, which gives the same
 * phi(q)^T S = sum_{i,j} q_i q_j S_ij (gist.science summary 2.2: the weight
 * is the squared inner product, symmetric in the feature indices).  Half the
 * bytes of the dense layout, so the HBM-bound decode step moves half the data.
 *
 *   state_p  [B, H, R, dv] fp32      z_p  [B, H, R] fp32
 *
 * kata_state_pack converts a dense state (as the forward exports it) into
 * this layout, reading the rows i <= j; kata_state_unpack writes both (i, j)
 * and (j, i) of the dense layout from row r(i, j).  Sources and destinations
 * must not overlap.  kata_decode_step_packed is kata_decode_step on this
 * layout: same arguments, same results up to fp32 summation order.
 */
kata_status kata_state_pack(const float *state, const float *z, float *state_p, float *z_p, int B,
                            int H, int dk, int dv, kata_stream_t stream);
kata_status kata_state_unpack(const float *state_p, const float *z_p, float *state, float *z,
                              int B, int H, int dk, int dv, kata_stream_t stream);
kata_status kata_decode_step_packed(const void *q, const void *k, const void *v, void *out,
                                    float *state_p, float *z_p, int B, int H, int dk, int dv,
                                    kata_dtype dtype, kata_stream_t stream);

/*
 * Synchronises `stream`, returns and clears the device status word that
 * kernels set when an on-device check fails (KATA_OK if none did), or
 * KATA_ERR_CUDA if the synchronisation itself reports an error.
 */
kata_status kata_get_device_status(kata_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KATA_H_ */
