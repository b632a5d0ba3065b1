"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Inputs are the seeded generator's bits (kernelized_linear_attention_fwd_b200
/inputs.py); the oracle widens exactly those bits to fp64.  The metric and
tolerances are in tests/gpu_util.py (row-normwise relative error, 1e-4 for
fp32 inputs, 2e-2 for bf16 inputs).
"""
from __future__ import annotations

import numpy as np
import pytest

from kernelized_linear_attention_fwd_b200 import inputs
from tests.gpu_util import (TOL, assert_state_close, from_device, row_err, sample_rows,
                            state_bounds, to_device)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # collected on CPU machines, run only with a GPU
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import kernelized_linear_attention_fwd_b200 as K  # noqa: E402
from kernelized_linear_attention_fwd_b200.csrc import build as kbuild  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()
    K.load_library()
    yield
    assert K.kata_get_device_status() == 0


def seg_len(d, C, dtype="bf16"):
    """Tokens between stored states: C itself for C >= 512, else a fixed
    length: 1024 on the tensor cores (bf16, every head size), per head size on
    the fp32 path (include/kata.h, argument C)."""
    if C >= 512:
        return C
    if dtype == "bf16":
        return 1024
    return 1024 if d >= 64 else (512 if d >= 32 else 256)


def run_forward(q, k, v, dtype, C, want_state=False):
    qd, kd, vd = to_device(q, dtype), to_device(k, dtype), to_device(v, dtype)
    B, H, T, dk = q.shape
    so = zo = None
    if want_state:
        # NaN-filled, so an entry the export does not write fails the comparison
        so = torch.full((B, H, dk * dk, dk), float("nan"), dtype=torch.float32, device="cuda")
        zo = torch.full((B, H, dk, dk), float("nan"), dtype=torch.float32, device="cuda")
    out = K.kata_chunked_forward(qd, kd, vd, C=C, state_out=so, z_out=zo)
    torch.cuda.synchronize()
    return out, so, zo


def full_check(oracle_mod, q, k, v, dtype, C, tol=None):
    out, _, _ = run_forward(q, k, v, dtype, C)
    yref = oracle_mod.forward(inputs.widen(q, dtype), inputs.widen(k, dtype),
                              inputs.widen(v, dtype))
    err = row_err(from_device(out), yref)
    assert err <= (tol or TOL[dtype]), f"row-normwise error {err:.3e} (C={C})"
    return err


# ---------------------------------------------------------------------------
# The named workloads
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("C", [16, 32, 64, 128, 256])
def test_tiny_f32_full(oracle_mod, C):
    w = inputs.WORKLOADS["tiny_B1H1_T256_d16_f32"]
    q, k, v = inputs.make_workload(w)
    full_check(oracle_mod, q, k, v, "f32", C)


def test_small_bf16_full(oracle_mod):
    w = inputs.WORKLOADS["small_B2H4_T4096_d32_bf16"]
    q, k, v = inputs.make_workload(w)
    full_check(oracle_mod, q, k, v, "bf16", w.C)


def _sampled_check(oracle_mod, q, k, v, dtype, Cs, n_uniform=512):
    B, H, T, d = q.shape
    q64, k64, v64 = (inputs.widen(x, dtype).reshape(B * H, T, -1) for x in (q, k, v))
    rows = sample_rows(T, min(Cs), min(seg_len(d, C, dtype) for C in Cs), n_uniform=n_uniform)
    bh = np.repeat(np.arange(B * H), len(rows))
    tt = np.tile(rows, B * H)
    yref = oracle_mod.forward_rows(q64, k64, v64, bh, tt)
    errs = {}
    for C in Cs:
        out, _, _ = run_forward(q, k, v, dtype, C)
        y = from_device(out).reshape(B * H, T, -1)[bh, tt]
        errs[C] = row_err(y, yref)
        assert errs[C] <= TOL[dtype], f"C={C}: row-normwise error {errs[C]:.3e}"
    return errs


def test_lm340m_layer_sampled(oracle_mod):
    w = inputs.WORKLOADS["lm340m_B4H16_T16384_d64_bf16"]
    q, k, v = inputs.make_workload(w)
    _sampled_check(oracle_mod, q, k, v, "bf16", [w.C], n_uniform=128)


@pytest.mark.parametrize("T", [8192, 32768, 131072])
def test_long_context_sampled(oracle_mod, T):
    w = inputs.WORKLOADS["long_B1H8_T131072_d64_bf16"]
    q, k, v = inputs.make_workload(w, T=T)
    Cs = list(w.chunk_sweep) if T == w.T else [w.C]
    _sampled_check(oracle_mod, q, k, v, "bf16", Cs, n_uniform=512 if T == w.T else 256)


@pytest.mark.parametrize("dtype,d,T", [("bf16", 64, 32768), ("bf16", 64, 9000),
                                       ("f32", 64, 5000), ("f32", 32, 5000)])
def test_chunk_sizes_that_set_the_segment(oracle_mod, dtype, d, T):
    # C >= 512 keeps states every C tokens: other segment boundaries, other
    # scan lengths (64 segments at C = 512, T = 32768), longer intra terms
    q, k, v = inputs.make_qkv(1, 2, T, d, d, dtype, seed=T + 5)
    Cs = [512, 1024, 2048, 4096] if T >= 9000 else [512, 2048]
    for C in Cs:
        _sampled_check(oracle_mod, q, k, v, dtype, [C], n_uniform=192)


def test_maximum_length_sampled(oracle_mod):
    # 2^20 tokens per head: 1024 segments, so the scan makes 8 passes of 128
    T = 1 << 20
    q, k, v = inputs.make_qkv(1, 2, T, 64, 64, "bf16", seed=17)
    out, _, _ = run_forward(q, k, v, "bf16", 64)
    rows = sample_rows(T, 64, 1024, n_uniform=48, n_bound=16)
    bh = np.repeat(np.arange(2), len(rows))
    tt = np.tile(rows, 2)
    q64, k64, v64 = (inputs.widen(x, "bf16").reshape(2, T, -1) for x in (q, k, v))
    yref = oracle_mod.forward_rows(q64, k64, v64, bh, tt)
    err = row_err(from_device(out).reshape(2, T, -1)[bh, tt], yref)
    assert err <= TOL["bf16"], f"row-normwise error {err:.3e}"


# ---------------------------------------------------------------------------
# Edge cases
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 2, 63, 257, 1000, 2049])
def test_ragged_lengths_all_head_sizes(oracle_mod, dtype, d, T):
    q, k, v = inputs.make_qkv(1, 2, T, d, d, dtype, seed=T + d)
    full_check(oracle_mod, q, k, v, dtype, 64)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_multi_segment_f32_and_bf16(oracle_mod, dtype):
    # several segments, ragged tail, every chunk size
    q, k, v = inputs.make_qkv(1, 2, 3 * 1024 + 77, 64, 64, dtype, seed=11)
    for C in (16, 64, 256):
        full_check(oracle_mod, q, k, v, dtype, C)


@pytest.mark.parametrize("T", [600, 2500, 1024 + 128])
def test_many_heads_every_cta_walks_several_items(oracle_mod, T):
    # More 256-query work items than streaming multiprocessors, so each
    # persistent readout CTA runs several items back to back (barrier phases
    # and accumulator zeroing carried across items), with ragged tails, an
    # empty second query tile (T = 1152) and single-segment heads (T = 600).
    B, H = 2, 80
    q, k, v = inputs.make_qkv(B, H, T, 64, 64, "bf16", seed=T)
    out, _, _ = run_forward(q, k, v, "bf16", 64)
    rows = np.unique(np.concatenate([np.arange(0, T, 7), [T - 1]]))
    BH = B * H
    bh = np.repeat(np.arange(BH), len(rows))
    tt = np.tile(rows, BH)
    q64, k64, v64 = (inputs.widen(x, "bf16").reshape(BH, T, -1) for x in (q, k, v))
    yref = oracle_mod.forward_rows(q64, k64, v64, bh, tt)
    y = from_device(out).reshape(BH, T, -1)[bh, tt]
    err = row_err(y, yref)
    assert err <= TOL["bf16"], f"row-normwise error {err:.3e}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zero_denominator_rows(oracle_mod, dtype):
    q, k, v = inputs.make_qkv(1, 2, 1500, 32, 32, dtype, seed=3)
    zero = inputs.f32_to_bf16_bits(np.zeros(1, np.float32))[0] if dtype == "bf16" else 0.0
    for t in (0, 5, 511, 512, 1499):
        q[0, 0, t] = zero
    q[0, 1, 700] = zero
    out, _, _ = run_forward(q, k, v, dtype, 64)
    y = from_device(out)
    for (h, t) in [(0, 0), (0, 5), (0, 511), (0, 512), (0, 1499), (1, 700)]:
        assert np.all(y[0, h, t] == 0.0), (h, t)
    yref = oracle_mod.forward(inputs.widen(q, dtype), inputs.widen(k, dtype),
                              inputs.widen(v, dtype))
    assert row_err(y, yref) <= TOL[dtype]


def test_convex_combination_invariant():
    """Every output coordinate lies within [min, max] of the prefix values
    (gist.science summary 2.1, convex output gate), up to bf16 rounding."""
    q, k, v = inputs.make_qkv(2, 2, 4096, 64, 64, "bf16", seed=21)
    out, _, _ = run_forward(q, k, v, "bf16", 64)
    y = from_device(out)
    vv = inputs.widen(v, "bf16")
    lo = np.minimum.accumulate(vv, axis=2)
    hi = np.maximum.accumulate(vv, axis=2)
    slack = 1e-2 * np.maximum(np.abs(lo), np.abs(hi)) + 1e-3
    assert np.all(y >= lo - slack) and np.all(y <= hi + slack)


# ---------------------------------------------------------------------------
# State export and decode
# ---------------------------------------------------------------------------


# state_bounds (tests/gpu_util.py): per-entry bound of an exported state.  For
# bf16 it scales with the expected error of the bf16-rounded products
# (STATE_SIGMAS conservative standard deviations of it, plus the fp32 sums);
# the worst-case bound STATE_BOUND * sum_s |k_si k_sj v_se| is kept as an
# outer check.  tests/test_state_bound.py pins the bound on the CPU from both
# sides (rounded arithmetic passes, a 1% error on one tile fails).


def check_state(oracle_mod, k, v, so, zo, dtype, planted=True):
    """Exported (so, zo) against the oracle's state of the same input bits."""
    B, H, T, d = k.shape
    k64, v64 = inputs.widen(k, dtype), inputs.widen(v, dtype)
    Sg, Zg = from_device(so), from_device(zo)
    # Z = sum k k^T: the tensor-core path forms it from the same bf16-rounded
    # products k_i k_j as the state (one extra operand column of ones), so the
    # same kind of bound applies
    worst = assert_state_close(oracle_mod, Sg, Zg, k64, v64, dtype)
    # symmetric in (i, j), as the decode step requires
    S4 = Sg.reshape(B, H, d, d, d)
    assert np.array_equal(S4, S4.transpose(0, 1, 3, 2, 4))
    if planted:
        # a reference with one tile of 128 state rows off by 1% must fail the check
        S, _ = oracle_mod.state(k64, v64)
        bS, _ = state_bounds(oracle_mod, k64, v64, dtype)
        bad = S.copy()
        bad[..., :128, :] *= 1.01
        assert np.any(np.abs(Sg - bad) > bS), "a 1% error on one state tile would pass"
    return worst


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d,T", [(16, 300), (32, 1500), (64, 2500)])
def test_state_export(oracle_mod, dtype, d, T):
    q, k, v = inputs.make_qkv(1, 3, T, d, d, dtype, seed=d)
    out, so, zo = run_forward(q, k, v, dtype, 64, want_state=True)
    check_state(oracle_mod, k, v, so, zo, dtype)


def test_state_export_long(oracle_mod):
    # 32 segments of 1024 tokens: the bound grows like sqrt(T), as the entries do
    T = 32768
    q, k, v = inputs.make_qkv(1, 1, T, 64, 64, "bf16", seed=64)
    out, so, zo = run_forward(q, k, v, "bf16", 64, want_state=True)
    check_state(oracle_mod, k, v, so, zo, "bf16")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64])
def test_forward_then_decode_steps(oracle_mod, dtype, d):
    """forward(T) + n decode steps == rows T..T+n-1 of forward(T + n)."""
    T, n = 1100, 6
    q, k, v = inputs.make_qkv(2, 2, T + n, d, d, dtype, seed=100 + d)
    _, so, zo = run_forward(q[:, :, :T], k[:, :, :T], v[:, :, :T], dtype, 64, want_state=True)
    ys = []
    for s in range(n):
        qs = to_device(np.ascontiguousarray(q[:, :, T + s]), dtype)
        ks = to_device(np.ascontiguousarray(k[:, :, T + s]), dtype)
        vs = to_device(np.ascontiguousarray(v[:, :, T + s]), dtype)
        ys.append(from_device(K.kata_decode_step(qs, ks, vs, so, zo)))
    torch.cuda.synchronize()
    yd = np.stack(ys, axis=2)
    q64, k64, v64 = (inputs.widen(x, dtype) for x in (q, k, v))
    yref = oracle_mod.forward(q64, k64, v64)[:, :, T:]
    assert row_err(yd, yref) <= TOL[dtype]


def test_recall_decode_workload(oracle_mod):
    """Prefill of 64 x 16 heads over 32768 tokens, then 1024 decode steps whose
    queries repeat the keys of 4096 marked pairs (recall-shaped workload).
    Checked against the oracle: 16 seeded heads at every decode step, plus 64
    seeded prefill rows of each of those heads."""
    w = inputs.WORKLOADS["recall_decode_B64H16_T32768_d64_bf16"]
    B, H, T, d, n = w.B, w.H, w.T, w.d, w.decode_steps
    q, k, v = inputs.make_qkv_device(B, H, T, d, d, seed=w.seed)
    so = torch.empty((B, H, d * d, d), dtype=torch.float32, device="cuda")
    zo = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    out = K.kata_chunked_forward(q, k, v, C=w.C, state_out=so, z_out=zo)
    pair_pos, pick = inputs.recall_decode_plan(w)
    # fresh unit keys and N(0, 1) values for the decode tokens
    _, k_dec, v_dec = inputs.make_qkv_device(B, H, n, d, d, seed=w.seed + 1)
    pos_t = torch.from_numpy(pair_pos[pick]).cuda()  # [n, B, H]
    ys = torch.empty((n, B, H, d), dtype=torch.bfloat16, device="cuda")
    q_dec = torch.empty((n, B, H, d), dtype=torch.bfloat16, device="cuda")
    bidx = torch.arange(B, device="cuda")[:, None].expand(B, H)
    hidx = torch.arange(H, device="cuda")[None, :].expand(B, H)
    for s in range(n):
        q_dec[s] = k[bidx, hidx, pos_t[s]]
        K.kata_decode_step(q_dec[s], k_dec[:, :, s].contiguous(), v_dec[:, :, s].contiguous(),
                           so, zo, out=ys[s])
    torch.cuda.synchronize()
    assert K.kata_get_device_status() == 0

    g = np.random.default_rng(5)
    heads = g.choice(B * H, size=16, replace=False)
    tq, tk, tv = (x.view(B * H, T, d) for x in (q, k, v))
    for hh in heads:
        b, h = divmod(int(hh), H)
        qa = np.concatenate([from_device(tq[hh]), from_device(q_dec[:, b, h])])
        ka = np.concatenate([from_device(tk[hh]), from_device(k_dec[b, h])])
        va = np.concatenate([from_device(tv[hh]), from_device(v_dec[b, h])])
        rows = np.concatenate([np.arange(T, T + n), g.integers(0, T, size=64)])
        yref = oracle_mod.forward_rows(qa[None], ka[None], va[None], np.zeros_like(rows), rows)
        ydec = from_device(ys[:, b, h])
        ypre = from_device(out[b, h])[rows[n:]]
        assert row_err(ydec, yref[:n]) <= TOL["bf16"], f"decode head {hh}"
        assert row_err(ypre, yref[n:]) <= TOL["bf16"], f"prefill head {hh}"
