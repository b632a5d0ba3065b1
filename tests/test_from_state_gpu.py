"""GPU parity of the state-only call, the forward from a given state, and the
sequence-sharded forward, against the fp64 oracle.

- kata_chunked_state against the oracle's state by direct summation.
- kata_chunked_forward_from_state: a history of tokens, then a block; the
  block's outputs must equal the rows of the oracle's quadratic forward of the
  whole sequence, whether the history's state is given as one input, as the
  sum of several stacked inputs, or carried piece by piece in place.
- The sequence-sharded forward with its ranks emulated one after another on
  this GPU (every rank's kernels are independent; the all-gather becomes a
  stack of the ranks' flat totals in the layout the collective produces).
Tolerances: tests/gpu_util.py.
"""
from __future__ import annotations

import numpy as np
import pytest

from kernelized_linear_attention_fwd_b200 import inputs
from tests.gpu_util import (TOL, assert_state_close, from_device, row_err, sample_rows,
                            to_device)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # collected on CPU machines, run only with a GPU
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import kernelized_linear_attention_fwd_b200 as K  # noqa: E402
from kernelized_linear_attention_fwd_b200 import sharded  # noqa: E402
from kernelized_linear_attention_fwd_b200.csrc import build as kbuild  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()
    K.load_library()
    yield
    assert K.kata_get_device_status() == 0


def dev(x, dtype):
    return to_device(np.ascontiguousarray(x), dtype)


def f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def check_state(oracle_mod, Sg, Zg, k64, v64, dtype):
    assert_state_close(oracle_mod, from_device(Sg), from_device(Zg), k64, v64, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d,T", [(16, 1), (16, 700), (32, 1500), (64, 63), (64, 3000)])
def test_state_only(oracle_mod, dtype, d, T):
    q, k, v = inputs.make_qkv(2, 2, T, d, d, dtype, seed=7 * T + d)
    S, Z = K.kata_chunked_state(dev(k, dtype), dev(v, dtype), C=64)
    torch.cuda.synchronize()
    k64, v64 = inputs.widen(k, dtype), inputs.widen(v, dtype)
    check_state(oracle_mod, S, Z, k64, v64, dtype)
    # the state the forward exports, within the same bound (not bitwise: on the
    # tensor-core path two MMA issuers add into one accumulator in issue order)
    so = torch.full_like(S, float("nan"))  # an entry left unwritten fails the check
    zo = torch.full_like(Z, float("nan"))
    K.kata_chunked_forward(dev(q, dtype), dev(k, dtype), dev(v, dtype), C=64, state_out=so,
                           z_out=zo)
    torch.cuda.synchronize()
    check_state(oracle_mod, so, zo, k64, v64, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64])
@pytest.mark.parametrize("Th,Tb", [(1, 1), (300, 100), (1000, 2049), (2500, 1500)])
def test_forward_from_one_state(oracle_mod, dtype, d, Th, Tb):
    q, k, v = inputs.make_qkv(1, 3, Th + Tb, d, d, dtype, seed=Th + 3 * Tb + d)
    q64, k64, v64 = (inputs.widen(x, dtype) for x in (q, k, v))
    S0, Z0 = oracle_mod.state(k64[:, :, :Th], v64[:, :, :Th])
    so = torch.full((1, 3, d * d, d), float("nan"), dtype=torch.float32, device="cuda")
    zo = torch.full((1, 3, d, d), float("nan"), dtype=torch.float32, device="cuda")
    blk = [dev(x[:, :, Th:], dtype) for x in (q, k, v)]
    out = K.kata_chunked_forward_from_state(*blk, f32(S0), f32(Z0), C=64, state_out=so, z_out=zo)
    torch.cuda.synchronize()
    yref = oracle_mod.forward(q64, k64, v64)[:, :, Th:]
    err = row_err(from_device(out), yref)
    assert err <= TOL[dtype], f"row-normwise error {err:.3e}"
    check_state(oracle_mod, so, zo, k64, v64, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64])
def test_inputs_are_summed(oracle_mod, dtype, d):
    # the history's state given as the states of three pieces, stacked
    cuts = (0, 400, 1300, 2000)
    Tb = 1200
    q, k, v = inputs.make_qkv(2, 2, cuts[-1] + Tb, d, d, dtype, seed=d + 1)
    q64, k64, v64 = (inputs.widen(x, dtype) for x in (q, k, v))
    parts = [oracle_mod.state(k64[:, :, a:b], v64[:, :, a:b]) for a, b in zip(cuts, cuts[1:])]
    S_in = f32(np.stack([p[0] for p in parts]))
    Z_in = f32(np.stack([p[1] for p in parts]))
    blk = [dev(x[:, :, cuts[-1]:], dtype) for x in (q, k, v)]
    out = K.kata_chunked_forward_from_state(*blk, S_in, Z_in, C=64)
    torch.cuda.synchronize()
    yref = oracle_mod.forward(q64, k64, v64)[:, :, cuts[-1]:]
    assert row_err(from_device(out), yref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,d", [("f32", 32), ("bf16", 64)])
def test_no_inputs_is_the_plain_forward(oracle_mod, dtype, d):
    q, k, v = inputs.make_qkv(1, 2, 2500, d, d, dtype, seed=9)
    qd, kd, vd = (dev(x, dtype) for x in (q, k, v))
    empty_s = torch.empty((0, 1, 2, d * d, d), dtype=torch.float32, device="cuda")
    empty_z = torch.empty((0, 1, 2, d, d), dtype=torch.float32, device="cuda")
    a = from_device(K.kata_chunked_forward_from_state(qd, kd, vd, empty_s, empty_z, C=64))
    b = from_device(K.kata_chunked_forward(qd, kd, vd, C=64))
    # the same kernels; on the tensor-core path the fp32 sums may differ in order
    # (two MMA issuers into one accumulator), so up to one bf16 rounding apart
    assert row_err(a, b) <= (0.0 if dtype == "f32" else 2.0 ** -7)
    yref = oracle_mod.forward(*(inputs.widen(x, dtype) for x in (q, k, v)))
    assert row_err(a, yref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 64])
def test_pieces_in_place(oracle_mod, dtype, d):
    # a long prompt processed in pieces, the state updated in place between them
    cuts = (0, 1, 500, 1524, 3100, 3101)
    q, k, v = inputs.make_qkv(1, 2, cuts[-1], d, d, dtype, seed=40 + d)
    S = torch.zeros((1, 2, d * d, d), dtype=torch.float32, device="cuda")
    Z = torch.zeros((1, 2, d, d), dtype=torch.float32, device="cuda")
    ys = []
    for a, b in zip(cuts, cuts[1:]):
        blk = [dev(x[:, :, a:b], dtype) for x in (q, k, v)]
        ys.append(from_device(K.kata_chunked_forward_from_state(*blk, S, Z, C=64, state_out=S,
                                                                z_out=Z)))
    torch.cuda.synchronize()
    q64, k64, v64 = (inputs.widen(x, dtype) for x in (q, k, v))
    assert row_err(np.concatenate(ys, axis=2), oracle_mod.forward(q64, k64, v64)) <= TOL[dtype]
    check_state(oracle_mod, S, Z, k64, v64, dtype)


def emulated_sharded(q, k, v, bounds, dtype, C=64, reuse=True):
    """The sequence-sharded forward with its ranks run one after another, each
    keeping its own workspace from the state pass to the forward."""
    blocks = [[dev(x[:, :, a:b], dtype) for x in (q, k, v)] for a, b in zip(bounds, bounds[1:])]
    wss = [sharded.LibkataOps.workspace(bk, bv, C) for _, bk, bv in blocks]
    flats = [sharded.block_state(bk, bv, C, workspace=ws) for (_, bk, bv), ws in zip(blocks, wss)]
    gathered = torch.stack(flats)  # the all-gather's [world, |S| + |Z|] layout
    B, H, _, d = q.shape
    outs, states = [], []
    for r, (bq, bk, bv) in enumerate(blocks):
        so = torch.empty((B, H, d * d, d), dtype=torch.float32, device="cuda")
        zo = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
        outs.append(sharded.block_forward(bq, bk, bv, gathered, r, C, state_out=so, z_out=zo,
                                          workspace=wss[r], reuse=reuse))
        states.append((so, zo))
    torch.cuda.synchronize()
    return np.concatenate([from_device(o) for o in outs], axis=2), states


@pytest.mark.parametrize("dtype,d,bounds", [
    ("f32", 32, (0, 700, 1400, 2900)),
    ("bf16", 64, (0, 1024, 2048, 3000, 4100)),
    ("bf16", 64, (0, 1, 1500, 1501, 2600)),
    # small heads: the two-factor state layout, its segment states reused
    ("bf16", 32, (0, 1024, 2048, 3000, 4100)),
    ("bf16", 16, (0, 700, 1500, 2600)),
])
def test_sequence_sharded_ranks_emulated(oracle_mod, dtype, d, bounds):
    q, k, v = inputs.make_qkv(1, 2, bounds[-1], d, d, dtype, seed=len(bounds) + d)
    y, states = emulated_sharded(q, k, v, bounds, dtype)
    q64, k64, v64 = (inputs.widen(x, dtype) for x in (q, k, v))
    assert row_err(y, oracle_mod.forward(q64, k64, v64)) <= TOL[dtype]
    for r, (so, zo) in enumerate(states):  # each rank's state: after its block
        n = bounds[r + 1]
        check_state(oracle_mod, so, zo, k64[:, :, :n], v64[:, :, :n], dtype)


@pytest.mark.parametrize("dtype,d", [("f32", 32), ("bf16", 64), ("bf16", 32)])
def test_reused_segment_states_match_rebuilt(oracle_mod, dtype, d):
    # the forward after the state pass, with and without the reuse flag
    bounds = (0, 1500, 3600)
    q, k, v = inputs.make_qkv(1, 2, bounds[-1], d, d, dtype, seed=77 + d)
    y1, s1 = emulated_sharded(q, k, v, bounds, dtype, reuse=True)
    y0, s0 = emulated_sharded(q, k, v, bounds, dtype, reuse=False)
    q64, k64, v64 = (inputs.widen(x, dtype) for x in (q, k, v))
    yref = oracle_mod.forward(q64, k64, v64)
    assert row_err(y1, yref) <= TOL[dtype] and row_err(y0, yref) <= TOL[dtype]
    assert row_err(y1, y0) <= (1e-6 if dtype == "f32" else 2.0 ** -7)
    check_state(oracle_mod, *s1[-1], k64, v64, dtype)


def test_sequence_sharded_long_context(oracle_mod):
    # the long-context workload's sequence over 8 emulated ranks, sampled rows
    w = inputs.WORKLOADS["long_B1H8_T131072_d64_bf16"]
    q, k, v = inputs.make_workload(w)
    T = w.T
    bounds = tuple(range(0, T + 1, T // 8))
    y, _ = emulated_sharded(q, k, v, bounds, "bf16", C=w.C)
    rows = sample_rows(T, w.C, T // 8, n_uniform=128, n_bound=16)
    BH = w.B * w.H
    bh = np.repeat(np.arange(BH), len(rows))
    tt = np.tile(rows, BH)
    q64, k64, v64 = (inputs.widen(x, "bf16").reshape(BH, T, -1) for x in (q, k, v))
    yref = oracle_mod.forward_rows(q64, k64, v64, bh, tt)
    err = row_err(y.reshape(BH, T, -1)[bh, tt], yref)
    assert err <= TOL["bf16"], f"row-normwise error {err:.3e}"


@pytest.mark.parametrize("d", [16, 32, 64])
def test_short_history_error_bound(oracle_mod, d):
    """A history of one or a few tokens: the inter term phi(q) . S is a sum of
    c_ij q_i q_j S_ij,e over the pairs, formed from bf16 products and a bf16
    state prefix, so its rounding error scales with sum_s (sum_i |q_i k_s,i|)^2
    |v_s,e|, not with the term sum_s (q . k_s)^2 v_s,e itself.  Where the few
    history keys are nearly orthogonal to the query and carry most of a row's
    small weight, the row's relative error can exceed the 2e-2 tolerance (the
    plain forward has no inter term there).  Checked: every row stays within
    the tolerance plus that term's worst-case bound over the row's
    denominator, and rows whose bound is small meet the tolerance itself."""
    U = 2.0 ** -8  # bf16 rounding of the products and of the state prefix
    worst_plain = 0.0
    for seed in range(4):
        for Th in (1, 3):
            Tb = 200
            q, k, v = inputs.make_qkv(1, 2, Th + Tb, d, d, "bf16", seed=100 * d + 10 * seed + Th)
            q64, k64, v64 = (inputs.widen(x, "bf16") for x in (q, k, v))
            yref = oracle_mod.forward(q64, k64, v64)[:, :, Th:]
            S0, Z0 = oracle_mod.state(k64[:, :, :Th], v64[:, :, :Th])
            y = from_device(K.kata_chunked_forward_from_state(
                *(dev(x[:, :, Th:], "bf16") for x in (q, k, v)), f32(S0), f32(Z0), C=64))
            qb, kh, vh = q64[:, :, Th:], k64[:, :, :Th], v64[:, :, :Th]
            # per row t: den_t and the inter term's bound sum_s (sum_i |q_i k_s,i|)^2 |v_s,e|
            scores = np.einsum("bhtd,bhsd->bhts", q64, k64)
            causal = np.tril(np.ones((Th + Tb, Th + Tb)))[Th:]
            den = np.einsum("bhts,ts->bht", scores[:, :, Th:] ** 2, causal)
            absq = np.einsum("bhtd,bhsd->bhts", np.abs(qb), np.abs(kh)) ** 2
            bound = U * np.einsum("bhts,bhse->bhte", absq, np.abs(vh)).max(-1) / den
            err = np.abs(y - yref).max(-1)
            scale = np.abs(yref).max(-1)
            assert np.all(err <= TOL["bf16"] * scale + bound), \
                f"d={d} Th={Th} seed={seed}: an error beyond the tolerance and the inter-term bound"
            calm = bound <= 1e-3 * scale  # the inter term cannot move these rows
            if calm.any():
                worst_plain = max(worst_plain, float((err[calm] / scale[calm]).max()))
    assert worst_plain <= TOL["bf16"]
