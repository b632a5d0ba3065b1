"""GPU parity of KATA-Mg (two rank-one PSD factors) against the fp64 oracle.

KATA-Mg (gist.science summary, Technical summary 2.3, "Variantes") in the
reading of the oracle (oracle/kata_oracle.c): factor m acts on coordinates
[m p, (m + 1) p), p = dk / 2, and the weight is sum_m (q^(m).k^(m))^2.  The
calls go through the C ABI (kata_mg_chunked_forward, kata_mg_decode_step) and
are compared with the oracle's Mg functions on the same input bits, with the
bars of the other parity tests (tests/gpu_util.py).  bf16 heads of d = 64 run
the tensor-core kernels on the two-factor layout; fp32 and the smaller bf16
heads run the CUDA-core path.
"""
from __future__ import annotations

import numpy as np
import pytest

from kernelized_linear_attention_fwd_b200 import inputs
from tests.gpu_util import TOL, assert_state_close, from_device, row_err, sample_rows, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # collected on CPU machines, run only with a GPU
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import kernelized_linear_attention_fwd_b200 as K  # noqa: E402
from kernelized_linear_attention_fwd_b200.csrc import build as kbuild  # noqa: E402

G = 2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()
    K.load_library()
    yield
    assert K.kata_get_device_status() == 0


def dev(x, dtype):
    return to_device(np.ascontiguousarray(x), dtype)


def run_mg(q, k, v, dtype, C=64, want_state=False):
    B, H, T, d = q.shape
    so = zo = None
    if want_state:
        so = torch.empty((B, H, d * d, d), dtype=torch.float32, device="cuda")
        zo = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    out = K.kata_mg_chunked_forward(dev(q, dtype), dev(k, dtype), dev(v, dtype), g=G, C=C,
                                    state_out=so, z_out=zo)
    torch.cuda.synchronize()
    return from_device(out), so, zo


def widen_all(dtype, *xs):
    return tuple(inputs.widen(x, dtype) for x in xs)


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("bf16", 32), ("bf16", 16), ("f32", 64),
                                     ("f32", 32), ("f32", 16)])
@pytest.mark.parametrize("T", [1, 2, 63, 257, 1000, 2049, 3 * 1024 + 77])
def test_full_oracle_ragged_lengths(oracle_mod, dtype, d, T):
    q, k, v = inputs.make_qkv(1, 2, T, d, d, dtype, seed=5 * T + d)
    y, _, _ = run_mg(q, k, v, dtype)
    yref = oracle_mod.forward_mg(*widen_all(dtype, q, k, v), G)
    err = row_err(y, yref)
    assert err <= TOL[dtype], f"row-normwise error {err:.3e}"


def test_differs_from_one_factor(oracle_mod):
    # the two-factor weight is a different method: the M1 oracle must not match
    q, k, v = inputs.make_qkv(1, 2, 3000, 64, 64, "bf16", seed=3)
    y, _, _ = run_mg(q, k, v, "bf16")
    q64, k64, v64 = widen_all("bf16", q, k, v)
    assert row_err(y, oracle_mod.forward_mg(q64, k64, v64, G)) <= TOL["bf16"]
    assert row_err(y, oracle_mod.forward(q64, k64, v64)) > 10 * TOL["bf16"]


@pytest.mark.parametrize("dtype,d,T", [("bf16", 64, 2500), ("bf16", 64, 5000), ("f32", 32, 1500),
                                       ("bf16", 16, 700)])
def test_state_export(oracle_mod, dtype, d, T):
    q, k, v = inputs.make_qkv(1, 3, T, d, d, dtype, seed=d + T)
    _, so, zo = run_mg(q, k, v, dtype, want_state=True)
    Sg, Zg = from_device(so), from_device(zo)
    k64, v64 = widen_all(dtype, k, v)
    assert_state_close(oracle_mod, Sg, Zg, k64, v64, dtype, g=G)
    # pairs across the factors hold exactly zero
    p = d // G
    cross = (np.arange(d)[:, None] // p) != (np.arange(d)[None, :] // p)
    assert np.all(Zg[..., cross] == 0.0)
    assert np.all(Sg.reshape(1, 3, d, d, d)[:, :, cross, :] == 0.0)


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 32), ("bf16", 16)])
def test_forward_then_decode_steps(oracle_mod, dtype, d):
    """forward(T) + n Mg decode steps == rows T..T+n-1 of the Mg forward of T + n."""
    T, n = 1100, 6
    q, k, v = inputs.make_qkv(2, 2, T + n, d, d, dtype, seed=300 + d)
    _, so, zo = run_mg(q[:, :, :T], k[:, :, :T], v[:, :, :T], dtype, want_state=True)
    ys = []
    for s in range(n):
        xs = [dev(x[:, :, T + s], dtype) for x in (q, k, v)]
        ys.append(from_device(K.kata_mg_decode_step(*xs, so, zo, g=G)))
    torch.cuda.synchronize()
    q64, k64, v64 = widen_all(dtype, q, k, v)
    yref = oracle_mod.forward_mg(q64, k64, v64, G)[:, :, T:]
    assert row_err(np.stack(ys, axis=2), yref) <= TOL[dtype]
    # the state after the steps is the Mg state of all T + n tokens, zeros across factors
    assert_state_close(oracle_mod, from_device(so), from_device(zo), k64, v64, dtype, g=G)


@pytest.mark.parametrize("T", [32768, 131072])
def test_long_sequences_sampled(oracle_mod, T):
    H = 2 if T == 32768 else 8
    q, k, v = inputs.make_qkv(1, H, T, 64, 64, "bf16", seed=T + 1)
    y, _, _ = run_mg(q, k, v, "bf16")
    rows = sample_rows(T, 64, 1024, n_uniform=192 if T > 32768 else 384, n_bound=32)
    bh = np.repeat(np.arange(H), len(rows))
    tt = np.tile(rows, H)
    q64, k64, v64 = (inputs.widen(x, "bf16").reshape(H, T, -1) for x in (q, k, v))
    yref = oracle_mod.forward_mg_rows(q64, k64, v64, G, bh, tt)
    err = row_err(y.reshape(H, T, -1)[bh, tt], yref)
    assert err <= TOL["bf16"], f"row-normwise error {err:.3e}"


@pytest.mark.parametrize("T", [600, 2500])
def test_many_heads_every_cta_walks_several_items(oracle_mod, T):
    B, H = 2, 80
    q, k, v = inputs.make_qkv(B, H, T, 64, 64, "bf16", seed=T + 9)
    y, _, _ = run_mg(q, k, v, "bf16")
    rows = np.unique(np.concatenate([np.arange(0, T, 7), [T - 1]]))
    BH = B * H
    bh = np.repeat(np.arange(BH), len(rows))
    tt = np.tile(rows, BH)
    q64, k64, v64 = (inputs.widen(x, "bf16").reshape(BH, T, -1) for x in (q, k, v))
    yref = oracle_mod.forward_mg_rows(q64, k64, v64, G, bh, tt)
    assert row_err(y.reshape(BH, T, -1)[bh, tt], yref) <= TOL["bf16"]


@pytest.mark.parametrize("C", [512, 2048])
def test_chunk_sizes_that_set_the_segment(oracle_mod, C):
    T = 9000
    q, k, v = inputs.make_qkv(1, 2, T, 64, 64, "bf16", seed=C)
    y, _, _ = run_mg(q, k, v, "bf16", C=C)
    rows = sample_rows(T, 64, C, n_uniform=256, n_bound=32)
    bh = np.repeat(np.arange(2), len(rows))
    tt = np.tile(rows, 2)
    q64, k64, v64 = (inputs.widen(x, "bf16").reshape(2, T, -1) for x in (q, k, v))
    yref = oracle_mod.forward_mg_rows(q64, k64, v64, G, bh, tt)
    assert row_err(y.reshape(2, T, -1)[bh, tt], yref) <= TOL["bf16"]


@pytest.mark.parametrize("qk", ["raw", "spread"])
@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 64)])
def test_unnormalised_inputs(oracle_mod, qk, dtype, d):
    q, k, v = inputs.make_qkv(1, 2, 2 * 1024 + 301, d, d, dtype, seed=41, qk=qk)
    y, so, zo = run_mg(q, k, v, dtype, want_state=True)
    q64, k64, v64 = widen_all(dtype, q, k, v)
    assert row_err(y, oracle_mod.forward_mg(q64, k64, v64, G)) <= TOL[dtype]
    assert_state_close(oracle_mod, from_device(so), from_device(zo), k64, v64, dtype, g=G)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zero_denominator_rows(oracle_mod, dtype):
    q, k, v = inputs.make_qkv(1, 2, 1500, 64, 64, dtype, seed=4)
    zero = inputs.f32_to_bf16_bits(np.zeros(1, np.float32))[0] if dtype == "bf16" else 0.0
    for t in (0, 5, 1024, 1499):
        q[0, 0, t] = zero
    y, _, _ = run_mg(q, k, v, dtype)
    for t in (0, 5, 1024, 1499):
        assert np.all(y[0, 0, t] == 0.0), t
    assert row_err(y, oracle_mod.forward_mg(*widen_all(dtype, q, k, v), G)) <= TOL[dtype]


def test_one_factor_is_the_plain_forward(oracle_mod):
    q, k, v = inputs.make_qkv(1, 2, 2500, 64, 64, "bf16", seed=12)
    qd, kd, vd = (dev(x, "bf16") for x in (q, k, v))
    a = from_device(K.kata_mg_chunked_forward(qd, kd, vd, g=1))
    b = from_device(K.kata_chunked_forward(qd, kd, vd))
    assert row_err(a, b) <= 2.0 ** -7
    assert row_err(a, oracle_mod.forward(*widen_all("bf16", q, k, v))) <= TOL["bf16"]


def test_unsupported_factor_counts_are_refused():
    x = torch.zeros((1, 1, 64, 64), dtype=torch.bfloat16, device="cuda")
    for g in (3, 4):
        with pytest.raises(K.KataError) as e:
            K.kata_mg_chunked_forward(x, x, x, g=g)
        assert e.value.status == 2  # KATA_ERR_UNSUPPORTED
