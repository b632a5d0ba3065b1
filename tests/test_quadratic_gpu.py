"""GPU parity of the quadratic (flash-attention-style) forward against the fp64 oracle.

kata_quadratic_forward computes the same y_t as the chunked form from the
T x T causal weights, with no state.  The oracle's `forward` is the definition
itself, so it is the reference here too; the tolerances are those of the
chunked form (tests/gpu_util.py).  Long sequences are checked on sampled rows
(first and last 64, both sides of seeded 64-token boundaries, seeded uniform
rows), and against the chunked form on the same inputs.
"""
from __future__ import annotations

import numpy as np
import pytest

from kernelized_linear_attention_fwd_b200 import inputs
from tests.gpu_util import TOL, from_device, row_err, sample_rows, to_device

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


def run_quadratic(q, k, v, dtype):
    out = K.kata_quadratic_forward(to_device(q, dtype), to_device(k, dtype), to_device(v, dtype))
    torch.cuda.synchronize()
    return from_device(out)


def sampled_check(oracle_mod, q, k, v, dtype, rows):
    B, H, T, _ = q.shape
    BH = B * H
    q64, k64, v64 = (inputs.widen(x, dtype).reshape(BH, T, -1) for x in (q, k, v))
    bh = np.repeat(np.arange(BH), len(rows))
    tt = np.tile(rows, BH)
    yref = oracle_mod.forward_rows(q64, k64, v64, bh, tt)
    y = run_quadratic(q, k, v, dtype).reshape(BH, T, -1)
    err = row_err(y[bh, tt], yref)
    assert err <= TOL[dtype], f"row-normwise error {err:.3e}"
    return y


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 2, 63, 129, 257, 1000, 2049])
def test_ragged_lengths_all_head_sizes(oracle_mod, dtype, d, T):
    q, k, v = inputs.make_qkv(1, 2, T, d, d, dtype, seed=3 * T + d)
    y = run_quadratic(q, k, v, dtype)
    yref = oracle_mod.forward(inputs.widen(q, dtype), inputs.widen(k, dtype),
                              inputs.widen(v, dtype))
    err = row_err(y, yref)
    assert err <= TOL[dtype], f"row-normwise error {err:.3e}"


@pytest.mark.parametrize("T", [600, 1152, 2500])
def test_many_heads_longest_items_first(oracle_mod, T):
    # More 256-query work items than streaming multiprocessors: every CTA
    # walks several items of different heads, latest queries first, with
    # ragged tails and (T = 1152) an empty second query tile.
    q, k, v = inputs.make_qkv(2, 80, T, 64, 64, "bf16", seed=T + 7)
    sampled_check(oracle_mod, q, k, v, "bf16", np.unique(np.r_[np.arange(0, T, 7), T - 1]))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_long_single_segment(oracle_mod, dtype):
    # 16384 keys for the last queries, far past the chunked form's 1024-token segments
    T = 16384
    q, k, v = inputs.make_qkv(1, 4, T, 64, 64, dtype, seed=21)
    sampled_check(oracle_mod, q, k, v, dtype, sample_rows(T, 64, T, n_uniform=128))


def test_lm340m_layer_matches_oracle_and_chunked_form(oracle_mod):
    w = inputs.WORKLOADS["lm340m_B4H16_T16384_d64_bf16"]
    q, k, v = inputs.make_workload(w)
    y = sampled_check(oracle_mod, q, k, v, "bf16", sample_rows(w.T, w.C, 1024, n_uniform=64))
    yc = K.kata_chunked_forward(to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"),
                                C=w.C)
    torch.cuda.synchronize()
    # two bf16 results of the same exact quantity: each within TOL of it
    err = row_err(y, from_device(yc).reshape(y.shape))
    assert err <= 2 * TOL["bf16"], f"quadratic vs chunked: {err:.3e}"


def test_long_context_sampled(oracle_mod):
    # the longest sequence of the long-context workload, in the quadratic form
    w = inputs.WORKLOADS["long_B1H8_T131072_d64_bf16"]
    q, k, v = inputs.make_workload(w)
    sampled_check(oracle_mod, q, k, v, "bf16", sample_rows(w.T, 64, w.T, n_uniform=64, n_bound=16))


def test_maximum_length_single_head(oracle_mod):
    # 2^20 keys for the last queries of one head: 4096 work items, one segment
    T = 1 << 20
    q, k, v = inputs.make_qkv(1, 1, T, 64, 64, "bf16", seed=23)
    sampled_check(oracle_mod, q, k, v, "bf16", sample_rows(T, 64, T, n_uniform=48, n_bound=16))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zero_denominator_rows(oracle_mod, dtype):
    for d in (32, 64):
        q, k, v = inputs.make_qkv(1, 2, 700, d, d, dtype, seed=5 + d)
        zero = inputs.f32_to_bf16_bits(np.zeros(1, np.float32))[0] if dtype == "bf16" else 0.0
        for t in (0, 64, 255, 256, 699):
            q[0, 0, t] = zero
        y = run_quadratic(q, k, v, dtype)
        for t in (0, 64, 255, 256, 699):
            assert np.all(y[0, 0, t] == 0.0), (d, t)
        yref = oracle_mod.forward(inputs.widen(q, dtype), inputs.widen(k, dtype),
                                  inputs.widen(v, dtype))
        assert row_err(y, yref) <= TOL[dtype]
