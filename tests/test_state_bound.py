"""The exported-state bound of the bf16 parity tests, checked on the CPU.

The tensor-core path rounds every product k_i k_j of two bf16 key entries to
bf16 (round to nearest even) and sums the products times v in fp32.  Here that
rounding is reproduced in numpy (the product of two bf16 values is exact in
fp32, then rounded to bf16 on its bit pattern) with the sums kept in fp64, and
the result is compared with the fp64 oracle's state under the bound the GPU
tests enforce (tests/gpu_util.py): the rounded state must pass with room to
spare, and a state with one tile of entries off by 1% must fail.  This pins
the bound from both sides without a GPU: it is neither so tight that correct
bf16 arithmetic fails it nor so loose that a small state error passes.
"""
import numpy as np
import pytest

from kernelized_linear_attention_fwd_b200 import inputs
from tests.gpu_util import U_BF16, state_bounds


def rounded_product_state(k64, v64):
    """S[i*d+j, e] = sum_s bf16(k_si k_sj) v_se and Z[i, j] = sum_s bf16(k_si k_sj),
    the products rounded as the tensor-core path rounds them, the sums in fp64."""
    H, T, d = k64.shape
    S = np.empty((H, d * d, v64.shape[-1]))
    Z = np.empty((H, d, d))
    for h in range(H):
        p32 = (k64[h][:, :, None] * k64[h][:, None, :]).astype(np.float32)  # exact in fp32
        p = inputs.widen(inputs.f32_to_bf16_bits(p32), "bf16").reshape(T, d * d)
        S[h] = p.T @ v64[h]
        Z[h] = p.sum(axis=0).reshape(d, d)
    return S, Z


@pytest.mark.parametrize("d,T,qk", [(16, 300, "unit"), (64, 2500, "unit"), (32, 1500, "spread"),
                                    (16, 32768, "unit")])
def test_rounded_state_passes_and_a_one_percent_tile_fails(oracle_mod, d, T, qk):
    _, k, v = inputs.make_qkv(1, 2, T, d, d, "bf16", seed=d, qk=qk)
    k64, v64 = inputs.widen(k, "bf16")[0], inputs.widen(v, "bf16")[0]
    S, Z = oracle_mod.state(k64, v64)
    bS, bZ = state_bounds(oracle_mod, k64, v64, "bf16")
    Sr, Zr = rounded_product_state(k64, v64)
    # correct bf16-product arithmetic stays well inside the bound
    assert np.all(np.abs(Sr - S) <= bS) and np.all(np.abs(Zr - Z) <= bZ)
    S2, _ = oracle_mod.state(k64 * k64, v64 * v64)
    ratio = np.abs(Sr - S) / (U_BF16 * np.sqrt(S2) + 1e-300)
    assert ratio.max() < 0.75 * (bS / (U_BF16 * np.sqrt(S2) + 1e-300)).min()
    # the rounding is really there: the rounded state differs from the exact one
    assert ratio.max() > 0.5
    # one tile of 128 state rows off by 1% fails the check
    bad = Sr.copy()
    bad[:, :128] *= 1.01
    assert np.any(np.abs(bad - S) > bS)
    # and so does 1% on one row of Z
    badz = Zr.copy()
    badz[:, 3] *= 1.01
    assert np.any(np.abs(badz - Z) > bZ)


def test_rounding_bias_of_bf16_products_is_covered():
    """bf16(p) / p - 1 is not zero-mean: the low bits of products of 8-bit
    significands are not uniform, squares most of all.  The bias grows like
    T on sums of positive terms (the diagonal of Z), which a zero-mean model
    would miss; BIAS_BF16 must cover it with room."""
    from tests.gpu_util import BIAS_BF16

    g = np.random.default_rng(0)
    k = inputs.widen(inputs.f32_to_bf16_bits((g.standard_normal(2_000_000) / 8).astype(np.float32)),
                     "bf16")
    k2 = inputs.widen(inputs.f32_to_bf16_bits((g.standard_normal(2_000_000) / 8).astype(np.float32)),
                      "bf16")
    for p in (k * k, k * k2):
        pr = inputs.widen(inputs.f32_to_bf16_bits(p.astype(np.float32)), "bf16")
        mean = float(np.mean((pr - p) / p))
        assert abs(mean) <= BIAS_BF16 / 2
    sq_mean = float(np.mean((inputs.widen(inputs.f32_to_bf16_bits((k * k).astype(np.float32)),
                                          "bf16") - k * k) / (k * k)))
    assert sq_mean > 2.0 ** -14  # the squares' bias is real, and positive
    # on Z's diagonal over 32768 unit keys the bias dominates the zero-mean part
    _, kk, vv = inputs.make_qkv(1, 1, 32768, 16, 16, "bf16", seed=5)
    k64, v64 = inputs.widen(kk, "bf16")[0], inputs.widen(vv, "bf16")[0]
    _, Z = oracle_mod_state(k64, v64)
    _, Zr = rounded_product_state(k64, v64)
    diag = np.arange(16)
    err = (Zr - Z)[:, diag, diag]
    assert np.all(err > 0)  # every diagonal entry is pushed up
    assert np.all(np.abs(err) <= BIAS_BF16 * np.abs(Z[:, diag, diag]))


def oracle_mod_state(k64, v64):
    from oracle import oracle

    return oracle.state(k64, v64)
