"""Pins of the fp64 oracle's KATA-Mg functions (no GPU).

KATA-Mg (gist.science summary, Technical summary 2.3, "Variantes": several
PSD factors) is read as the product of g rank-one PSD cones, factor m acting
on coordinates [m p, (m + 1) p) of q and k, p = dk / g, so the weight is
w_ts = sum_m (q_t^(m) . k_s^(m))^2 (the reading and its grounds are in the
design notes and in oracle/kata_oracle.c).  The pins, none of which re-types
the oracle's formula:

* exact        — Python Fractions (oracle/exact.py forward_exact_mg) on small
                 integer inputs, and the fixtures of tests/golden/
                 exact_mg_tiny.json, one of them worked by hand.
* g = dk       — every factor is one coordinate, so w_ts = sum_i q_ti^2 k_si^2:
                 linear attention with the feature x -> x * x, computed here
                 by cumulative sums (a different algorithm).
* factors      — the weight is a sum over factors, so numerator and
                 denominator are sums of the single-factor ones: y equals the
                 denominator-weighted mean of the single-factor oracle (itself
                 pinned in test_oracle_pins.py) run on each block.
* symmetries   — rotations inside each block and a permutation of the blocks
                 (applied to q and k together) leave y unchanged; a rotation
                 mixing the blocks changes it (so the factors are really
                 separate).
* the single-factor pins that hold for any g (first row, equal keys,
                 orthogonal keys, zero denominator, convexity, affine values,
                 key sign flips, prefix permutations).
Planted mistakes in a copy of the Mg routine (square of the sum, a dropped
factor, overlapping blocks, a strict mask, no normalisation) must each fail.
The state, recurrent and decode forms must agree with the quadratic one.
"""
from __future__ import annotations

import ctypes
import json
import os
import shutil
import subprocess
import tempfile
from fractions import Fraction

import numpy as np
import pytest

from oracle.exact import forward_exact_mg
from tests import oracle_pins as P1

HERE = os.path.dirname(os.path.abspath(__file__))


def g_for(dk):
    """Factor count used for a head size in the shared checks: two factors
    when dk is even, one per coordinate otherwise."""
    return 2 if dk % 2 == 0 else dk


# ---------------------------------------------------------------------------
# checks taking fwd_mg(q, k, v, g)
# ---------------------------------------------------------------------------


def check_mg_exact(fwd_mg, seed=20, trials=12):
    g_ = np.random.default_rng(seed)
    for trial in range(trials):
        g = int(g_.integers(1, 4))
        p = int(g_.integers(1, 3))
        dk, T, dv = g * p, int(g_.integers(1, 11)), int(g_.integers(1, 3))
        q = g_.integers(-3, 4, size=(1, T, dk)).astype(np.float64)
        k = g_.integers(-3, 4, size=(1, T, dk)).astype(np.float64)
        v = g_.integers(-3, 4, size=(1, T, dv)).astype(np.float64)
        if trial % 3 == 0:
            q[0, g_.integers(0, T)] = 0.0
        y = fwd_mg(q, k, v, g)
        ye = forward_exact_mg(q[0].tolist(), k[0].tolist(), v[0].tolist(), g)
        ye = np.array([[float(x) for x in row] for row in ye]).reshape(1, T, dv)
        if not np.allclose(y, ye, rtol=4e-16, atol=4e-16):
            return False, f"exact mismatch trial {trial} (g={g})"
    return True, ""


def check_mg_one_coordinate_factors(fwd_mg, seed=21):
    g_ = np.random.default_rng(seed)
    BH, T, dk, dv = 2, 40, 6, 3
    q, k, v = (g_.standard_normal((BH, T, d)) for d in (dk, dk, dv))
    y = fwd_mg(q, k, v, dk)
    # linear attention with features x * x: running sums of (k*k) v^T and k*k
    kk = k * k
    num_state = np.cumsum(kk[..., :, None] * v[..., None, :], axis=1)   # [BH, T, dk, dv]
    den_state = np.cumsum(kk, axis=1)                                   # [BH, T, dk]
    qq = q * q
    num = np.einsum("bti,btie->bte", qq, num_state)
    den = np.einsum("bti,bti->bt", qq, den_state)
    ref = num / den[..., None]
    return bool(np.allclose(y, ref, rtol=1e-11, atol=1e-12)), "g = dk closed form"


def check_mg_factor_decomposition(fwd_mg, oracle_mod, seed=22):
    g_ = np.random.default_rng(seed)
    BH, T, dk, dv, g = 2, 50, 8, 4, 2
    q, k, v = (g_.standard_normal((BH, T, d)) for d in (dk, dk, dv))
    y = fwd_mg(q, k, v, g)
    p = dk // g
    num = np.zeros((BH, T, dv))
    den = np.zeros((BH, T))
    for m in range(g):
        blk = slice(m * p, (m + 1) * p)
        ym, dm = oracle_mod.forward(q[..., blk], k[..., blk], v, return_den=True)
        num += ym * dm[..., None]
        den += dm
    ref = num / den[..., None]
    return bool(np.allclose(y, ref, rtol=1e-11, atol=1e-12)), "not the sum of its factors"


def check_mg_block_symmetries(fwd_mg, seed=23):
    g_ = np.random.default_rng(seed)
    BH, T, dk, dv, g = 2, 40, 6, 3, 2
    q, k, v = (g_.standard_normal((BH, T, d)) for d in (dk, dk, dv))
    y = fwd_mg(q, k, v, g)
    p = dk // g
    R = np.zeros((dk, dk))
    for m in range(g):
        Qm, _ = np.linalg.qr(g_.standard_normal((p, p)))
        R[m * p:(m + 1) * p, m * p:(m + 1) * p] = Qm
    y_rot = fwd_mg(q @ R, k @ R, v, g)
    perm = np.concatenate([np.arange(p, dk), np.arange(0, p)])  # swap the two blocks
    y_perm = fwd_mg(q[..., perm], k[..., perm], v, g)
    Qfull, _ = np.linalg.qr(g_.standard_normal((dk, dk)))
    y_mix = fwd_mg(q @ Qfull, k @ Qfull, v, g)
    ok = (np.allclose(y_rot, y, rtol=1e-10, atol=1e-11)
          and np.allclose(y_perm, y, rtol=1e-11, atol=1e-12)
          and not np.allclose(y_mix, y, rtol=1e-6, atol=1e-6))
    return bool(ok), "block rotation / block permutation / mixing rotation"


def shared_checks(fwd_mg):
    """The single-factor pins that hold for any g, run with g_for(dk) factors."""
    fwd = lambda q, k, v: fwd_mg(q, k, v, g_for(q.shape[-1]))  # noqa: E731
    return [(c.__name__, c(fwd)) for c in (
        P1.check_first_row, P1.check_equal_keys, P1.check_orthogonal, P1.check_zero_den,
        P1.check_convex, P1.check_affine, P1.check_key_sign_flip, P1.check_prefix_multiset)]


def run_all_mg(fwd_mg, oracle_mod):
    failed = []
    checks = [("exact", lambda: check_mg_exact(fwd_mg)),
              ("one_coordinate_factors", lambda: check_mg_one_coordinate_factors(fwd_mg)),
              ("factor_decomposition", lambda: check_mg_factor_decomposition(fwd_mg, oracle_mod)),
              ("block_symmetries", lambda: check_mg_block_symmetries(fwd_mg))]
    for name, chk in checks:
        try:
            ok, msg = chk()
        except Exception as e:  # a broken copy may crash or produce NaN
            ok, msg = False, f"raised {type(e).__name__}: {e}"
        if not ok:
            failed.append((name, msg))
    try:
        for name, (ok, msg) in shared_checks(fwd_mg):
            if not ok:
                failed.append((name, msg))
    except Exception as e:
        failed.append(("shared", f"raised {type(e).__name__}: {e}"))
    return failed


# ---------------------------------------------------------------------------
# the real oracle
# ---------------------------------------------------------------------------


def test_mg_oracle_passes_every_pin(oracle_mod):
    assert run_all_mg(oracle_mod.forward_mg, oracle_mod) == []


def test_mg_rows_and_recurrent_forms_pass_every_pin(oracle_mod):
    def rows(q, k, v, g):
        BH, T, _ = q.shape
        bh = np.repeat(np.arange(BH), T)
        tt = np.tile(np.arange(T), BH)
        return oracle_mod.forward_mg_rows(q, k, v, g, bh, tt).reshape(BH, T, v.shape[-1])

    assert run_all_mg(rows, oracle_mod) == []
    assert run_all_mg(oracle_mod.forward_mg_recurrent, oracle_mod) == []


def test_one_factor_is_the_single_factor_oracle(oracle_mod):
    g_ = np.random.default_rng(24)
    q, k, v = (g_.standard_normal((3, 37, d)) for d in (5, 5, 2))
    assert np.array_equal(oracle_mod.forward_mg(q, k, v, 1), oracle_mod.forward(q, k, v))


def test_mg_rejects_a_factor_count_that_does_not_divide_dk(oracle_mod):
    x = np.zeros((1, 3, 6))
    with pytest.raises(ValueError):
        oracle_mod.forward_mg(x, x, x, 4)


def test_golden_mg_fixtures(oracle_mod):
    """tests/golden/exact_mg_tiny.json: exact rationals from oracle/exact.py,
    written by tests/golden/make_golden.py.  Case T2_d2_g2_by_hand: two
    one-coordinate factors, so row 1 weighs key 0 by 1*1 + 1*1 = 2 and key 1 by
    (1*2)^2 + (1*-1)^2 = 5, giving y_1 = (2 * 1 + 5 * 3) / 7 = 17/7."""
    data = json.load(open(os.path.join(HERE, "golden", "exact_mg_tiny.json")))
    assert data["cases"]
    for case in data["cases"]:
        q = np.array(case["q"], np.float64)[None]
        k = np.array(case["k"], np.float64)[None]
        v = np.array(case["v"], np.float64)[None]
        want = np.array([[float(Fraction(x)) for x in row] for row in case["y"]])
        got = oracle_mod.forward_mg(q, k, v, case["g"])[0]
        assert np.allclose(got, want, rtol=4e-16, atol=0), case["name"]
    hand = [c for c in data["cases"] if c["name"] == "T2_d2_g2_by_hand"][0]
    assert hand["y"] == [["1/1"], ["17/7"]]


# ---------------------------------------------------------------------------
# planted mistakes in a copy of the Mg routine
# ---------------------------------------------------------------------------

# (name, [(original text, replacement), ...]); each replaces the first occurrence
MG_MUTANTS = [
    ("square_of_the_sum", [("        w += dot * dot;\n    }\n    return w;",
                            "        w += dot;\n    }\n    return w * w;")]),
    ("dropped_factor", [("    for (int m = 0; m < g; ++m) {\n        double dot = 0.0;",
                         "    for (int m = 1; m < g; ++m) {\n        double dot = 0.0;")]),
    ("overlapping_blocks", [("for (int i = m * p; i < (m + 1) * p; ++i) dot += qt[i] * ks[i];",
                             "for (int i = m; i < m + p; ++i) dot += qt[i] * ks[i];")]),
    ("strict_causal_mask", [("    for (long s = 0; s <= t; ++s) {\n        const double *vs = x->v",
                             "    for (long s = 0; s < t; ++s) {\n        const double *vs = x->v")]),
    ("no_normalisation", [("y[e] = (den == 0.0) ? 0.0 : y[e] / den;\n    if (x->den)",
                           "y[e] = (den == 0.0) ? 0.0 : y[e];\n    if (x->den)")]),
]


@pytest.fixture(scope="module")
def mutant_dir():
    d = tempfile.mkdtemp(prefix="kata_oracle_mg_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def _mutant_forward_mg(src_text, mutant_dir, name):
    c = os.path.join(mutant_dir, name + ".c")
    so = os.path.join(mutant_dir, name + ".so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", so, c, "-lpthread", "-lm"])
    lib = ctypes.CDLL(so)
    Pd = ctypes.POINTER(ctypes.c_double)
    i32, i64 = ctypes.c_int, ctypes.c_long
    lib.kata_oracle_forward_mg.argtypes = [Pd, Pd, Pd, Pd, Pd, i64, i64, i32, i32, i32, i32]
    lib.kata_oracle_forward_mg.restype = i32

    def fwd(q, k, v, g):
        q, k, v = (np.ascontiguousarray(a, np.float64) for a in (q, k, v))
        BH, T, dk = q.shape
        dv = v.shape[-1]
        y = np.zeros((BH, T, dv))
        den = np.zeros((BH, T))
        p = lambda a: a.ctypes.data_as(Pd)  # noqa: E731
        if lib.kata_oracle_forward_mg(p(q), p(k), p(v), p(y), p(den), BH, T, dk, dv, g, 1):
            raise ValueError("g does not divide dk")
        return y

    return fwd


@pytest.mark.parametrize("mutant", MG_MUTANTS, ids=lambda m: m[0])
def test_planted_mg_mistake_is_caught(oracle_mod, mutant, mutant_dir):
    name, edits = mutant
    src = open(os.path.join(HERE, "..", "oracle", "kata_oracle.c")).read()
    for old, new in edits:
        assert old in src, f"mutation site for {name} not found in the oracle source"
        src = src.replace(old, new, 1)
    failed = run_all_mg(_mutant_forward_mg(src, mutant_dir, name), oracle_mod)
    assert failed, f"mutant {name} passed every pin"


# ---------------------------------------------------------------------------
# state, recurrent and decode forms
# ---------------------------------------------------------------------------


def test_mg_state_is_the_block_part_of_the_single_factor_state(oracle_mod):
    g_ = np.random.default_rng(25)
    BH, T, dk, dv = 2, 70, 6, 3
    k, v = g_.standard_normal((BH, T, dk)), g_.standard_normal((BH, T, dv))
    S1, Z1 = oracle_mod.state(k, v, 50)
    for g in (1, 2, 3, 6):
        S, Z = oracle_mod.state_mg(k, v, g, 50)
        p = dk // g
        same = (np.arange(dk)[:, None] // p) == (np.arange(dk)[None, :] // p)
        assert np.array_equal(Z, Z1 * same)
        assert np.array_equal(S, S1 * same.reshape(1, dk * dk, 1))


def test_mg_recurrent_and_decode_extend_the_forward(oracle_mod):
    g_ = np.random.default_rng(26)
    BH, T, dk, dv, g = 3, 60, 8, 4, 2
    q, k, v = (g_.standard_normal((BH, T + 1, d)) for d in (dk, dk, dv))
    y = oracle_mod.forward_mg(q, k, v, g)
    assert np.allclose(oracle_mod.forward_mg_recurrent(q, k, v, g), y, rtol=1e-11, atol=1e-12)
    S, Z = oracle_mod.state_mg(k[:, :T], v[:, :T], g)
    yd, S2, Z2, _ = oracle_mod.decode_step_mg(q[:, T], k[:, T], v[:, T], S, Z, g)
    assert np.allclose(yd, y[:, T], rtol=1e-11, atol=1e-12)
    S3, Z3 = oracle_mod.state_mg(k, v, g)
    assert np.allclose(S2, S3) and np.allclose(Z2, Z3)
    # a zero key and value add nothing: the step's readout is that of the state
    for n in (1, 30, T):
        S, Z = oracle_mod.state_mg(k, v, g, n)
        yq, _, _, _ = oracle_mod.decode_step_mg(q[:, n - 1], np.zeros((BH, dk)),
                                                np.zeros((BH, dv)), S, Z, g)
        assert np.allclose(yq, y[:, n - 1], rtol=1e-11, atol=1e-12)
