"""Pins of the fp64 CPU oracle (no GPU).

1. Every oracle form (quadratic, selected rows, recurrent, chunked) passes the
   checks in tests/oracle_pins.py, whose expected values come from exact
   rational arithmetic, closed forms and invariants -- never from the oracle.
2. Broken copies of the oracle (a mistake planted in a copy of its C source,
   compiled on the CPU) each fail at least one of those checks, so the checks
   are strong enough to notice a dropped term, a wrong index or sign, a strict
   mask, a missing square or a missing normalisation.
3. The state and decode entry points agree with the quadratic definition.
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

from tests.oracle_pins import ALL_CHECKS, run_all

# ---------------------------------------------------------------------------
# 1. the real oracle passes every pin
# ---------------------------------------------------------------------------


def _fwd_rows(oracle_mod):
    def f(q, k, v):
        BH, T, _ = q.shape
        bh = np.repeat(np.arange(BH), T)
        tt = np.tile(np.arange(T), BH)
        return oracle_mod.forward_rows(q, k, v, bh, tt).reshape(BH, T, v.shape[-1])

    return f


def _fwd_chunked(oracle_mod, C):
    return lambda q, k, v: oracle_mod.forward_chunked(q, k, v, C)


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__)
def test_quadratic_oracle_pins(oracle_mod, check):
    ok, msg = check(oracle_mod.forward)
    assert ok, msg


@pytest.mark.parametrize("form", ["rows", "recurrent", "chunked1", "chunked3", "chunked16"])
def test_other_forms_pass_all_pins(oracle_mod, form):
    fwd = {
        "rows": _fwd_rows(oracle_mod),
        "recurrent": oracle_mod.forward_recurrent,
        "chunked1": _fwd_chunked(oracle_mod, 1),
        "chunked3": _fwd_chunked(oracle_mod, 3),
        "chunked16": _fwd_chunked(oracle_mod, 16),
    }[form]
    assert run_all(fwd) == []


def test_second_forms_match_quadratic(oracle_mod):
    """Recurrent and chunked forms (every C, including C = T and C > T) equal
    the quadratic definition (arXiv abstract: "exact O(T) chunked-state
    form"; gist.science summary 2.3)."""
    g = np.random.default_rng(123)
    for (BH, T, dk, dv) in [(2, 200, 16, 16), (1, 130, 8, 5), (3, 64, 4, 7)]:
        q = g.standard_normal((BH, T, dk))
        k = g.standard_normal((BH, T, dk))
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        v = g.standard_normal((BH, T, dv))
        y = oracle_mod.forward(q, k, v)
        scale = np.abs(y).max(axis=-1, keepdims=True)
        yr = oracle_mod.forward_recurrent(q, k, v)
        assert (np.abs(yr - y) / scale).max() < 1e-12
        for C in [1, 2, 3, 16, 64, T, T + 5]:
            yc = oracle_mod.forward_chunked(q, k, v, C)
            assert (np.abs(yc - y) / scale).max() < 1e-12, C


def test_weights_nonnegative_and_den_positive(oracle_mod):
    g = np.random.default_rng(5)
    q = g.standard_normal((2, 100, 8))
    k = g.standard_normal((2, 100, 8))
    v = g.standard_normal((2, 100, 3))
    _, den = oracle_mod.forward(q, k, v, return_den=True)
    assert (den > 0).all()
    # with one query repeated on every row, den_t is a running sum of
    # nonnegative weights and therefore nondecreasing in t
    q[:] = q[:, :1]
    _, den = oracle_mod.forward(q, k, v, return_den=True)
    assert (np.diff(den, axis=-1) >= 0).all()


# ---------------------------------------------------------------------------
# 2. planted mistakes are caught
# ---------------------------------------------------------------------------

# (name, original text, replacement); each replaces the first occurrence,
# which lies in the quadratic-definition routine of kata_oracle.c.
MUTANTS = [
    ("weight_not_squared", "double w = dot * dot;", "double w = fabs(dot);"),
    ("strict_causal_mask", "for (long s = 0; s <= t; ++s) {", "for (long s = 0; s < t; ++s) {"),
    ("no_normalisation", "for (int e = 0; e < dv; ++e) y[e] /= den;",
     "for (int e = 0; e < dv; ++e) y[e] /= 1.0;"),
    ("keys_read_from_q", "const double *ks = k + (bh * T + s) * dk;",
     "const double *ks = q + (bh * T + s) * dk;"),
    ("dropped_dot_term", "for (int i = 0; i < dk; ++i) dot += qt[i] * ks[i];",
     "for (int i = 1; i < dk; ++i) dot += qt[i] * ks[i];"),
    ("one_term_wrong_sign", "for (int i = 0; i < dk; ++i) dot += qt[i] * ks[i];",
     "for (int i = 0; i < dk; ++i) dot += (i == 0 ? -1.0 : 1.0) * qt[i] * ks[i];"),
    ("value_of_query_row", "const double *vs = v + (bh * T + s) * dv;",
     "const double *vs = v + (bh * T + t) * dv;"),
    ("value_index_transposed", "for (int e = 0; e < dv; ++e) y[e] += w * vs[e];",
     "for (int e = 0; e < dv; ++e) y[e] += w * vs[dv - 1 - e];"),
    ("query_of_key_row", "for (int i = 0; i < dk; ++i) dot += qt[i] * ks[i];",
     "for (int i = 0; i < dk; ++i) dot += q[(bh * T + s) * dk + i] * ks[i];"),
    ("no_zero_den_guard", "    if (den == 0.0) {\n        for (int e = 0; e < dv; ++e) y[e] = 0.0;\n    } else {",
     "    if (0) {\n    } else {"),
]


@pytest.fixture(scope="module")
def mutant_dir():
    d = tempfile.mkdtemp(prefix="kata_oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def _mutant_forward(src_text, mutant_dir, name):
    c = os.path.join(mutant_dir, name + ".c")
    so = os.path.join(mutant_dir, name + ".so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", so, c, "-lpthread", "-lm"])
    lib = ctypes.CDLL(so)
    P = ctypes.POINTER(ctypes.c_double)
    lib.kata_oracle_forward.argtypes = [P, P, P, P, P, ctypes.c_long, ctypes.c_long,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int]

    def fwd(q, k, v):
        q = np.ascontiguousarray(q, np.float64)
        k = np.ascontiguousarray(k, np.float64)
        v = np.ascontiguousarray(v, np.float64)
        BH, T, dk = q.shape
        dv = v.shape[-1]
        y = np.zeros((BH, T, dv))
        den = np.zeros((BH, T))
        p = lambda a: a.ctypes.data_as(P)  # noqa: E731
        lib.kata_oracle_forward(p(q), p(k), p(v), p(y), p(den), BH, T, dk, dv, 1)
        return y

    return fwd


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m[0])
def test_planted_mistake_is_caught(mutant, mutant_dir):
    name, old, new = mutant
    src = open(os.path.join(os.path.dirname(__file__), "..", "oracle", "kata_oracle.c")).read()
    assert old in src, f"mutation site for {name} not found in the oracle source"
    fwd = _mutant_forward(src.replace(old, new, 1), mutant_dir, name)
    failed = run_all(fwd)
    assert failed, f"mutant {name} passed every pin"


# ---------------------------------------------------------------------------
# 3. state, decode step and selected rows
# ---------------------------------------------------------------------------


def test_state_reads_out_the_definition(oracle_mod):
    """phi(q)^T S_n / (q^T Z_n q) must equal the quadratic row n-1 when q is
    that row's query (the state is the sum the recurrent form reads)."""
    g = np.random.default_rng(7)
    BH, T, dk, dv = 3, 90, 6, 4
    q = g.standard_normal((BH, T, dk))
    k = g.standard_normal((BH, T, dk))
    v = g.standard_normal((BH, T, dv))
    y = oracle_mod.forward(q, k, v)
    for n in [1, 2, 45, 90]:
        S, Z = oracle_mod.state(k, v, n)
        # symmetric in (i, j), Z positive semi-definite with trace sum |k|^2
        S4 = S.reshape(BH, dk, dk, dv)
        assert np.allclose(S4, S4.transpose(0, 2, 1, 3))
        assert np.allclose(Z, Z.transpose(0, 2, 1))
        assert np.linalg.eigvalsh(Z).min() > -1e-9
        assert np.allclose(np.trace(Z, axis1=1, axis2=2), (k[:, :n] ** 2).sum(axis=(1, 2)))
        # a decode step with a zero key and value adds nothing, so its readout
        # is phi(q)^T S / q^T Z q on the state as given
        yq, _, _, _ = oracle_mod.decode_step(q[:, n - 1], np.zeros((BH, dk)), np.zeros((BH, dv)),
                                             S, Z)
        assert np.allclose(yq, y[:, n - 1], rtol=1e-11, atol=1e-12)


def test_decode_step_extends_the_forward(oracle_mod):
    g = np.random.default_rng(8)
    BH, T, dk, dv = 4, 60, 8, 8
    q = g.standard_normal((BH, T + 1, dk))
    k = g.standard_normal((BH, T + 1, dk))
    v = g.standard_normal((BH, T + 1, dv))
    S, Z = oracle_mod.state(k[:, :T], v[:, :T])
    yd, S2, Z2, _ = oracle_mod.decode_step(q[:, T], k[:, T], v[:, T], S, Z)
    y = oracle_mod.forward(q, k, v)
    assert np.allclose(yd, y[:, T], rtol=1e-11, atol=1e-12)
    S3, Z3 = oracle_mod.state(k, v)
    assert np.allclose(S2, S3) and np.allclose(Z2, Z3)


def test_rows_equal_full(oracle_mod):
    g = np.random.default_rng(9)
    q = g.standard_normal((3, 77, 5))
    k = g.standard_normal((3, 77, 5))
    v = g.standard_normal((3, 77, 2))
    y = oracle_mod.forward(q, k, v)
    bh = g.integers(0, 3, size=40)
    tt = g.integers(0, 77, size=40)
    yr = oracle_mod.forward_rows(q, k, v, bh, tt)
    assert np.array_equal(yr, y[bh, tt])


def test_symmetric_feature_identity():
    """(q.k)^2 = <vec(qq^T), vec(kk^T)> = sum_i q_i^2 k_i^2 + 2 sum_{i<j} q_i q_j k_i k_j.
    The first equality is the rank-one PSD feature of gist.science summary
    2.2; the second is the half-triangle packing the CUDA kernels use."""
    g = np.random.default_rng(10)
    for d in [1, 2, 16, 64]:
        q = g.standard_normal(d)
        k = g.standard_normal(d)
        lhs = float(q @ k) ** 2
        full = float(np.outer(q, q).ravel() @ np.outer(k, k).ravel())
        iu = np.triu_indices(d, 1)
        half = float((q * q) @ (k * k) + 2 * (np.outer(q, q)[iu] @ np.outer(k, k)[iu]))
        assert abs(lhs - full) <= 1e-12 * max(1, lhs)
        assert abs(lhs - half) <= 1e-12 * max(1, lhs)


def test_golden_exact_fixtures(oracle_mod):
    """tests/golden/exact_tiny.json holds exact rationals written by
    tests/golden/make_golden.py from oracle/exact.py (hand-checkable: e.g. in
    case T4_d2, row 1 has weights (q_1.k_0)^2 = 4 and (q_1.k_1)^2 = 1, so
    y_1 = (4 v_0 + v_1) / 5 = (7/5, -8/5))."""
    import json
    from fractions import Fraction

    path = os.path.join(os.path.dirname(__file__), "golden", "exact_tiny.json")
    data = json.load(open(path))
    assert data["cases"]
    for case in data["cases"]:
        q = np.array(case["q"], np.float64)[None]
        k = np.array(case["k"], np.float64)[None]
        v = np.array(case["v"], np.float64)[None]
        want = np.array([[float(Fraction(x)) for x in row] for row in case["y"]])
        got = oracle_mod.forward(q, k, v)[0]
        assert np.allclose(got, want, rtol=4e-16, atol=0), case["name"]
    t4 = [c for c in data["cases"] if c["name"] == "T4_d2"][0]
    assert t4["y"][1] == ["7/5", "-8/5"]
