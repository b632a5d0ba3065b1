"""Checks that pin the fp64 oracle to facts fixed by the pages and by mathematics.

Each check takes a forward callable ``fwd(q, k, v) -> y`` (arrays
[BH, T, d] float64) so that the same checks run on the real oracle (they must
all pass) and on deliberately broken copies of it (each copy must fail at
least one), see tests/test_oracle_pins.py.

What fixes each expected value (no check re-types the oracle's own formula):

* exact      — Python Fractions on small integer inputs (oracle/exact.py):
               the weights, numerator and denominator are exact integers.
* first row  — y_0 = v_0: the convex gate includes the current token
               (gist.science summary of "Kernelized Linear Attention: Breaking
               the Capacity Wall with Symmetric Cones", Technical summary 2.1).
* equal keys — all keys equal and q.k != 0: every weight is the same, so y_t
               is the running mean of v_0..v_t.
* d = 1      — (q k_s)^2 = q^2 k_s^2, so y_t = sum k_s^2 v_s / sum k_s^2,
               independent of q.
* orthogonal — q_t orthogonal to every earlier key: only the current token has
               weight, y_t = v_t.
* zero den   — q_t = 0: the denominator is 0 and y_t = 0 (reading: no epsilon).
* convexity  — every coordinate of y_t lies in [min, max] of v_0..v_t
               (summary 2.1 "convex gate"; nonnegative weights, 2.1/2.2).
* affine     — v -> a v + b gives y -> a y + b (weights sum to one).
* scale/sign/rotation — the squared inner product is unchanged by q -> a q,
               k -> b k, sign flips and a shared orthogonal rotation.
* prefix multiset — y_t depends only on the set {(k_s, v_s) : s <= t}:
               permuting earlier tokens leaves y_t unchanged.
"""
from __future__ import annotations

import numpy as np

from oracle.exact import forward_exact


def _rng(seed):
    return np.random.default_rng(seed)


def check_exact(fwd, seed=0, trials=12):
    g = _rng(seed)
    for trial in range(trials):
        T = int(g.integers(1, 13))
        dk = int(g.integers(1, 4))
        dv = int(g.integers(1, 4))
        q = g.integers(-3, 4, size=(1, T, dk)).astype(np.float64)
        k = g.integers(-3, 4, size=(1, T, dk)).astype(np.float64)
        v = g.integers(-3, 4, size=(1, T, dv)).astype(np.float64)
        if trial % 3 == 0:  # force some zero denominators
            q[0, g.integers(0, T)] = 0.0
        y = fwd(q, k, v)
        ye = forward_exact(q[0].tolist(), k[0].tolist(), v[0].tolist())
        ye = np.array([[float(x) for x in row] for row in ye]).reshape(1, T, dv)
        if not np.allclose(y, ye, rtol=4e-16, atol=4e-16):
            return False, f"exact mismatch trial {trial}: max |d| = {np.abs(y - ye).max()}"
    return True, ""


def _rand(g, BH, T, dk, dv):
    q = g.standard_normal((BH, T, dk))
    k = g.standard_normal((BH, T, dk))
    v = g.standard_normal((BH, T, dv))
    return q, k, v


def check_first_row(fwd, seed=1):
    g = _rng(seed)
    q, k, v = _rand(g, 3, 17, 5, 4)
    y = fwd(q, k, v)
    return bool(np.allclose(y[:, 0], v[:, 0], rtol=1e-13, atol=1e-13)), "y_0 != v_0"


def check_equal_keys(fwd, seed=2):
    g = _rng(seed)
    q, k, v = _rand(g, 2, 40, 6, 3)
    k[:] = k[:, :1]
    y = fwd(q, k, v)
    mean = np.cumsum(v, axis=1) / np.arange(1, 41)[None, :, None]
    return bool(np.allclose(y, mean, rtol=1e-11, atol=1e-12)), "equal keys: not the running mean"


def check_d1(fwd, seed=3):
    g = _rng(seed)
    q, k, v = _rand(g, 2, 50, 1, 3)
    q[np.abs(q) < 1e-3] = 1.0
    y = fwd(q, k, v)
    w = k[..., 0] ** 2
    ref = np.cumsum(w[..., None] * v, axis=1) / np.cumsum(w, axis=1)[..., None]
    return bool(np.allclose(y, ref, rtol=1e-11, atol=1e-12)), "d=1 closed form"


def check_orthogonal(fwd, seed=4):
    g = _rng(seed)
    T, dk, dv = 12, 12, 5
    # keys along basis vectors e_0..e_{T-1}; q_t along e_t: q_t.k_s = 0 for s != t
    k = np.zeros((1, T, dk))
    q = np.zeros((1, T, dk))
    for t in range(T):
        k[0, t, t] = g.uniform(0.5, 2.0)
        q[0, t, t] = g.uniform(0.5, 2.0) * (1 if t % 2 else -1)
    v = g.standard_normal((1, T, dv))
    y = fwd(q, k, v)
    return bool(np.allclose(y, v, rtol=1e-13, atol=1e-13)), "orthogonal keys: y_t != v_t"


def check_zero_den(fwd, seed=5):
    g = _rng(seed)
    q, k, v = _rand(g, 2, 20, 4, 3)
    q[0, 7] = 0.0
    q[1, 0] = 0.0
    y = fwd(q, k, v)
    ok = np.all(y[0, 7] == 0.0) and np.all(y[1, 0] == 0.0) and np.isfinite(y).all()
    return bool(ok), "zero denominator must give y = 0"


def check_convex(fwd, seed=6):
    g = _rng(seed)
    q, k, v = _rand(g, 3, 64, 8, 6)
    y = fwd(q, k, v)
    lo = np.minimum.accumulate(v, axis=1)
    hi = np.maximum.accumulate(v, axis=1)
    ok = np.all(y >= lo - 1e-12) and np.all(y <= hi + 1e-12)
    return bool(ok), "output outside the [min, max] of prefix values"


def check_affine(fwd, seed=7):
    g = _rng(seed)
    q, k, v = _rand(g, 2, 48, 6, 4)
    a, b = -1.75, 0.625
    y1 = fwd(q, k, v)
    y2 = fwd(q, k, a * v + b)
    return bool(np.allclose(y2, a * y1 + b, rtol=1e-11, atol=1e-11)), "affine equivariance"


def check_scale_sign_rotation(fwd, seed=8):
    g = _rng(seed)
    q, k, v = _rand(g, 2, 48, 6, 4)
    y = fwd(q, k, v)
    # Per-row rescaling (and sign) of q cancels between numerator and
    # denominator of that row.  Keys may flip sign per row, but only a common
    # per-head factor b keeps the ratio (it multiplies every w_ts by b^2).
    qs = q * g.uniform(0.3, 3.0, size=(2, 48, 1)) * g.choice([-1.0, 1.0], size=(2, 48, 1))
    ks = k * np.array([0.5, 2.5])[:, None, None] * g.choice([-1.0, 1.0], size=(2, 48, 1))
    y2 = fwd(qs, ks, v)
    Qm, _ = np.linalg.qr(g.standard_normal((6, 6)))
    y3 = fwd(q @ Qm, k @ Qm, v)
    ok = np.allclose(y2, y, rtol=1e-10, atol=1e-11) and np.allclose(y3, y, rtol=1e-10, atol=1e-11)
    return bool(ok), "scale / sign / rotation invariance"


def check_key_sign_flip(fwd, seed=9):
    """Flipping the sign of any individual key leaves every weight unchanged."""
    g = _rng(seed)
    q, k, v = _rand(g, 2, 40, 5, 3)
    y = fwd(q, k, v)
    k2 = k * g.choice([-1.0, 1.0], size=(2, 40, 1))
    return bool(np.allclose(fwd(q, k2, v), y, rtol=1e-11, atol=1e-12)), "key sign flip"


def check_prefix_multiset(fwd, seed=10):
    g = _rng(seed)
    q, k, v = _rand(g, 1, 30, 5, 3)
    t = 29
    perm = g.permutation(t)
    k2 = k.copy()
    v2 = v.copy()
    k2[0, :t] = k[0, perm]
    v2[0, :t] = v[0, perm]
    y1 = fwd(q, k, v)[0, t]
    y2 = fwd(q, k2, v2)[0, t]
    return bool(np.allclose(y1, y2, rtol=1e-11, atol=1e-12)), "prefix permutation changed y_t"


ALL_CHECKS = [
    check_exact,
    check_first_row,
    check_equal_keys,
    check_d1,
    check_orthogonal,
    check_zero_den,
    check_convex,
    check_affine,
    check_scale_sign_rotation,
    check_key_sign_flip,
    check_prefix_multiset,
]


def run_all(fwd):
    """Returns the list of (check name, message) that failed."""
    failed = []
    for chk in ALL_CHECKS:
        try:
            ok, msg = chk(fwd)
        except Exception as e:  # a broken copy may crash or produce NaN
            ok, msg = False, f"raised {type(e).__name__}: {e}"
        if not ok:
            failed.append((chk.__name__, msg))
    return failed
