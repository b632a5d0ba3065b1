"""fp64 CPU oracle for the KATA causal forward — TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import this module.  The CUDA library never does, and this
module imports nothing from the package except nothing at all: it takes
plain numpy arrays (already widened to float64 from the exact bf16/fp32 input
bits) and returns numpy arrays.

The arithmetic lives in ``kata_oracle.c`` (plain C, fp64), compiled on first
use with gcc into ``liboracle_kata.so`` beside it.  What each entry computes,
and the passages it follows, is documented there:

* ``forward``            — the quadratic definition, every row
  (gist.science summary of "Kernelized Linear Attention: Breaking the
  Capacity Wall with Symmetric Cones", Technical summary 2.1 and 2.2).
* ``forward_rows``       — the same definition for selected (head, row) pairs.
* ``state``              — S = sum phi(k) v^T, Z = sum k k^T by direct summation.
* ``forward_recurrent``  — token-by-token state update then readout
  (arXiv abstract, "constant-time recurrent inference").
* ``forward_chunked``    — chunk sums, exclusive prefix over chunks, then
  inter + intra terms (summary 2.3; abstract, "exact O(T) chunked-state form").
* ``decode_step``        — one recurrent step on a given state.
* ``forward_mg``, ``forward_mg_rows``, ``state_mg``, ``forward_mg_recurrent``,
  ``decode_step_mg`` — the same for KATA-Mg, g rank-one PSD factors on
  consecutive blocks of dk / g coordinates (summary 2.3, "Variantes", in the
  reading documented in kata_oracle.c).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kata_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_kata.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no GPU, no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lpthread", "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.POINTER(ctypes.c_double)
        L = ctypes.POINTER(ctypes.c_long)
        lib.kata_oracle_forward.argtypes = [P, P, P, P, P, ctypes.c_long, ctypes.c_long,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.kata_oracle_forward_rows.argtypes = [P, P, P, ctypes.c_long, ctypes.c_int,
                                                 ctypes.c_int, L, L, ctypes.c_long, P, P,
                                                 ctypes.c_int]
        lib.kata_oracle_state.argtypes = [P, P, ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                          ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int]
        lib.kata_oracle_forward_recurrent.argtypes = [P, P, P, P, ctypes.c_long, ctypes.c_long,
                                                      ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.kata_oracle_forward_chunked.argtypes = [P, P, P, P, ctypes.c_long, ctypes.c_long,
                                                    ctypes.c_int, ctypes.c_int, ctypes.c_long,
                                                    ctypes.c_int]
        lib.kata_oracle_forward_chunked.restype = ctypes.c_int
        lib.kata_oracle_decode_step.argtypes = [P, P, P, P, P, P, P, ctypes.c_long,
                                                ctypes.c_int, ctypes.c_int]
        i32, i64 = ctypes.c_int, ctypes.c_long
        lib.kata_oracle_forward_mg.argtypes = [P, P, P, P, P, i64, i64, i32, i32, i32, i32]
        lib.kata_oracle_forward_mg_rows.argtypes = [P, P, P, i64, i32, i32, i32, L, L, i64, P,
                                                    P, i32]
        lib.kata_oracle_state_mg.argtypes = [P, P, i64, i64, i64, i32, i32, i32, P, P, i32]
        lib.kata_oracle_forward_mg_recurrent.argtypes = [P, P, P, P, i64, i64, i32, i32, i32,
                                                         i32]
        lib.kata_oracle_decode_step_mg.argtypes = [P, P, P, P, P, P, P, i64, i32, i32, i32]
        for name in ("kata_oracle_forward_mg", "kata_oracle_forward_mg_rows",
                     "kata_oracle_state_mg", "kata_oracle_forward_mg_recurrent",
                     "kata_oracle_decode_step_mg"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _threads(n):
    return int(n) if n else (os.cpu_count() or 1)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _heads(x, d):
    """[..., T, d] -> ([BH, T, d] float64, leading shape)."""
    x = _f64(x)
    lead = x.shape[:-2]
    return np.ascontiguousarray(x.reshape(-1, x.shape[-2], d)), lead


def forward(q, k, v, nthreads=None, return_den=False):
    """y[..., t, :] = sum_{s<=t} (q_t.k_s)^2 v_s / sum_{s<=t} (q_t.k_s)^2 (0 if 0)."""
    lib = _load()
    dk, dv = q.shape[-1], v.shape[-1]
    qh, lead = _heads(q, dk)
    kh, _ = _heads(k, dk)
    vh, _ = _heads(v, dv)
    BH, T = qh.shape[0], qh.shape[1]
    y = np.zeros((BH, T, dv))
    den = np.zeros((BH, T))
    lib.kata_oracle_forward(_p(qh), _p(kh), _p(vh), _p(y), _p(den), BH, T, dk, dv,
                            _threads(nthreads))
    y = y.reshape(*lead, T, dv)
    return (y, den.reshape(*lead, T)) if return_den else y


def forward_rows(q, k, v, bh_idx, t_idx, nthreads=None, return_den=False):
    """Selected rows of ``forward``; q,k,v are [BH, T, d]; returns [nrows, dv]."""
    lib = _load()
    dk, dv = q.shape[-1], v.shape[-1]
    qh, _ = _heads(q, dk)
    kh, _ = _heads(k, dk)
    vh, _ = _heads(v, dv)
    T = qh.shape[1]
    bh = np.ascontiguousarray(bh_idx, dtype=np.int64)
    tt = np.ascontiguousarray(t_idx, dtype=np.int64)
    assert bh.shape == tt.shape and bh.ndim == 1
    assert (bh >= 0).all() and (bh < qh.shape[0]).all() and (tt >= 0).all() and (tt < T).all()
    n = bh.shape[0]
    y = np.zeros((n, dv))
    den = np.zeros(n)
    Lp = ctypes.POINTER(ctypes.c_long)
    lib.kata_oracle_forward_rows(_p(qh), _p(kh), _p(vh), T, dk, dv, bh.ctypes.data_as(Lp),
                                 tt.ctypes.data_as(Lp), n, _p(y), _p(den), _threads(nthreads))
    return (y, den) if return_den else y


def state(k, v, n=None, nthreads=None):
    """S[..., i*dk+j, e] = sum_{s<n} k_si k_sj v_se and Z[..., i, j] = sum_{s<n} k_si k_sj."""
    lib = _load()
    dk, dv = k.shape[-1], v.shape[-1]
    kh, lead = _heads(k, dk)
    vh, _ = _heads(v, dv)
    BH, T = kh.shape[0], kh.shape[1]
    n = T if n is None else int(n)
    assert 0 <= n <= T
    S = np.zeros((BH, dk * dk, dv))
    Z = np.zeros((BH, dk, dk))
    lib.kata_oracle_state(_p(kh), _p(vh), BH, T, n, dk, dv, _p(S), _p(Z), _threads(nthreads))
    return S.reshape(*lead, dk * dk, dv), Z.reshape(*lead, dk, dk)


def forward_recurrent(q, k, v, nthreads=None):
    lib = _load()
    dk, dv = q.shape[-1], v.shape[-1]
    qh, lead = _heads(q, dk)
    kh, _ = _heads(k, dk)
    vh, _ = _heads(v, dv)
    BH, T = qh.shape[0], qh.shape[1]
    y = np.zeros((BH, T, dv))
    lib.kata_oracle_forward_recurrent(_p(qh), _p(kh), _p(vh), _p(y), BH, T, dk, dv,
                                      _threads(nthreads))
    return y.reshape(*lead, T, dv)


def forward_chunked(q, k, v, C, nthreads=None):
    lib = _load()
    dk, dv = q.shape[-1], v.shape[-1]
    qh, lead = _heads(q, dk)
    kh, _ = _heads(k, dk)
    vh, _ = _heads(v, dv)
    BH, T = qh.shape[0], qh.shape[1]
    y = np.zeros((BH, T, dv))
    rc = lib.kata_oracle_forward_chunked(_p(qh), _p(kh), _p(vh), _p(y), BH, T, dk, dv, int(C),
                                         _threads(nthreads))
    if rc != 0:
        raise ValueError("chunked oracle: C must be >= 1 and dv <= 512")
    return y.reshape(*lead, T, dv)


def decode_step(q, k, v, S, Z):
    """One step on copies of (S, Z); q,k: [BH, dk]; v: [BH, dv].  Returns (y, S', Z', den)."""
    lib = _load()
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    BH, dk = q.shape
    dv = v.shape[1]
    S2 = _f64(S).reshape(BH, dk * dk, dv).copy()
    Z2 = _f64(Z).reshape(BH, dk, dk).copy()
    y = np.zeros((BH, dv))
    den = np.zeros(BH)
    lib.kata_oracle_decode_step(_p(q), _p(k), _p(v), _p(S2), _p(Z2), _p(y), _p(den), BH, dk, dv)
    return y, S2, Z2, den


# ---------------------------------------------------------------------------
# KATA-Mg: g rank-one PSD factors, factor m on coordinates [m p, (m + 1) p)
# ---------------------------------------------------------------------------


def _check_g(dk, g):
    if g < 1 or dk % g != 0:
        raise ValueError(f"g = {g} must divide dk = {dk}")


def forward_mg(q, k, v, g, nthreads=None, return_den=False):
    """y[..., t, :] = sum_{s<=t} w_ts v_s / sum_{s<=t} w_ts with
    w_ts = sum_m (q_t^(m).k_s^(m))^2 (0 if the sum is 0)."""
    lib = _load()
    dk, dv = q.shape[-1], v.shape[-1]
    _check_g(dk, g)
    qh, lead = _heads(q, dk)
    kh, _ = _heads(k, dk)
    vh, _ = _heads(v, dv)
    BH, T = qh.shape[0], qh.shape[1]
    y = np.zeros((BH, T, dv))
    den = np.zeros((BH, T))
    lib.kata_oracle_forward_mg(_p(qh), _p(kh), _p(vh), _p(y), _p(den), BH, T, dk, dv, int(g),
                               _threads(nthreads))
    y = y.reshape(*lead, T, dv)
    return (y, den.reshape(*lead, T)) if return_den else y


def forward_mg_rows(q, k, v, g, bh_idx, t_idx, nthreads=None):
    """Selected rows of ``forward_mg``; q,k,v are [BH, T, d]; returns [nrows, dv]."""
    lib = _load()
    dk, dv = q.shape[-1], v.shape[-1]
    _check_g(dk, g)
    qh, _ = _heads(q, dk)
    kh, _ = _heads(k, dk)
    vh, _ = _heads(v, dv)
    T = qh.shape[1]
    bh = np.ascontiguousarray(bh_idx, dtype=np.int64)
    tt = np.ascontiguousarray(t_idx, dtype=np.int64)
    assert bh.shape == tt.shape and bh.ndim == 1
    assert (bh >= 0).all() and (bh < qh.shape[0]).all() and (tt >= 0).all() and (tt < T).all()
    n = bh.shape[0]
    y = np.zeros((n, dv))
    den = np.zeros(n)
    Lp = ctypes.POINTER(ctypes.c_long)
    lib.kata_oracle_forward_mg_rows(_p(qh), _p(kh), _p(vh), T, dk, dv, int(g),
                                    bh.ctypes.data_as(Lp), tt.ctypes.data_as(Lp), n, _p(y),
                                    _p(den), _threads(nthreads))
    return y


def state_mg(k, v, g, n=None, nthreads=None):
    """The Mg state in the dense layout: S[..., i*dk+j, e] = sum_{s<n} k_si k_sj v_se
    and Z[..., i, j] = sum_{s<n} k_si k_sj for i, j in the same block, else 0."""
    lib = _load()
    dk, dv = k.shape[-1], v.shape[-1]
    _check_g(dk, g)
    kh, lead = _heads(k, dk)
    vh, _ = _heads(v, dv)
    BH, T = kh.shape[0], kh.shape[1]
    n = T if n is None else int(n)
    assert 0 <= n <= T
    S = np.zeros((BH, dk * dk, dv))
    Z = np.zeros((BH, dk, dk))
    lib.kata_oracle_state_mg(_p(kh), _p(vh), BH, T, n, dk, dv, int(g), _p(S), _p(Z),
                             _threads(nthreads))
    return S.reshape(*lead, dk * dk, dv), Z.reshape(*lead, dk, dk)


def forward_mg_recurrent(q, k, v, g, nthreads=None):
    lib = _load()
    dk, dv = q.shape[-1], v.shape[-1]
    _check_g(dk, g)
    qh, lead = _heads(q, dk)
    kh, _ = _heads(k, dk)
    vh, _ = _heads(v, dv)
    BH, T = qh.shape[0], qh.shape[1]
    y = np.zeros((BH, T, dv))
    lib.kata_oracle_forward_mg_recurrent(_p(qh), _p(kh), _p(vh), _p(y), BH, T, dk, dv, int(g),
                                         _threads(nthreads))
    return y.reshape(*lead, T, dv)


def decode_step_mg(q, k, v, S, Z, g):
    """One Mg step on copies of (S, Z); q,k: [BH, dk]; v: [BH, dv].  Returns (y, S', Z', den)."""
    lib = _load()
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    BH, dk = q.shape
    dv = v.shape[1]
    _check_g(dk, g)
    S2 = _f64(S).reshape(BH, dk * dk, dv).copy()
    Z2 = _f64(Z).reshape(BH, dk, dk).copy()
    y = np.zeros((BH, dv))
    den = np.zeros(BH)
    lib.kata_oracle_decode_step_mg(_p(q), _p(k), _p(v), _p(S2), _p(Z2), _p(y), _p(den), BH, dk,
                                   dv, int(g))
    return y, S2, Z2, den
