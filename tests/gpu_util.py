"""Helpers shared by the GPU parity tests: device transfer of the generator's
bits, the error metric, and the sampled-row plan for long sequences."""
from __future__ import annotations

import numpy as np

from kernelized_linear_attention_fwd_b200 import inputs

# Tolerances of the parity bar: max row-normwise relative error
#   err = max_rows ||y - y_ref||_inf / ||y_ref||_inf
# against the fp64 oracle on the same input bits.  fp32 inputs: 1e-4; bf16
# inputs with fp32 accumulation: 2e-2.  A row whose reference is exactly zero
# (zero denominator) must be exactly zero.
TOL = {"f32": 1e-4, "bf16": 2e-2}

# Worst-case bound of an exported state entry: |S - S_ref| <= u * R1 (+1e-6),
# with R1 = sum_s |k_si k_sj v_se| the state of |k|, |v| (for Z, v = 1).
# bf16: every product k_si k_sj is rounded once to bf16 (8 significant bits,
# unit roundoff 2^-8) before the fp32 accumulation, so |error| <= 2^-8 R1 even
# if every rounding went the same way; fp32 rounds only in fp32 (2^-16 R1
# covers T <= 2^16 tokens of accumulation error).  This bound grows like T
# while the entries grow like sqrt(T), so it is kept only as an outer check.
STATE_BOUND = {"f32": 2.0 ** -16, "bf16": 2.0 ** -8}

# The bound the state tests enforce for bf16 inputs, scaled to the expected
# error.  Rounding products to nearest gives errors delta_s p_s with
# |delta_s| <= u = 2^-8, zero mean, independent across tokens, so the error of
# an entry, E = sum_s delta_s p_s v_se, has standard deviation at most
# (u / sqrt(3)) R2 with R2 = sqrt(sum_s (k_si k_sj v_se)^2) (a uniform delta
# has standard deviation u / sqrt(3); round to nearest is tighter, about
# 0.43 u).  The test allows STATE_SIGMAS of those, plus 2^-16 R1 for the fp32
# sums (in the tensor cores and across segments) and 1e-6 absolute.  Six
# conservative standard deviations are about eight true ones: no rounding
# pattern of a sound kernel reaches them on any entry, while a 1% error on a
# tile of entries exceeds them on every entry larger than about 1.4 R2.
# The rounding is not exactly zero-mean, though: the low bits of a product of
# two 8-bit significands are not uniform (squares most of all), so bf16(p) / p
# - 1 has a small mean, +1.2e-4 for squares k_i^2 and -4e-5 for products of
# independent entries (measured over 2e6 samples; tests/test_state_bound.py).
# That bias adds mean * S to an entry, which grows like T where the entry is a
# sum of positive terms: the diagonal of Z, sum_s k_si^2.  The bound carries
# BIAS_BF16 |S_ref| for it, twice the larger measured mean.
STATE_SIGMAS = 6.0
U_BF16 = 2.0 ** -8
BIAS_BF16 = 2.0 ** -12


def _state_fn(oracle_mod, g):
    """The oracle's state of one factor (g = 1) or of KATA-Mg with g factors."""
    if g == 1:
        return oracle_mod.state
    return lambda k, v: oracle_mod.state_mg(k, v, g)


def state_bounds(oracle_mod, k64, v64, dtype, g=1, ref=None):
    """Per-entry bounds (S, Z) of an exported state against the fp64 oracle's:
    the expected-error bound above for bf16 (ref: the oracle's (S, Z), computed
    here when not given), 2^-16 R1 for fp32."""
    state = _state_fn(oracle_mod, g)
    S1, Z1 = state(np.abs(k64), np.abs(v64))
    if dtype != "bf16":
        u = STATE_BOUND[dtype]
        return u * S1 + 1e-6, u * Z1 + 1e-6
    S, Z = state(k64, v64) if ref is None else ref
    S2, Z2 = state(k64 * k64, v64 * v64)
    c = STATE_SIGMAS * U_BF16 / np.sqrt(3.0)
    return (c * np.sqrt(S2) + BIAS_BF16 * np.abs(S) + 2.0 ** -16 * S1 + 1e-6,
            c * np.sqrt(Z2) + BIAS_BF16 * np.abs(Z) + 2.0 ** -16 * Z1 + 1e-6)


def assert_state_close(oracle_mod, Sg, Zg, k64, v64, dtype, g=1):
    """Exported state (numpy S [..., d*d, dv], Z [..., d, d]) against the fp64
    oracle's state of the same tokens (g > 1: of KATA-Mg with g factors, zeros
    across factors): state_bounds, and the worst-case STATE_BOUND as an outer
    check.  Returns the largest error / bound."""
    state = _state_fn(oracle_mod, g)
    S, Z = state(k64, v64)
    bS, bZ = state_bounds(oracle_mod, k64, v64, dtype, g, ref=(S, Z))
    eS, eZ = np.abs(Sg - S), np.abs(Zg - Z)
    assert np.all(eS <= bS), f"state entry off by {np.max(eS / bS):.2f} x its bound"
    assert np.all(eZ <= bZ), f"Z entry off by {np.max(eZ / bZ):.2f} x its bound"
    Sabs, Zabs = state(np.abs(k64), np.abs(v64))
    u = STATE_BOUND[dtype]
    assert np.all(eS <= u * Sabs + 1e-6) and np.all(eZ <= u * Zabs + 1e-6)
    return float(max(np.max(eS / bS), np.max(eZ / bZ)))


def to_device(a: np.ndarray, dtype: str):
    import torch

    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def from_device(t) -> np.ndarray:
    """Device tensor (bf16 or fp32) -> exact float64 numpy values."""
    import torch

    if t.dtype == torch.bfloat16:
        bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        return inputs.bf16_bits_to_f32(bits).astype(np.float64)
    return t.detach().cpu().numpy().astype(np.float64)


def row_err(y: np.ndarray, yref: np.ndarray) -> float:
    """max over rows of ||y - yref||_inf / ||yref||_inf (inf for a wrong zero row)."""
    y = np.asarray(y, np.float64).reshape(-1, yref.shape[-1])
    yref = np.asarray(yref, np.float64).reshape(-1, yref.shape[-1])
    if not np.isfinite(y).all():
        return float("inf")
    scale = np.abs(yref).max(axis=1)
    zero = scale == 0
    if zero.any() and np.abs(y[zero]).max() != 0:
        return float("inf")
    if (~zero).sum() == 0:
        return 0.0
    d = np.abs(y[~zero] - yref[~zero]).max(axis=1) / scale[~zero]
    return float(d.max())


def sample_rows(T: int, C: int, L: int, n_uniform: int = 512, n_bound: int = 64, seed: int = 0):
    """Row indices checked on long sequences: every row of the first and last
    chunk, the rows on both sides of 64 seeded chunk boundaries and of 64
    seeded segment boundaries, and n_uniform seeded rows."""
    g = np.random.default_rng(seed)
    rows = set(range(0, min(C, T)))
    rows |= set(range(max(0, T - C), T))
    nc = (T + C - 1) // C
    for c in g.integers(1, max(2, nc), size=n_bound):
        rows |= {int(c) * C - 1, int(c) * C}
    ns = (T + L - 1) // L
    if ns > 1:
        for s in g.integers(1, ns, size=n_bound):
            rows |= {int(s) * L - 1, int(s) * L}
    rows |= set(int(x) for x in g.integers(0, T, size=n_uniform))
    return np.array(sorted(r for r in rows if 0 <= r < T), dtype=np.int64)
