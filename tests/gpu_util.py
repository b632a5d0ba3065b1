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

# Bound of an exported state entry: |S - S_ref| <= u * B (+1e-6), with
# B = sum_s |k_si k_sj v_se| the state of |k|, |v| (for Z, v = 1).  bf16: the
# tensor-core path rounds each product k_si k_sj to bf16 (unit roundoff 2^-9)
# before the fp32 accumulation, so 2^-9 B plus the fp32 accumulation stays
# within 2^-8 B; fp32 rounds only in fp32 (2^-16 B covers T <= 2^16 tokens of
# random-walk accumulation error).
STATE_BOUND = {"f32": 2.0 ** -16, "bf16": 2.0 ** -8}


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
