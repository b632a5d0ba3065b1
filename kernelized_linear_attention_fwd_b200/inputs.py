"""Seeded synthetic inputs for the KATA causal forward and decode.

This module holds none of the method's arithmetic: it draws random numbers,
normalises rows, and rounds to the storage type.  Both the CUDA path (tests,
benchmark) and the fp64 oracle consume exactly the bits it produces.

Recipe (all workloads): q, k i.i.d. N(0, 1), each row divided by its L2 norm
in float64 (the small bf16 workload first scales by 1/sqrt(d), which the
normalisation undoes, kept for fidelity to its description); v i.i.d. N(0, 1).
Two unnormalised recipes exercise the dynamic range of the public calls (the
feature u u^T needs no normalisation): qk="raw" keeps the N(0, 1) rows as
drawn, qk="spread" gives each unit row a norm 2^e with e uniform in [-6, 6].
Values are rounded float64 -> float32 (round to nearest even) and, for bf16,
float32 -> bf16 (round to nearest even on the bit pattern).

Host path (numpy): one PCG64 stream per (seed, tag, b, h) head, so that any
head can be regenerated alone; draws in the order q, k, v.
Device path (torch, for the 64 x 16 head decode workload whose prefill is
6.4e9 values): a seeded ``torch.Generator`` on the device; the oracle is then
fed the same bits copied back for the heads it checks.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

# ---------------------------------------------------------------------------
# Named workloads (sizes of the pages' / benchmark's configurations).
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int
    C: int
    dtype: str            # "f32" or "bf16"
    qk: str = "unit"      # "unit" | "scaled_unit" | "raw" | "spread"
    seed: int = 0
    decode_steps: int = 0  # > 0: recall-shaped decode workload
    n_pairs: int = 0
    chunk_sweep: tuple = field(default_factory=tuple)
    t_sweep: tuple = field(default_factory=tuple)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_B1H1_T256_d16_f32", 1, 1, 256, 16, 64, "f32"),
        Workload("small_B2H4_T4096_d32_bf16", 2, 4, 4096, 32, 64, "bf16", qk="scaled_unit"),
        Workload("lm340m_B4H16_T16384_d64_bf16", 4, 16, 16384, 64, 64, "bf16"),
        Workload("long_B1H8_T131072_d64_bf16", 1, 8, 131072, 64, 64, "bf16",
                 chunk_sweep=(64, 128, 256), t_sweep=(8192, 32768, 131072)),
        Workload("recall_decode_B64H16_T32768_d64_bf16", 64, 16, 32768, 64, 64, "bf16",
                 decode_steps=1024, n_pairs=4096),
    ]
}

# ---------------------------------------------------------------------------
# Rounding helpers (storage formats only).
# ---------------------------------------------------------------------------


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + (((u >> 16) & 1) + 0x7FFF)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array (uint16 bf16 bits or float32) -> exact float64 values."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _store(x64: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x64.astype(np.float32)
    return f32_to_bf16_bits(x32) if dtype == "bf16" else x32


def _unit_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
    n[n == 0] = 1.0
    return x / n


# ---------------------------------------------------------------------------
# Host generator.
# ---------------------------------------------------------------------------


def head_rng(seed: int, tag: int, b: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, b, h])))


def _one_head(args):
    seed, tag, b, h, T, dk, dv, qk, dtype = args
    g = head_rng(seed, tag, b, h)
    q = g.standard_normal((T, dk))
    k = g.standard_normal((T, dk))
    v = g.standard_normal((T, dv))
    if qk == "scaled_unit":
        q = q / math.sqrt(dk)
        k = k / math.sqrt(dk)
    if qk in ("unit", "scaled_unit", "spread"):
        q = _unit_rows(q)
        k = _unit_rows(k)
    if qk == "spread":
        # row norms 2^e, e ~ U[-6, 6] (drawn after v, so q, k, v keep their draws)
        q = q * np.exp2(g.uniform(-6.0, 6.0, size=(T, 1)))
        k = k * np.exp2(g.uniform(-6.0, 6.0, size=(T, 1)))
    elif qk not in ("unit", "scaled_unit", "raw"):
        raise ValueError(f"unknown q/k recipe {qk!r}")
    return _store(q, dtype), _store(k, dtype), _store(v, dtype)


def make_qkv(B, H, T, dk, dv, dtype="bf16", seed=0, qk="unit", tag=0, threads=None):
    """Host arrays q, k [B,H,T,dk] and v [B,H,T,dv] in storage format.

    bf16 arrays are uint16 bit patterns; f32 arrays are float32.
    """
    st = np.uint16 if dtype == "bf16" else np.float32
    q = np.empty((B, H, T, dk), st)
    k = np.empty((B, H, T, dk), st)
    v = np.empty((B, H, T, dv), st)
    jobs = [(seed, tag, b, h, T, dk, dv, qk, dtype) for b in range(B) for h in range(H)]
    with ThreadPoolExecutor(max_workers=threads or 8) as ex:
        for (a, _b, _c), (_, _, b, h, *_r) in zip(ex.map(_one_head, jobs), jobs):
            q[b, h], k[b, h], v[b, h] = a, _b, _c
    return q, k, v


def make_workload(w: Workload, T=None, tag=0):
    """Host q, k, v of a named workload (optionally with another T)."""
    return make_qkv(w.B, w.H, w.T if T is None else T, w.d, w.d, w.dtype, w.seed, w.qk, tag)


# ---------------------------------------------------------------------------
# Device generator (torch), for workloads too large to draw on the host.
# ---------------------------------------------------------------------------


def make_qkv_device(B, H, T, dk, dv, seed=0, device="cuda", qk="unit", chunk_heads=64):
    """bf16 q, k, v drawn on the device with a seeded torch.Generator.

    Rows are normalised in float64, rounded to float32, then to bf16
    (torch's round-to-nearest-even), chunk by chunk of heads to bound memory.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    out = []
    for d, unit in ((dk, qk == "unit"), (dk, qk == "unit"), (dv, False)):
        t = torch.empty((B * H, T, d), dtype=torch.bfloat16, device=device)
        for h0 in range(0, B * H, chunk_heads):
            h1 = min(B * H, h0 + chunk_heads)
            x = torch.randn((h1 - h0, T, d), generator=g, device=device, dtype=torch.float32)
            if unit:
                x64 = x.double()
                x = (x64 / x64.norm(dim=-1, keepdim=True)).float()
            t[h0:h1] = x.to(torch.bfloat16)
        out.append(t.view(B, H, T, d))
    return tuple(out)


def recall_decode_plan(w: Workload, seed=None):
    """Positions of the marked key-value pairs and, per decode step and head,
    which marked pair the step's query repeats (host, numpy, seeded)."""
    g = head_rng(w.seed if seed is None else seed, 7, 0, 0)
    pair_pos = np.sort(g.choice(w.T, size=w.n_pairs, replace=False)).astype(np.int64)
    pick = g.integers(0, w.n_pairs, size=(w.decode_steps, w.B, w.H)).astype(np.int64)
    return pair_pos, pick
