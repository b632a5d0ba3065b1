"""Exact rational brute force of the KATA causal forward — TEST INFRASTRUCTURE ONLY.

Pure Python ``fractions.Fraction`` arithmetic on small integer (or rational)
inputs: the weights (q_t.k_s)^2, the numerator and the denominator are exact,
so the fp64 oracle must agree with this to within one rounding of the final
division.  Written independently of ``kata_oracle.c`` (different language,
different loop order: the dot products are formed first for the whole row).

Definition followed: gist.science summary of "Kernelized Linear Attention:
Breaking the Capacity Wall with Symmetric Cones", Technical summary 2.2
(psi(u) = u u^T, so the weight is the squared inner product) and 2.1 (the
normalised denominator; the current token is part of the convex gate).
"""
from __future__ import annotations

from fractions import Fraction


def forward_exact(q, k, v):
    """q, k: T lists of dk numbers; v: T lists of dv numbers (one head).

    Returns y as a T x dv list of Fractions (0 where the denominator is 0).
    """
    T = len(q)
    dv = len(v[0]) if T else 0
    qf = [[Fraction(x) for x in row] for row in q]
    kf = [[Fraction(x) for x in row] for row in k]
    vf = [[Fraction(x) for x in row] for row in v]
    out = []
    for t in range(T):
        weights = [sum(a * b for a, b in zip(qf[t], kf[s])) ** 2 for s in range(t + 1)]
        den = sum(weights, Fraction(0))
        if den == 0:
            out.append([Fraction(0)] * dv)
            continue
        out.append([sum((w * vf[s][e] for s, w in enumerate(weights)), Fraction(0)) / den
                    for e in range(dv)])
    return out


def weights_exact(q, k):
    """Lower-triangular exact weight matrix W[t][s] = (q_t.k_s)^2 for s <= t."""
    T = len(q)
    return [[sum(Fraction(a) * Fraction(b) for a, b in zip(q[t], k[s])) ** 2 for s in range(t + 1)]
            for t in range(T)]


def forward_exact_mg(q, k, v, g):
    """KATA-Mg (gist.science summary 2.3, "Variantes"; reading: a product of g
    rank-one PSD cones on consecutive blocks of dk / g coordinates) in exact
    arithmetic: weight sum_m (q_t^(m) . k_s^(m))^2.  Same arguments as
    forward_exact plus g, which must divide dk."""
    T = len(q)
    dv = len(v[0]) if T else 0
    dk = len(q[0]) if T else 0
    if g < 1 or dk % g:
        raise ValueError("g must divide dk")
    p = dk // g
    qf = [[Fraction(x) for x in row] for row in q]
    kf = [[Fraction(x) for x in row] for row in k]
    vf = [[Fraction(x) for x in row] for row in v]
    out = []
    for t in range(T):
        weights = []
        for s in range(t + 1):
            w = Fraction(0)
            for m in range(g):
                dot = sum(qf[t][i] * kf[s][i] for i in range(m * p, (m + 1) * p))
                w += dot * dot
            weights.append(w)
        den = sum(weights, Fraction(0))
        if den == 0:
            out.append([Fraction(0)] * dv)
            continue
        out.append([sum((w * vf[s][e] for s, w in enumerate(weights)), Fraction(0)) / den
                    for e in range(dv)])
    return out
