"""Seeded input generator (host path): determinism, shapes, rounding (no GPU)."""
import numpy as np
import torch

from kernelized_linear_attention_fwd_b200 import inputs


def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(0)
    x = np.concatenate([g.standard_normal(100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40], np.float32)])
    ours = inputs.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = inputs.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generator_is_deterministic_and_per_head():
    q1, k1, v1 = inputs.make_qkv(2, 3, 50, 8, 8, "bf16", seed=0)
    q2, k2, v2 = inputs.make_qkv(2, 3, 50, 8, 8, "bf16", seed=0)
    assert np.array_equal(q1, q2) and np.array_equal(k1, k2) and np.array_equal(v1, v2)
    # one head regenerated alone gives the same bits
    qa, ka, va = inputs._one_head((0, 0, 1, 2, 50, 8, 8, "unit", "bf16"))
    assert np.array_equal(qa, q1[1, 2]) and np.array_equal(va, v1[1, 2])
    q3, _, _ = inputs.make_qkv(2, 3, 50, 8, 8, "bf16", seed=1)
    assert not np.array_equal(q1, q3)


def test_unit_rows_and_value_distribution():
    q, k, v = inputs.make_qkv(1, 2, 4000, 16, 16, "f32", seed=0)
    nq = np.linalg.norm(q.astype(np.float64), axis=-1)
    assert np.allclose(nq, 1.0, atol=1e-6)
    vv = v.astype(np.float64)
    assert abs(vv.mean()) < 0.02 and abs(vv.std() - 1.0) < 0.02


def test_named_workloads():
    w = inputs.WORKLOADS["tiny_B1H1_T256_d16_f32"]
    q, k, v = inputs.make_workload(w)
    assert q.shape == (1, 1, 256, 16) and q.dtype == np.float32
    plan_w = inputs.WORKLOADS["recall_decode_B64H16_T32768_d64_bf16"]
    pos, pick = inputs.recall_decode_plan(plan_w)
    assert pos.shape == (4096,) and len(np.unique(pos)) == 4096 and pos.max() < 32768
    assert pick.shape == (1024, 64, 16) and pick.max() < 4096


def test_unnormalised_recipes():
    # raw: the N(0, 1) rows as drawn (norms near sqrt(d)); spread: unit
    # directions with norms 2^e, e uniform in [-6, 6]; v is the same draw in
    # every recipe, and the directions of spread rows are those of unit rows
    qr, kr, vr = inputs.make_qkv(1, 2, 4000, 64, 64, "f32", seed=3, qk="raw")
    qs, ks, vs = inputs.make_qkv(1, 2, 4000, 64, 64, "f32", seed=3, qk="spread")
    qu, ku, vu = inputs.make_qkv(1, 2, 4000, 64, 64, "f32", seed=3, qk="unit")
    assert np.array_equal(vr, vu) and np.array_equal(vs, vu)
    nr = np.linalg.norm(kr.astype(np.float64), axis=-1)
    assert abs(nr.mean() - 8.0) < 0.2
    ns = np.log2(np.linalg.norm(ks.astype(np.float64), axis=-1))
    assert ns.min() >= -6.001 and ns.max() <= 6.001 and ns.max() - ns.min() > 11.5
    assert abs(ns.mean()) < 0.3
    cos = (ks.astype(np.float64) * ku).sum(-1) / np.linalg.norm(ks.astype(np.float64), axis=-1)
    assert np.allclose(cos, 1.0, atol=1e-5)
    try:
        inputs.make_qkv(1, 1, 4, 8, 8, "f32", qk="bogus")
    except ValueError:
        pass
    else:
        raise AssertionError("unknown recipe accepted")
