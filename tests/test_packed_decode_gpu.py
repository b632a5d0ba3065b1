"""GPU parity of the packed decode-state layout (rows i <= j) against the fp64 oracle.

- kata_state_pack / kata_state_unpack: the packed rows are the dense rows
  (i, j), i <= j, bit for bit, and unpacking a symmetric dense state gives it
  back bit for bit.
- kata_decode_step_packed: a forward over T tokens, its state packed, then n
  packed decode steps give rows T .. T+n-1 of the oracle's forward over
  T + n tokens; the unpacked final state is the oracle's state within the
  state bound; and packed and dense decode agree on every head count that
  changes the cluster split (1 to 1024 heads).
Tolerances: tests/gpu_util.py.
"""
from __future__ import annotations

import numpy as np
import pytest

from kernelized_linear_attention_fwd_b200 import inputs
from tests.gpu_util import TOL, assert_state_close, from_device, row_err, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # collected on CPU machines, run only with a GPU
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import kernelized_linear_attention_fwd_b200 as K  # noqa: E402
from kernelized_linear_attention_fwd_b200.csrc import build as kbuild  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()
    K.load_library()
    yield
    assert K.kata_get_device_status() == 0


def dev(x, dtype):
    return to_device(np.ascontiguousarray(x), dtype)


def prefill(q, k, v, dtype):
    B, H, _, d = q.shape
    so = torch.empty((B, H, d * d, d), dtype=torch.float32, device="cuda")
    zo = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    K.kata_chunked_forward(dev(q, dtype), dev(k, dtype), dev(v, dtype), C=64, state_out=so,
                           z_out=zo)
    return so, zo


@pytest.mark.parametrize("d", [16, 32, 64])
def test_pack_unpack_exact(d):
    q, k, v = inputs.make_qkv(2, 3, 700, d, d, "f32", seed=d)
    S, Z = prefill(q, k, v, "f32")
    Sp, Zp = K.kata_state_pack(S, Z)
    S2, Z2 = K.kata_state_unpack(Sp, Zp)
    torch.cuda.synchronize()
    ii, jj = np.triu_indices(d)  # row-major i outer: the packed order
    Sn, Zn = S.cpu().numpy(), Z.cpu().numpy()
    assert np.array_equal(Sp.cpu().numpy(), Sn[:, :, ii * d + jj])
    assert np.array_equal(Zp.cpu().numpy(), Zn.reshape(2, 3, d * d)[:, :, ii * d + jj])
    assert torch.equal(S2, S) and torch.equal(Z2, Z)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64])
def test_packed_decode_steps(oracle_mod, dtype, d):
    """forward(T), pack, n packed steps == rows T..T+n-1 of forward(T + n)."""
    T, n = 1100, 6
    q, k, v = inputs.make_qkv(2, 2, T + n, d, d, dtype, seed=200 + d)
    S, Z = prefill(q[:, :, :T], k[:, :, :T], v[:, :, :T], dtype)
    Sp, Zp = K.kata_state_pack(S, Z)
    ys = []
    for s in range(n):
        xs = [dev(x[:, :, T + s], dtype) for x in (q, k, v)]
        ys.append(from_device(K.kata_decode_step_packed(*xs, Sp, Zp)))
    torch.cuda.synchronize()
    q64, k64, v64 = (inputs.widen(x, dtype) for x in (q, k, v))
    yref = oracle_mod.forward(q64, k64, v64)[:, :, T:]
    assert row_err(np.stack(ys, axis=2), yref) <= TOL[dtype]
    S2, Z2 = K.kata_state_unpack(Sp, Zp)
    assert_state_close(oracle_mod, from_device(S2), from_device(Z2), k64, v64, dtype)


@pytest.mark.parametrize("BH", [1, 8, 37, 148, 1024])
@pytest.mark.parametrize("d", [16, 32, 64])
def test_packed_matches_dense_at_every_split(BH, d):
    # random symmetric states: the cluster split changes with the head count
    g = torch.Generator(device="cuda")
    g.manual_seed(BH * 100 + d)
    S = torch.randn((1, BH, d, d, d), generator=g, device="cuda")
    S = (S + S.transpose(2, 3)).reshape(1, BH, d * d, d).contiguous()
    Z = torch.randn((1, BH, d, d), generator=g, device="cuda")
    Z = Z @ Z.transpose(-1, -2)
    Z = 0.5 * (Z + Z.transpose(-1, -2))  # exactly symmetric, as every state the library writes
    q, k, v = (torch.randn((1, BH, d), generator=g, device="cuda") for _ in range(3))
    Sp, Zp = K.kata_state_pack(S, Z)
    yd = K.kata_decode_step(q, k, v, S, Z)
    yp = K.kata_decode_step_packed(q, k, v, Sp, Zp)
    S2, Z2 = K.kata_state_unpack(Sp, Zp)
    torch.cuda.synchronize()
    assert row_err(from_device(yp), from_device(yd)) <= 1e-4
    torch.testing.assert_close(S2, S, rtol=1e-6, atol=1e-6)
    torch.testing.assert_close(Z2, Z, rtol=1e-6, atol=1e-5)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_packed_zero_denominator(dtype):
    d, BH = 64, 4
    q, k, v = inputs.make_qkv(1, BH, 300, d, d, dtype, seed=3)
    S, Z = prefill(q, k, v, dtype)
    Sp, Zp = K.kata_state_pack(S, Z)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    qz = torch.zeros((1, BH, d), dtype=tdt, device="cuda")
    y = K.kata_decode_step_packed(qz, dev(k[:, :, 0], dtype), dev(v[:, :, 0], dtype), Sp, Zp)
    torch.cuda.synchronize()
    assert torch.all(y == 0)
