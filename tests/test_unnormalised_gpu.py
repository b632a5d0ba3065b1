"""GPU parity on unnormalised queries and keys, through every entry point.

The feature psi(u) = u u^T (gist.science summary, Technical summary 2.2) needs
no normalisation, and the public calls accept any q and k.  The named
workloads all draw unit rows, so these cases cover the rest of the range:
"raw" rows as drawn from N(0, 1) (norms near sqrt(d)), and "spread" rows, unit
directions with norms 2^e, e uniform in [-6, 6], so weights (q.k)^2 of one
query span about 2^24 across its keys.  This exercises the bf16 range of the
squared scores and of the split hi + lo normaliser on the tensor-core path,
and the fp32 sums of the CUDA-core path.  Same oracle and bars as the other
parity tests (tests/gpu_util.py).
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

RECIPES = ("raw", "spread")
# (dtype, d): the tensor-core path at d = 64 and below (heads read as 64; d = 32 on the
# two-factor state layout), the CUDA-core path
PATHS = (("bf16", 64), ("bf16", 32), ("f32", 64), ("f32", 16))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()
    K.load_library()
    yield
    assert K.kata_get_device_status() == 0


def dev(x, dtype):
    return to_device(np.ascontiguousarray(x), dtype)


def f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def widen_all(dtype, *xs):
    return tuple(inputs.widen(x, dtype) for x in xs)


@pytest.mark.parametrize("qk", RECIPES)
@pytest.mark.parametrize("dtype,d", PATHS)
def test_chunked_forward_and_state(oracle_mod, qk, dtype, d):
    # three segments with a ragged tail, state exported
    T = 2 * 1024 + 701
    q, k, v = inputs.make_qkv(1, 2, T, d, d, dtype, seed=31 + d, qk=qk)
    so = torch.empty((1, 2, d * d, d), dtype=torch.float32, device="cuda")
    zo = torch.empty((1, 2, d, d), dtype=torch.float32, device="cuda")
    out = K.kata_chunked_forward(dev(q, dtype), dev(k, dtype), dev(v, dtype), C=64, state_out=so,
                                 z_out=zo)
    torch.cuda.synchronize()
    q64, k64, v64 = widen_all(dtype, q, k, v)
    err = row_err(from_device(out), oracle_mod.forward(q64, k64, v64))
    assert err <= TOL[dtype], f"row-normwise error {err:.3e}"
    assert_state_close(oracle_mod, from_device(so), from_device(zo), k64, v64, dtype)


@pytest.mark.parametrize("qk", RECIPES)
@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 64), ("f32", 32)])
def test_quadratic_forward(oracle_mod, qk, dtype, d):
    T = 1500
    q, k, v = inputs.make_qkv(1, 2, T, d, d, dtype, seed=57 + d, qk=qk)
    out = K.kata_quadratic_forward(dev(q, dtype), dev(k, dtype), dev(v, dtype))
    torch.cuda.synchronize()
    err = row_err(from_device(out), oracle_mod.forward(*widen_all(dtype, q, k, v)))
    assert err <= TOL[dtype], f"row-normwise error {err:.3e}"


@pytest.mark.parametrize("qk", RECIPES)
@pytest.mark.parametrize("dtype,d", PATHS)
def test_forward_then_decode_steps(oracle_mod, qk, dtype, d):
    """forward(T) + n decode steps (dense and packed layouts) == rows T.. of forward(T + n)."""
    T, n = 1300, 5
    q, k, v = inputs.make_qkv(1, 2, T + n, d, d, dtype, seed=77 + d, qk=qk)
    so = torch.empty((1, 2, d * d, d), dtype=torch.float32, device="cuda")
    zo = torch.empty((1, 2, d, d), dtype=torch.float32, device="cuda")
    K.kata_chunked_forward(dev(q[:, :, :T], dtype), dev(k[:, :, :T], dtype),
                           dev(v[:, :, :T], dtype), C=64, state_out=so, z_out=zo)
    sp, zp = K.kata_state_pack(so, zo)
    ys, yp = [], []
    for s in range(n):
        xs = [dev(x[:, :, T + s], dtype) for x in (q, k, v)]
        ys.append(from_device(K.kata_decode_step(*xs, so, zo)))
        yp.append(from_device(K.kata_decode_step_packed(*xs, sp, zp)))
    torch.cuda.synchronize()
    yref = oracle_mod.forward(*widen_all(dtype, q, k, v))[:, :, T:]
    assert row_err(np.stack(ys, axis=2), yref) <= TOL[dtype]
    assert row_err(np.stack(yp, axis=2), yref) <= TOL[dtype]


@pytest.mark.parametrize("qk", RECIPES)
@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 64), ("f32", 32)])
def test_forward_from_state_and_state_only(oracle_mod, qk, dtype, d):
    # history of Th tokens given as its state (computed by the state-only call),
    # then the forward of the next Tb tokens continuing from it
    Th, Tb = 2100, 1300
    q, k, v = inputs.make_qkv(1, 2, Th + Tb, d, d, dtype, seed=91 + d, qk=qk)
    q64, k64, v64 = widen_all(dtype, q, k, v)
    S0, Z0 = K.kata_chunked_state(dev(k[:, :, :Th], dtype), dev(v[:, :, :Th], dtype), C=64)
    torch.cuda.synchronize()
    assert_state_close(oracle_mod, from_device(S0), from_device(Z0), k64[:, :, :Th],
                       v64[:, :, :Th], dtype)
    blk = [dev(x[:, :, Th:], dtype) for x in (q, k, v)]
    so = torch.empty_like(S0)
    zo = torch.empty_like(Z0)
    out = K.kata_chunked_forward_from_state(*blk, S0, Z0, C=64, state_out=so, z_out=zo)
    torch.cuda.synchronize()
    yref = oracle_mod.forward(q64, k64, v64)[:, :, Th:]
    err = row_err(from_device(out), yref)
    assert err <= TOL[dtype], f"row-normwise error {err:.3e}"
    assert_state_close(oracle_mod, from_device(so), from_device(zo), k64, v64, dtype)
    # the same history given as the oracle's exact state
    S0o, Z0o = oracle_mod.state(k64[:, :, :Th], v64[:, :, :Th])
    out2 = K.kata_chunked_forward_from_state(*blk, f32(S0o), f32(Z0o), C=64)
    torch.cuda.synchronize()
    assert row_err(from_device(out2), yref) <= TOL[dtype]
