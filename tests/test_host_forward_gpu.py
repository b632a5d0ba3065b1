"""GPU parity of kata_chunked_forward_host (host q, k, v, out; heads in groups,
copies overlapped with the compute) against the fp64 oracle and against the
device-buffer forward on the same inputs.  Tolerances: tests/gpu_util.py."""
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


def host(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if dtype == "bf16" else
                         np.ascontiguousarray(a, dtype=np.float32))
    return (t.view(torch.bfloat16) if dtype == "bf16" else t).pin_memory()


@pytest.mark.parametrize("dtype,d,B,H,T,G", [
    ("bf16", 64, 1, 8, 5000, 0),     # the library's grouping
    ("bf16", 64, 1, 8, 5000, 1),     # one head per group: 8 groups through 2 slots
    ("bf16", 64, 2, 4, 2100, 3),     # a ragged last group
    ("bf16", 64, 1, 3, 700, 8),      # one group larger than the heads
    ("f32", 32, 2, 3, 1500, 2),      # the fp32 CUDA-core path
])
def test_host_forward(oracle_mod, dtype, d, B, H, T, G):
    q, k, v = inputs.make_qkv(B, H, T, d, d, dtype, seed=T + G)
    hq, hk, hv = (host(x, dtype) for x in (q, k, v))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    hout = torch.empty((B, H, T, d), dtype=tdt).pin_memory()
    so = torch.empty((B, H, d * d, d), dtype=torch.float32, device="cuda")
    zo = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    K.kata_chunked_forward_host(hq, hk, hv, hout, C=64, state_out=so, z_out=zo,
                                heads_per_group=G)
    torch.cuda.synchronize()
    y = from_device(hout)
    q64, k64, v64 = (inputs.widen(x, dtype) for x in (q, k, v))
    assert row_err(y, oracle_mod.forward(q64, k64, v64)) <= TOL[dtype]
    yd = from_device(K.kata_chunked_forward(to_device(q, dtype), to_device(k, dtype),
                                            to_device(v, dtype), C=64))
    assert row_err(y, yd) <= (1e-6 if dtype == "f32" else 2.0 ** -7)
    assert_state_close(oracle_mod, from_device(so), from_device(zo), k64, v64, dtype)


def test_host_forward_orders_after_the_stream():
    # inputs written on the device stream, then copied to pinned host buffers
    # without a host synchronisation: the host forward must see the values
    d, T = 64, 2048
    stream = torch.cuda.current_stream()
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    qd = torch.nn.functional.normalize(torch.randn((1, 2, T, d), generator=g, device="cuda"), dim=-1)
    kd = torch.nn.functional.normalize(torch.randn((1, 2, T, d), generator=g, device="cuda"), dim=-1)
    vd = torch.randn((1, 2, T, d), generator=g, device="cuda")
    qd, kd, vd = (x.to(torch.bfloat16) for x in (qd, kd, vd))
    hq, hk, hv = (torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in (qd, kd, vd))
    for h, x in zip((hq, hk, hv), (qd, kd, vd)):
        h.copy_(x, non_blocking=True)
    hout = torch.empty((1, 2, T, d), dtype=torch.bfloat16).pin_memory()
    # the host copies above are on `stream`; the forward's own copies wait for them
    K.kata_chunked_forward_host(hq, hk, hv, hout, C=64, stream=stream)
    torch.cuda.synchronize()
    yd = K.kata_chunked_forward(qd, kd, vd, C=64)
    torch.cuda.synchronize()
    assert row_err(from_device(hout), from_device(yd)) <= 2.0 ** -7
