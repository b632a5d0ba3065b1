"""kata_chunked_forward_noalloc: the forward for callers that cannot allocate
device memory (a host framework that owns all device memory through its own
pool, a loop whose memory is fixed up front).  Its scratch is a static device
array inside libkata instead of a caller-provided workspace.

Checked through the C ABI: two calls in a row (different inputs, so the second
call runs on an array that still holds the first call's contents) give the
same output and final state as kata_chunked_forward with a workspace, within
the parity tolerance; a problem larger than the array is refused on the host.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

from kernelized_linear_attention_fwd_b200 import inputs
from tests.gpu_util import TOL, from_device, row_err, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import kernelized_linear_attention_fwd_b200 as K  # noqa: E402
from kernelized_linear_attention_fwd_b200 import binding  # noqa: E402
from kernelized_linear_attention_fwd_b200.csrc import build as kbuild  # noqa: E402


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return binding.load_library()


def _noalloc_call(lib, q, k, v, out, C, so=None, zo=None):
    B, H, T, d = q.shape
    code = binding.KATA_BF16 if q.dtype == torch.bfloat16 else binding.KATA_F32
    vp = ctypes.c_void_p
    st = lib.kata_chunked_forward_noalloc(
        vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()), vp(out.data_ptr()), B, H, T, d, d,
        C, code, vp(so.data_ptr()) if so is not None else None,
        vp(zo.data_ptr()) if zo is not None else None,
        vp(torch.cuda.current_stream().cuda_stream))
    return st


# bf16 d = 64, 32 and 16: the tensor-core route (heads below 64 read as 64
# by the tensor maps, on the two-factor state layout); fp32: the CUDA-core
# route.
@pytest.mark.parametrize("dtype,d,T,H", [("bf16", 64, 3000, 2), ("bf16", 32, 2000, 2),
                                         ("bf16", 16, 2000, 2), ("f32", 32, 2100, 3)])
def test_noalloc_matches_workspace_forward_twice(lib, dtype, d, T, H):
    B = 1
    code = binding.KATA_BF16 if dtype == "bf16" else binding.KATA_F32
    assert lib.kata_chunked_forward_workspace_bytes(B, H, T, d, d, 64, code) <= \
        binding.KATA_NOALLOC_SCRATCH_BYTES
    for call, seed in enumerate((101, 202)):
        qh, kh, vh = inputs.make_qkv(B, H, T, d, d, dtype, seed=seed)
        q, k, v = to_device(qh, dtype), to_device(kh, dtype), to_device(vh, dtype)
        # reference: the workspace entry point
        so_ref = torch.empty((B, H, d * d, d), dtype=torch.float32, device="cuda")
        zo_ref = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
        ref = K.kata_chunked_forward(q, k, v, C=64, state_out=so_ref, z_out=zo_ref)
        # no-alloc entry point, all buffers passed in by the caller
        out = torch.empty_like(ref)
        so = torch.empty_like(so_ref)
        zo = torch.empty_like(zo_ref)
        assert _noalloc_call(lib, q, k, v, out, 64, so, zo) == binding.KATA_OK, f"call {call}"
        torch.cuda.synchronize()
        assert K.kata_get_device_status() == 0
        y, yref = from_device(out), from_device(ref)
        assert row_err(y, yref) <= TOL[dtype], f"call {call}"
        s_ref = from_device(so_ref)
        assert np.abs(from_device(so) - s_ref).max() <= 1e-5 * np.abs(s_ref).max()
        # output only, no state export
        out2 = torch.empty_like(ref)
        assert _noalloc_call(lib, q, k, v, out2, 64) == binding.KATA_OK
        torch.cuda.synchronize()
        assert row_err(from_device(out2), yref) <= TOL[dtype]


def test_noalloc_refuses_problems_larger_than_its_scratch(lib):
    # 8 heads x 131072 tokens at d = 64 need far more than the static scratch;
    # the call must fail on the host, before any launch (pointers are never read).
    B, H, T, d = 1, 8, 131072, 64
    assert lib.kata_chunked_forward_workspace_bytes(B, H, T, d, d, 64, binding.KATA_BF16) > \
        binding.KATA_NOALLOC_SCRATCH_BYTES
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    vp = ctypes.c_void_p
    st = lib.kata_chunked_forward_noalloc(vp(x.data_ptr()), vp(x.data_ptr()), vp(x.data_ptr()),
                                          vp(y.data_ptr()), B, H, T, d, d, 64, binding.KATA_BF16,
                                          None, None, None)
    assert st == binding.KATA_ERR_WORKSPACE
