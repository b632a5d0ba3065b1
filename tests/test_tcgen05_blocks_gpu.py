"""The sm_100a building blocks the tensor-core kernels rely on, checked on the
GPU against CPU arithmetic: the 128-byte TMA swizzle, shared-memory
descriptors (K-major and MN-major), the instruction descriptor, the layout of
an A operand written to tensor memory, and the accumulator read-back.  Also
the bounded-wait failure path: a wait that can never complete gives up after
the library's cycle budget, the kernel reports the time-out and returns, and
the context stays usable."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from tests.csrc import build_blocks  # noqa: E402


@pytest.fixture(scope="module")
def blocks():
    lib = ctypes.CDLL(build_blocks.build())
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.blocks_tma_raw.argtypes = [vp, vp, i32, vp]
    lib.blocks_mma_ss.argtypes = [vp, vp, vp, i32, i32, vp]
    lib.blocks_mma_ts.argtypes = [vp, vp, vp, i32, vp]
    lib.blocks_wait_timeout.argtypes = [vp, vp]
    return lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.fixture
def status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _bf16(shape, g):
    return torch.from_numpy(g.standard_normal(shape).astype(np.float32)).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("rows", [8, 64, 128, 256])
def test_tma_swizzle_128b(blocks, status, rows):
    src = torch.arange(rows * 64, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    src = src.reshape(rows, 64).cuda()
    dst = torch.zeros(rows * 64, dtype=torch.int16, device="cuda")
    assert blocks.blocks_tma_raw(_p(src), _p(dst), rows, _p(status)) == 0
    raw = dst.cpu().numpy().reshape(rows, 8, 8)       # [row][physical chunk][element]
    want = np.arange(rows * 64, dtype=np.int64).astype(np.int16).reshape(rows, 8, 8)
    for r in range(rows):
        for c in range(8):
            assert np.array_equal(raw[r, c ^ (r % 8)], want[r, c]), (r, c)


@pytest.mark.parametrize("N", [16, 64, 128, 256])
def test_mma_ss_k_major(blocks, status, N):
    g = np.random.default_rng(N)
    A, B = _bf16((128, 64), g), _bf16((N, 64), g)
    D = torch.empty((128, N), dtype=torch.float32, device="cuda")
    assert blocks.blocks_mma_ss(_p(A), _p(B), _p(D), N, 0, _p(status)) == 0
    ref = A.float() @ B.float().T
    torch.testing.assert_close(D, ref, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("N", [64, 128])
def test_mma_ss_b_mn_major(blocks, status, N):
    g = np.random.default_rng(7 + N)
    A, B = _bf16((128, 64), g), _bf16((64, N), g)   # B stored [K rows][N]
    D = torch.empty((128, N), dtype=torch.float32, device="cuda")
    assert blocks.blocks_mma_ss(_p(A), _p(B), _p(D), N, 1, _p(status)) == 0
    ref = A.float() @ B.float()
    torch.testing.assert_close(D, ref, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("KK", [16, 64, 128, 256])
def test_mma_a_from_tensor_memory(blocks, status, KK):
    g = np.random.default_rng(100 + KK)
    A, B = _bf16((128, KK), g), _bf16((KK, 64), g)
    D = torch.empty((128, 64), dtype=torch.float32, device="cuda")
    assert blocks.blocks_mma_ts(_p(A), _p(B), _p(D), KK, _p(status)) == 0
    ref = A.float() @ B.float()
    torch.testing.assert_close(D, ref, rtol=1e-5, atol=1e-4)


def test_bounded_wait_gives_up_and_the_context_stays_usable(blocks, status):
    out = torch.full((4,), -1, dtype=torch.int64, device="cuda")
    assert blocks.blocks_wait_timeout(_p(out), _p(status)) == 5  # the library's time-out code
    ok0, ok1, c0, c1 = out.cpu().tolist()
    assert ok0 == 0 and ok1 == 0            # neither wait claims its phase completed
    assert max(c0, c1) >= 1 << 31           # the first to give up waited the whole budget
    assert min(c0, c1) <= (1 << 31) + (1 << 28)  # the other left soon after the abort flag
    # the context still runs work
    x = torch.arange(1000, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == 499500.0
