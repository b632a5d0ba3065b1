"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

Every call here carries arguments the library must reject before it launches
anything (sizes, null or misaligned pointers, short workspace), so nothing
reaches a device.  Also checks that libkata.so exports every function the
public header declares, and the workspace-size query.
"""
import ctypes
import os
import re

import pytest

from kernelized_linear_attention_fwd_b200 import binding
from kernelized_linear_attention_fwd_b200.csrc import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kata.h")


@pytest.fixture(scope="module")
def lib():
    # The calls below pass fake device addresses that only the host-side checks
    # may see; on a machine with a GPU a check that failed to reject one would
    # launch a kernel on them, so these tests run only where no GPU is visible.
    import torch

    if torch.cuda.is_available():
        pytest.skip("host-side ABI checks use fake device pointers: run without a GPU")
    kbuild.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kata_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_expected_entry_points():
    names = declared_functions()
    for n in ("kata_chunked_forward", "kata_decode_step", "kata_chunked_forward_workspace_bytes",
              "kata_get_device_status", "kata_status_string", "kata_version"):
        assert n in names
    assert set(names) == set(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert getattr(lib, name) is not None


def test_status_strings(lib):
    for code, name in [(0, "KATA_OK"), (1, "KATA_ERR_INVALID_ARG"), (2, "KATA_ERR_UNSUPPORTED"),
                       (3, "KATA_ERR_WORKSPACE"), (4, "KATA_ERR_CUDA"), (5, "KATA_ERR_TIMEOUT")]:
        assert binding.kata_status_string(code) == name
    assert binding.kata_status_string(99) == "KATA_ERR_UNKNOWN"
    assert binding.kata_version() >= 100


def test_workspace_query(lib):
    W = lib.kata_chunked_forward_workspace_bytes
    # rejected arguments -> 0
    assert W(0, 1, 16, 64, 64, 64, 1) == 0
    assert W(1, 1, 16, 48, 48, 64, 1) == 0   # unsupported head size
    assert W(1, 1, 16, 64, 32, 64, 1) == 0   # dk != dv
    assert W(1, 1, 16, 64, 64, 48, 1) == 0   # bad chunk
    assert W(1, 1, 16, 64, 64, 64, 7) == 0   # bad dtype
    # positive, monotone in T and in heads
    a = W(1, 8, 131072, 64, 64, 64, 1)
    b = W(1, 8, 65536, 64, 64, 64, 1)
    c = W(2, 8, 131072, 64, 64, 64, 1)
    assert a > b > 0 and c >= 2 * a - 512
    assert W(1, 1, 256, 16, 16, 64, 0) > 0
    # C <= 256 merges chunks into the same segments (same workspace); C >= 512
    # keeps a state every C tokens (more states for smaller C)
    assert W(1, 8, 131072, 64, 64, 16, 1) == W(1, 8, 131072, 64, 64, 256, 1) == a
    assert W(1, 8, 131072, 64, 64, 1024, 1) == a
    assert W(1, 8, 131072, 64, 64, 512, 1) > a > W(1, 8, 131072, 64, 64, 2048, 1) > 0
    assert W(1, 8, 131072, 64, 64, 4096, 1) > 0 and W(1, 8, 131072, 64, 64, 8192, 1) == 0


def test_small_bf16_heads_take_the_two_factor_tensor_core_workspace(lib):
    # bf16 heads of d <= 32 run the tensor-core kernels, which read them as
    # d = 64 (the tensor maps zero-fill the columns past d) on the two-factor
    # layout (coordinates 32-63 are a second factor that contributes nothing):
    # the workspace of a two-factor d = 64 head, smaller than the one-factor
    # one, with no padded copies; fp32 keeps its CUDA-core layout
    W = lib.kata_chunked_forward_workspace_bytes
    Wmg = lib.kata_mg_chunked_forward_workspace_bytes
    for B, H, T, d in [(2, 4, 4096, 32), (1, 3, 1000, 16), (1, 1, 1, 32), (4, 2, 2049, 16)]:
        for C in (64, 512):
            assert W(B, H, T, d, d, C, 1) == Wmg(B, H, T, 64, 64, C, 2, 1)
            assert W(B, H, T, d, d, C, 1) < W(B, H, T, 64, 64, C, 1)
        assert W(B, H, T, d, d, 64, 0) < W(B, H, T, 64, 64, 64, 0)


FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced: every call below fails first


def _fwd(lib, q=FAKE, k=FAKE + 0x10000000, v=FAKE + 0x20000000, out=FAKE + 0x30000000, B=1, H=1,
         T=64, dk=16, dv=16, C=64, dt=0, so=None, zo=None, ws=None, wsb=0):
    vp = ctypes.c_void_p
    return lib.kata_chunked_forward(vp(q) if q else None, vp(k) if k else None,
                                    vp(v) if v else None, vp(out) if out else None, B, H, T, dk,
                                    dv, C, dt, vp(so) if so else None, vp(zo) if zo else None,
                                    vp(ws) if ws else None, wsb, None)


def test_forward_rejects_bad_arguments(lib):
    E = binding
    assert _fwd(lib, q=0) == E.KATA_ERR_INVALID_ARG
    assert _fwd(lib, out=0) == E.KATA_ERR_INVALID_ARG
    assert _fwd(lib, q=FAKE + 2) == E.KATA_ERR_INVALID_ARG            # misaligned
    assert _fwd(lib, B=0) == E.KATA_ERR_INVALID_ARG
    assert _fwd(lib, T=0) == E.KATA_ERR_INVALID_ARG
    assert _fwd(lib, T=-5) == E.KATA_ERR_INVALID_ARG
    assert _fwd(lib, C=48) == E.KATA_ERR_INVALID_ARG
    assert _fwd(lib, C=8192) == E.KATA_ERR_INVALID_ARG
    assert _fwd(lib, C=768) == E.KATA_ERR_INVALID_ARG
    assert _fwd(lib, dk=128, dv=128) == E.KATA_ERR_UNSUPPORTED
    assert _fwd(lib, dk=16, dv=32) == E.KATA_ERR_UNSUPPORTED
    assert _fwd(lib, dt=3) == E.KATA_ERR_UNSUPPORTED
    # state_out without z_out
    assert _fwd(lib, so=FAKE + 0x40000000) == E.KATA_ERR_INVALID_ARG
    # out aliasing an input
    assert _fwd(lib, out=FAKE + 0x10000000) == E.KATA_ERR_INVALID_ARG
    # missing / short / misaligned workspace for a problem that needs one
    need = lib.kata_chunked_forward_workspace_bytes(1, 1, 4096, 16, 16, 64, 0)
    assert need > 0
    assert _fwd(lib, T=4096, ws=None, wsb=0) == E.KATA_ERR_WORKSPACE
    assert _fwd(lib, T=4096, ws=FAKE + 0x50000000, wsb=need - 1) == E.KATA_ERR_WORKSPACE
    assert _fwd(lib, T=4096, ws=FAKE + 0x50000010, wsb=need) == E.KATA_ERR_WORKSPACE


def test_quadratic_forward_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    E = binding

    def quad(q=FAKE, k=FAKE + 0x10000000, v=FAKE + 0x20000000, out=FAKE + 0x30000000, B=1, H=1,
             T=64, dk=16, dv=16, dt=0):
        return lib.kata_quadratic_forward(vp(q) if q else None, vp(k) if k else None,
                                          vp(v) if v else None, vp(out) if out else None, B, H,
                                          T, dk, dv, dt, None)

    assert quad(q=0) == E.KATA_ERR_INVALID_ARG
    assert quad(v=0) == E.KATA_ERR_INVALID_ARG
    assert quad(k=FAKE + 0x10000008) == E.KATA_ERR_INVALID_ARG         # misaligned
    assert quad(H=0) == E.KATA_ERR_INVALID_ARG
    assert quad(T=0) == E.KATA_ERR_INVALID_ARG
    assert quad(dk=48, dv=48) == E.KATA_ERR_UNSUPPORTED
    assert quad(dk=64, dv=32) == E.KATA_ERR_UNSUPPORTED
    assert quad(dt=2) == E.KATA_ERR_UNSUPPORTED
    assert quad(out=FAKE + 0x20000000 + 256) == E.KATA_ERR_INVALID_ARG  # out inside v


def test_state_only_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    E = binding
    need = lib.kata_chunked_forward_workspace_bytes(1, 1, 4096, 16, 16, 64, 0)

    def cs(k=FAKE, v=FAKE + 0x10000000, so=FAKE + 0x40000000, zo=FAKE + 0x48000000, T=4096,
           dk=16, C=64, ws=FAKE + 0x50000000, wsb=None):
        return lib.kata_chunked_state(vp(k) if k else None, vp(v) if v else None, 1, 1, T, dk, dk,
                                      C, 0, vp(so) if so else None, vp(zo) if zo else None,
                                      vp(ws) if ws else None, need if wsb is None else wsb, None)

    assert cs(k=0) == E.KATA_ERR_INVALID_ARG
    assert cs(so=0, zo=0) == E.KATA_ERR_INVALID_ARG              # the state is the output
    assert cs(zo=0) == E.KATA_ERR_INVALID_ARG
    assert cs(so=FAKE + 0x40000004) == E.KATA_ERR_INVALID_ARG    # misaligned
    assert cs(so=FAKE + 0x10000000) == E.KATA_ERR_INVALID_ARG    # state_out over v
    assert cs(zo=FAKE + 0x40000000 + 4096) == E.KATA_ERR_INVALID_ARG  # z_out inside state_out
    assert cs(C=40) == E.KATA_ERR_INVALID_ARG
    assert cs(dk=48) == E.KATA_ERR_UNSUPPORTED
    assert cs(ws=0, wsb=0) == E.KATA_ERR_WORKSPACE
    assert cs(wsb=need - 1) == E.KATA_ERR_WORKSPACE


def test_forward_from_state_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    E = binding
    need = lib.kata_chunked_forward_workspace_bytes(1, 1, 64, 16, 16, 64, 0)
    S0, Z0 = FAKE + 0x60000000, FAKE + 0x68000000

    def ffs(q=FAKE, out=FAKE + 0x30000000, si=S0, zi=Z0, n=1, ss=0, zs=0, so=None, zo=None,
            flags=0):
        return lib.kata_chunked_forward_from_state(
            vp(q) if q else None, vp(FAKE + 0x10000000), vp(FAKE + 0x20000000),
            vp(out) if out else None, 1, 1, 64, 16, 16, 64, 0, vp(si) if si else None,
            vp(zi) if zi else None, n, ss, zs, vp(so) if so else None, vp(zo) if zo else None,
            vp(FAKE + 0x50000000), need, flags, None)

    assert ffs(q=0) == E.KATA_ERR_INVALID_ARG
    assert ffs(n=-1) == E.KATA_ERR_INVALID_ARG
    assert ffs(si=0) == E.KATA_ERR_INVALID_ARG                   # n_in = 1 needs both inputs
    assert ffs(zi=0) == E.KATA_ERR_INVALID_ARG
    assert ffs(si=S0 + 8) == E.KATA_ERR_INVALID_ARG              # misaligned
    assert ffs(n=3, ss=16 * 16 * 16 + 2, zs=256) == E.KATA_ERR_INVALID_ARG  # rows off 16 bytes
    assert ffs(out=S0) == E.KATA_ERR_INVALID_ARG                 # out over an input state
    # state_out overlapping the inputs, unless it is the one input itself
    assert ffs(n=2, ss=4096, zs=256, so=S0 + 4 * 4096, zo=Z0 + 0x100000) == E.KATA_ERR_INVALID_ARG
    assert ffs(so=S0 + 256, zo=Z0 + 256) == E.KATA_ERR_INVALID_ARG
    assert ffs(so=S0, zo=0) == E.KATA_ERR_INVALID_ARG            # both or neither
    assert ffs(flags=2) == E.KATA_ERR_INVALID_ARG                # unknown flag bits
    assert ffs(q=0, flags=1) == E.KATA_ERR_INVALID_ARG


def test_host_forward_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    E = binding
    need = lib.kata_chunked_forward_host_buffer_bytes(1, 8, 4096, 64, 64, 64, 1, 1)
    assert need > 0
    assert lib.kata_chunked_forward_host_buffer_bytes(1, 8, 4096, 48, 48, 64, 1, 1) == 0
    # fewer heads per group, less staging
    assert need < lib.kata_chunked_forward_host_buffer_bytes(1, 8, 4096, 64, 64, 64, 1, 4)
    host = ctypes.create_string_buffer(64)  # host pointers are never read: every call fails first

    def fh(q=True, out=True, so=None, zo=None, buf=FAKE, nbytes=None, H=8, dk=64):
        a = vp(ctypes.addressof(host))
        return lib.kata_chunked_forward_host(a if q else None, a, a, a if out else None, 1, H,
                                             4096, dk, dk, 64, 1, vp(so) if so else None,
                                             vp(zo) if zo else None, vp(buf) if buf else None,
                                             need if nbytes is None else nbytes, 1, None)

    assert fh(q=False) == E.KATA_ERR_INVALID_ARG
    assert fh(out=False) == E.KATA_ERR_INVALID_ARG
    assert fh(so=FAKE + 0x1000) == E.KATA_ERR_INVALID_ARG      # state_out without z_out
    assert fh(dk=48) == E.KATA_ERR_UNSUPPORTED
    assert fh(H=0) == E.KATA_ERR_INVALID_ARG
    assert fh(buf=None) == E.KATA_ERR_WORKSPACE
    assert fh(nbytes=need - 1) == E.KATA_ERR_WORKSPACE
    assert fh(buf=FAKE + 16) == E.KATA_ERR_WORKSPACE             # not 256-byte aligned


def test_decode_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    E = binding

    def dec(q=FAKE, k=FAKE + 0x100, v=FAKE + 0x200, out=FAKE + 0x300, S=FAKE + 0x10000,
            Z=FAKE + 0x10000000, B=1, H=1, dk=16, dv=16, dt=0):
        return lib.kata_decode_step(vp(q) if q else None, vp(k) if k else None,
                                    vp(v) if v else None, vp(out) if out else None,
                                    vp(S) if S else None, vp(Z) if Z else None, B, H, dk, dv, dt,
                                    None)

    assert dec(q=0) == E.KATA_ERR_INVALID_ARG
    assert dec(S=0) == E.KATA_ERR_INVALID_ARG
    assert dec(B=0) == E.KATA_ERR_INVALID_ARG
    assert dec(dk=48, dv=48) == E.KATA_ERR_UNSUPPORTED
    assert dec(dt=9) == E.KATA_ERR_UNSUPPORTED
    assert dec(S=FAKE + 0x10008) == E.KATA_ERR_INVALID_ARG                 # misaligned
    assert dec(Z=FAKE + 0x10000 + 4096) == E.KATA_ERR_INVALID_ARG          # Z inside S
    assert dec(out=FAKE + 0x10000) == E.KATA_ERR_INVALID_ARG               # out inside S


def test_packed_layout_calls_reject_bad_arguments(lib):
    vp = ctypes.c_void_p
    E = binding
    S, Z, Sp, Zp = FAKE + 0x10000, FAKE + 0x10000000, FAKE + 0x20000000, FAKE + 0x30000000

    def dec(q=FAKE, S=Sp, Z=Zp, dk=16, dv=16, dt=0, out=FAKE + 0x300):
        return lib.kata_decode_step_packed(vp(q) if q else None, vp(FAKE + 0x100),
                                           vp(FAKE + 0x200), vp(out), vp(S) if S else None,
                                           vp(Z) if Z else None, 1, 1, dk, dv, dt, None)

    def conv(fn, a=S, b=Z, c=Sp, d=Zp, dk=16):
        return fn(vp(a) if a else None, vp(b) if b else None, vp(c) if c else None,
                  vp(d) if d else None, 1, 1, dk, dk, None)

    assert dec(q=0) == E.KATA_ERR_INVALID_ARG
    assert dec(S=0) == E.KATA_ERR_INVALID_ARG
    assert dec(dk=48, dv=48) == E.KATA_ERR_UNSUPPORTED
    assert dec(dt=4) == E.KATA_ERR_UNSUPPORTED
    # packed z right after the packed state: 136 rows x 16 x 4 B; one byte less overlaps
    assert dec(Z=Sp + 136 * 16 * 4 - 16) == E.KATA_ERR_INVALID_ARG
    assert dec(out=Sp + 64) == E.KATA_ERR_INVALID_ARG
    for fn in (lib.kata_state_pack, lib.kata_state_unpack):
        assert conv(fn, a=0) == E.KATA_ERR_INVALID_ARG
        assert conv(fn, d=0) == E.KATA_ERR_INVALID_ARG
        assert conv(fn, c=Sp + 4) == E.KATA_ERR_INVALID_ARG         # misaligned
        assert conv(fn, dk=24) == E.KATA_ERR_UNSUPPORTED
        assert conv(fn, c=S + 64) == E.KATA_ERR_INVALID_ARG          # destination over source
        assert conv(fn, d=Sp + 16) == E.KATA_ERR_INVALID_ARG         # destinations overlap


def test_binding_rejects_host_tensors_and_bad_shapes(lib):
    # checked in the binding before anything reaches the library
    import torch

    x = torch.zeros((1, 2, 8, 16), dtype=torch.bfloat16)
    for call in (lambda: binding.kata_chunked_forward(x, x, x),
                 lambda: binding.kata_quadratic_forward(x, x, x),
                 lambda: binding.kata_chunked_state(x, x),
                 lambda: binding.kata_decode_step(x[:, :, 0], x[:, :, 0], x[:, :, 0],
                                                  torch.zeros((1, 2, 256, 16)),
                                                  torch.zeros((1, 2, 16, 16)))):
        with pytest.raises(binding.KataError) as e:
            call()
        assert e.value.status == binding.KATA_ERR_INVALID_ARG
    # the host-buffer forward wants host tensors of matching shapes
    with pytest.raises(binding.KataError):
        binding.kata_chunked_forward_host(x, x, x, torch.zeros((1, 2, 8, 8), dtype=x.dtype))
    assert binding.packed_rows(64) == 2080 and binding.packed_rows(16) == 136


class _FakeCudaTensor:
    """Stands in for a CUDA tensor on a given device (no GPU needed): only the
    attributes the binding's checks read."""

    def __init__(self, shape, dtype, device):
        import torch

        self.shape = tuple(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self.is_cuda = True

    def is_contiguous(self):
        return True


def test_binding_rejects_tensors_on_another_device():
    # every tensor of a call must live on the first tensor's device; the call
    # then runs with that device current (the library launches on the current
    # device and takes its status word and static scratch from it)
    import torch

    shape = (1, 2, 8, 16)
    q = _FakeCudaTensor(shape, torch.bfloat16, "cuda:0")
    binding._check(q, "q", shape, torch.bfloat16, device=torch.device("cuda:0"))
    for name, dev in (("k", "cuda:1"), ("out", "cuda:3")):
        t = _FakeCudaTensor(shape, torch.bfloat16, dev)
        with pytest.raises(binding.KataError) as e:
            binding._check(t, name, shape, torch.bfloat16, device=q.device)
        assert e.value.status == binding.KATA_ERR_INVALID_ARG and name in str(e.value)
    s = _FakeCudaTensor((3, 1, 2, 256, 16), torch.float32, "cuda:1")
    with pytest.raises(binding.KataError):
        binding._stacked(s, "state_in", (1, 2, 256, 16), "n", q.device)


def test_noalloc_scratch_size_matches_the_header():
    text = open(HEADER).read()
    m = re.search(r"#define\s+KATA_NOALLOC_SCRATCH_BYTES\s+\(([^)]*)\)", text)
    assert m, "KATA_NOALLOC_SCRATCH_BYTES not found in kata.h"
    expr = m.group(1).replace("u", "")
    assert re.fullmatch(r"[0-9 *+]+", expr), expr
    assert eval(expr) == binding.KATA_NOALLOC_SCRATCH_BYTES


def test_binding_fails_loudly_without_library(tmp_path):
    saved = binding._lib
    try:
        binding._lib = None
        with pytest.raises(RuntimeError):
            binding.load_library(str(tmp_path / "missing.so"))
    finally:
        binding._lib = saved
