"""Python binding of libkata (the C ABI in include/kata.h).

Argument marshalling only: every step of the forward and the decode runs in
the library's CUDA kernels.  Tensors are torch CUDA tensors (torch supplies
device memory and streams); the functions carry the C names and raise
``KataError`` on any status other than KATA_OK.  There is no fallback: if
libkata.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkata.so")

KATA_OK = 0
KATA_ERR_INVALID_ARG = 1
KATA_ERR_UNSUPPORTED = 2
KATA_ERR_WORKSPACE = 3
KATA_ERR_CUDA = 4
KATA_ERR_TIMEOUT = 5

KATA_F32 = 0
KATA_BF16 = 1

# Every symbol include/kata.h declares.
EXPORTS = (
    "kata_version",
    "kata_status_string",
    "kata_chunked_forward_workspace_bytes",
    "kata_chunked_forward",
    "kata_chunked_state",
    "kata_chunked_forward_from_state",
    "kata_chunked_forward_noalloc",
    "kata_chunked_forward_host_buffer_bytes",
    "kata_chunked_forward_host",
    "kata_quadratic_forward",
    "kata_mg_chunked_forward_workspace_bytes",
    "kata_mg_chunked_forward",
    "kata_mg_decode_step",
    "kata_decode_step",
    "kata_decode_step_packed",
    "kata_state_pack",
    "kata_state_unpack",
    "kata_get_device_status",
)


class KataError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {kata_status_string(status)} ({status})")


_lib = None


def load_library(path: str = LIB_PATH):
    """Loads libkata.so once and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libkata.so not found at {path}; build it with "
            "`python kernelized_linear_attention_fwd_b200/csrc/build.py`")
    lib = ctypes.CDLL(path)
    vp, sz, i32, fp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p
    lib.kata_version.restype = i32
    lib.kata_version.argtypes = []
    lib.kata_status_string.restype = ctypes.c_char_p
    lib.kata_status_string.argtypes = [i32]
    lib.kata_chunked_forward_workspace_bytes.restype = sz
    lib.kata_chunked_forward_workspace_bytes.argtypes = [i32] * 7
    lib.kata_chunked_forward.restype = i32
    lib.kata_chunked_forward.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                         fp, fp, vp, sz, vp]
    lib.kata_chunked_state.restype = i32
    lib.kata_chunked_state.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, fp, fp, vp, sz, vp]
    lib.kata_chunked_forward_from_state.restype = i32
    lib.kata_chunked_forward_from_state.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                    i32, fp, fp, i32, sz, sz, fp, fp, vp, sz,
                                                    ctypes.c_uint, vp]
    lib.kata_chunked_forward_host_buffer_bytes.restype = sz
    lib.kata_chunked_forward_host_buffer_bytes.argtypes = [i32] * 8
    lib.kata_chunked_forward_host.restype = i32
    lib.kata_chunked_forward_host.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                              fp, fp, vp, sz, i32, vp]
    lib.kata_chunked_forward_noalloc.restype = i32
    lib.kata_chunked_forward_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                 i32, fp, fp, vp]
    lib.kata_mg_chunked_forward_workspace_bytes.restype = sz
    lib.kata_mg_chunked_forward_workspace_bytes.argtypes = [i32] * 8
    lib.kata_mg_chunked_forward.restype = i32
    lib.kata_mg_chunked_forward.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                            i32, fp, fp, vp, sz, vp]
    lib.kata_mg_decode_step.restype = i32
    lib.kata_mg_decode_step.argtypes = [vp, vp, vp, vp, fp, fp, i32, i32, i32, i32, i32, i32, vp]
    lib.kata_quadratic_forward.restype = i32
    lib.kata_quadratic_forward.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
    lib.kata_decode_step.restype = i32
    lib.kata_decode_step.argtypes = [vp, vp, vp, vp, fp, fp, i32, i32, i32, i32, i32, vp]
    lib.kata_decode_step_packed.restype = i32
    lib.kata_decode_step_packed.argtypes = [vp, vp, vp, vp, fp, fp, i32, i32, i32, i32, i32, vp]
    for name in ("kata_state_pack", "kata_state_unpack"):
        getattr(lib, name).restype = i32
        getattr(lib, name).argtypes = [fp, fp, fp, fp, i32, i32, i32, i32, vp]
    lib.kata_get_device_status.restype = i32
    lib.kata_get_device_status.argtypes = [vp]
    _lib = lib
    return lib


def kata_version() -> int:
    return load_library().kata_version()


def kata_status_string(status: int) -> str:
    return load_library().kata_status_string(int(status)).decode()


def _dtype_code(t):
    import torch

    if t.dtype == torch.bfloat16:
        return KATA_BF16
    if t.dtype == torch.float32:
        return KATA_F32
    raise KataError(KATA_ERR_UNSUPPORTED, f"dtype {t.dtype}")


def _stream_handle(stream, device=None):
    """Handle of `stream`, or of the current stream of `device` (the device the
    call's tensors live on) when None.  A given stream must belong to that
    device: kernels run on the stream's device, and pointers of another
    device's memory are not valid there."""
    import torch

    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != device:
        raise KataError(KATA_ERR_INVALID_ARG,
                        f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _on_device(device):
    """Context that makes `device` current for the call: the library launches
    on the current device and takes its per-device resources (status word,
    static scratch) from it."""
    import torch

    return torch.cuda.device(device)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t, name, shape, dtype=None, device=None):
    """t (optional) is a contiguous CUDA tensor of `shape` and `dtype` on
    `device` (the device of the call's first tensor)."""
    if t is None:
        return
    if not t.is_cuda:
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} is on {t.device}, want {device}")
    if not t.is_contiguous():
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} has shape {tuple(t.shape)}, want {shape}")
    if dtype is not None and t.dtype != dtype:
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} has dtype {t.dtype}, want {dtype}")


def kata_chunked_forward_workspace_bytes(B, H, T, dk, dv, C, dtype_code) -> int:
    return int(load_library().kata_chunked_forward_workspace_bytes(B, H, T, dk, dv, C,
                                                                   dtype_code))


def kata_chunked_forward(q, k, v, C=64, out=None, state_out=None, z_out=None, workspace=None,
                         stream=None):
    """out[B,H,T,dv] = causal KATA forward of q, k [B,H,T,dk] and v [B,H,T,dv].

    Optionally writes the final state S [B,H,dk*dk,dv] and Z [B,H,dk,dk] (fp32).
    `workspace` is a uint8 CUDA tensor of at least
    kata_chunked_forward_workspace_bytes(...) bytes; allocated here if None.
    """
    import torch

    lib = load_library()
    B, H, T, dk = q.shape
    dev = q.device
    dv = v.shape[-1]
    _check(q, "q", (B, H, T, dk), device=dev)
    _check(k, "k", (B, H, T, dk), q.dtype, device=dev)
    _check(v, "v", (B, H, T, dv), q.dtype, device=dev)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", (B, H, T, dv), q.dtype, device=dev)
    _check(state_out, "state_out", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z_out, "z_out", (B, H, dk, dk), torch.float32, device=dev)
    workspace, ws_bytes = _workspace(lib, workspace, B, H, T, dk, dv, C, code, dev)
    with _on_device(dev):
        st = lib.kata_chunked_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, dk, dv,
                                      int(C), code, _ptr(state_out), _ptr(z_out),
                                      _ptr(workspace), ws_bytes, _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_chunked_forward")
    return out


def _workspace(lib, workspace, B, H, T, dk, dv, C, code, device):
    """(workspace, bytes): the caller's (on `device`) or one allocated here."""
    import torch

    need = lib.kata_chunked_forward_workspace_bytes(B, H, T, dk, dv, C, code)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if workspace is not None and (not workspace.is_cuda or workspace.device != device):
        raise KataError(KATA_ERR_INVALID_ARG, f"workspace must be on {device}")
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return workspace, nbytes


def kata_chunked_state(k, v, C=64, state_out=None, z_out=None, workspace=None, stream=None):
    """(S [B,H,dk*dk,dv], Z [B,H,dk,dk]) fp32: the state after the T tokens of
    k, v [B,H,T,*], without the outputs.  Allocated here when not given."""
    import torch

    lib = load_library()
    B, H, T, dk = k.shape
    dev = k.device
    dv = v.shape[-1]
    _check(k, "k", (B, H, T, dk), device=dev)
    _check(v, "v", (B, H, T, dv), k.dtype, device=dev)
    code = _dtype_code(k)
    if state_out is None:
        state_out = torch.empty((B, H, dk * dk, dv), dtype=torch.float32, device=k.device)
    if z_out is None:
        z_out = torch.empty((B, H, dk, dk), dtype=torch.float32, device=k.device)
    _check(state_out, "state_out", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z_out, "z_out", (B, H, dk, dk), torch.float32, device=dev)
    workspace, nbytes = _workspace(lib, workspace, B, H, T, dk, dv, C, code, dev)
    with _on_device(dev):
        st = lib.kata_chunked_state(_ptr(k), _ptr(v), B, H, T, dk, dv, int(C), code,
                                    _ptr(state_out), _ptr(z_out), _ptr(workspace), nbytes,
                                    _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_chunked_state")
    return state_out, z_out


def _stacked(t, name, inner, n_name, device=None):
    """(n, stride in elements) of a stack of states: t is [n, *inner] whose
    blocks t[m] are each contiguous (any stride between blocks), or one state
    [*inner] (n = 1), on `device`."""
    import torch

    if t is None:
        return 0, 0
    if not t.is_cuda or t.dtype != torch.float32:
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} must be a CUDA float32 tensor")
    if device is not None and t.device != device:
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} is on {t.device}, want {device}")
    if tuple(t.shape) == tuple(inner):
        t = t.unsqueeze(0)
    if t.dim() != len(inner) + 1 or tuple(t.shape[1:]) != tuple(inner):
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} has shape {tuple(t.shape)}, want "
                                              f"[{n_name}, {', '.join(map(str, inner))}]")
    if t.shape[0] > 0 and not t[0].is_contiguous():
        raise KataError(KATA_ERR_INVALID_ARG, f"each state of {name} must be contiguous")
    return t.shape[0], t.stride(0)


KATA_REUSE_SEGMENT_STATES = 1


def kata_chunked_forward_from_state(q, k, v, state_in, z_in, C=64, out=None, state_out=None,
                                    z_out=None, workspace=None, stream=None,
                                    reuse_segment_states=False):
    """out[B,H,T,dv]: the chunked forward of q, k, v continuing from the state
    sum_m state_in[m], sum_m z_in[m].  state_in is [n, B, H, dk*dk, dv] (or one
    [B, H, dk*dk, dv] state), z_in [n, B, H, dk, dk]; each state contiguous,
    any stride between them.  state_out / z_out (optional) receive the state
    after the last token; they may be state_in / z_in themselves for one input.
    reuse_segment_states: `workspace` holds what kata_chunked_state last wrote
    into it for the same k, v and sizes (KATA_REUSE_SEGMENT_STATES)."""
    import torch

    lib = load_library()
    B, H, T, dk = q.shape
    dev = q.device
    dv = v.shape[-1]
    _check(q, "q", (B, H, T, dk), device=dev)
    _check(k, "k", (B, H, T, dk), q.dtype, device=dev)
    _check(v, "v", (B, H, T, dv), q.dtype, device=dev)
    code = _dtype_code(q)
    n_s, s_stride = _stacked(state_in, "state_in", (B, H, dk * dk, dv), "n", dev)
    n_z, z_stride = _stacked(z_in, "z_in", (B, H, dk, dk), "n", dev)
    if n_s != n_z:
        raise KataError(KATA_ERR_INVALID_ARG, f"state_in holds {n_s} states, z_in {n_z}")
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", (B, H, T, dv), q.dtype, device=dev)
    _check(state_out, "state_out", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z_out, "z_out", (B, H, dk, dk), torch.float32, device=dev)
    if reuse_segment_states and workspace is None:
        raise KataError(KATA_ERR_WORKSPACE, "reusing segment states needs the state call's workspace")
    workspace, nbytes = _workspace(lib, workspace, B, H, T, dk, dv, C, code, dev)
    with _on_device(dev):
        st = lib.kata_chunked_forward_from_state(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, dk, dv, int(C), code,
            _ptr(state_in) if n_s else None, _ptr(z_in) if n_z else None, n_s, s_stride, z_stride,
            _ptr(state_out), _ptr(z_out), _ptr(workspace), nbytes,
            KATA_REUSE_SEGMENT_STATES if reuse_segment_states else 0,
            _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_chunked_forward_from_state")
    return out


def _check_host(t, name, shape, dtype=None):
    if t.is_cuda:
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} has shape {tuple(t.shape)}, want {shape}")
    if dtype is not None and t.dtype != dtype:
        raise KataError(KATA_ERR_INVALID_ARG, f"{name} has dtype {t.dtype}, want {dtype}")


def kata_chunked_forward_host_buffer_bytes(B, H, T, dk, dv, C, dtype_code, heads_per_group=0):
    return int(load_library().kata_chunked_forward_host_buffer_bytes(
        B, H, T, dk, dv, C, dtype_code, heads_per_group))


def kata_chunked_forward_host(q, k, v, out, C=64, state_out=None, z_out=None,
                              device_buffer=None, heads_per_group=0, stream=None):
    """The chunked forward on host tensors q, k [B,H,T,dk], v, out [B,H,T,dv]
    (pinned for the copies to overlap with the compute), heads in groups.
    state_out / z_out are CUDA tensors; device_buffer a uint8 CUDA tensor of at
    least kata_chunked_forward_host_buffer_bytes(...) bytes (allocated here if
    None).  `out` holds the result once `stream` is synchronised."""
    import torch

    lib = load_library()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _check_host(q, "q", (B, H, T, dk))
    _check_host(k, "k", (B, H, T, dk), q.dtype)
    _check_host(v, "v", (B, H, T, dv), q.dtype)
    _check_host(out, "out", (B, H, T, dv), q.dtype)
    code = _dtype_code(q)
    # the device that runs the call: the device buffer's, else the state's, else the current one
    if device_buffer is not None:
        dev = device_buffer.device
    elif state_out is not None:
        dev = state_out.device
    else:
        dev = torch.device("cuda", torch.cuda.current_device())
    _check(state_out, "state_out", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z_out, "z_out", (B, H, dk, dk), torch.float32, device=dev)
    need = kata_chunked_forward_host_buffer_bytes(B, H, T, dk, dv, int(C), code,
                                                  int(heads_per_group))
    if device_buffer is None:
        device_buffer = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    if not device_buffer.is_cuda:
        raise KataError(KATA_ERR_INVALID_ARG, "device_buffer must be a CUDA tensor")
    nbytes = device_buffer.numel() * device_buffer.element_size()
    with _on_device(dev):
        st = lib.kata_chunked_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, dk,
                                           dv, int(C), code, _ptr(state_out), _ptr(z_out),
                                           _ptr(device_buffer), nbytes, int(heads_per_group),
                                           _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_chunked_forward_host")
    return out


# Bytes of the library's static scratch used by kata_chunked_forward_noalloc.
KATA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def kata_chunked_forward_noalloc(q, k, v, C=64, out=None, state_out=None, z_out=None,
                                 stream=None):
    """kata_chunked_forward with the library's static device scratch instead of
    a workspace: for callers that cannot allocate device memory.  `out`
    (and the optional state buffers) must be passed in by such callers; when
    `out` is None it is allocated here for convenience.  Problems needing more
    than KATA_NOALLOC_SCRATCH_BYTES of scratch raise KATA_ERR_WORKSPACE."""
    import torch

    lib = load_library()
    B, H, T, dk = q.shape
    dev = q.device
    dv = v.shape[-1]
    _check(q, "q", (B, H, T, dk), device=dev)
    _check(k, "k", (B, H, T, dk), q.dtype, device=dev)
    _check(v, "v", (B, H, T, dv), q.dtype, device=dev)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", (B, H, T, dv), q.dtype, device=dev)
    _check(state_out, "state_out", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z_out, "z_out", (B, H, dk, dk), torch.float32, device=dev)
    with _on_device(dev):
        st = lib.kata_chunked_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T,
                                              dk, dv, int(C), code, _ptr(state_out),
                                              _ptr(z_out), _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_chunked_forward_noalloc")
    return out


def kata_mg_chunked_forward_workspace_bytes(B, H, T, dk, dv, C, g, dtype_code) -> int:
    return int(load_library().kata_mg_chunked_forward_workspace_bytes(B, H, T, dk, dv, C, g,
                                                                      dtype_code))


def kata_mg_chunked_forward(q, k, v, g=2, C=64, out=None, state_out=None, z_out=None,
                            workspace=None, stream=None):
    """KATA-Mg forward: g rank-one PSD factors on consecutive blocks of dk / g
    coordinates, weight sum_m (q^(m).k^(m))^2.  Arguments as
    kata_chunked_forward; the exported state holds zeros across factors."""
    import torch

    lib = load_library()
    B, H, T, dk = q.shape
    dev = q.device
    dv = v.shape[-1]
    _check(q, "q", (B, H, T, dk), device=dev)
    _check(k, "k", (B, H, T, dk), q.dtype, device=dev)
    _check(v, "v", (B, H, T, dv), q.dtype, device=dev)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", (B, H, T, dv), q.dtype, device=dev)
    _check(state_out, "state_out", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z_out, "z_out", (B, H, dk, dk), torch.float32, device=dev)
    need = lib.kata_mg_chunked_forward_workspace_bytes(B, H, T, dk, dv, int(C), int(g), code)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace is not None and (not workspace.is_cuda or workspace.device != dev):
        raise KataError(KATA_ERR_INVALID_ARG, f"workspace must be on {dev}")
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _on_device(dev):
        st = lib.kata_mg_chunked_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, dk, dv,
                                         int(C), int(g), code, _ptr(state_out), _ptr(z_out),
                                         _ptr(workspace), nbytes, _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_mg_chunked_forward")
    return out


def kata_mg_decode_step(q, k, v, state, z, g=2, out=None, stream=None):
    """One KATA-Mg decode step, in place on the dense (state, z) of g factors."""
    import torch

    lib = load_library()
    B, H, dk = q.shape
    dev = q.device
    dv = v.shape[-1]
    _check(q, "q", (B, H, dk), device=dev)
    _check(k, "k", (B, H, dk), q.dtype, device=dev)
    _check(v, "v", (B, H, dv), q.dtype, device=dev)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", (B, H, dv), q.dtype, device=dev)
    _check(state, "state", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z, "z", (B, H, dk, dk), torch.float32, device=dev)
    with _on_device(dev):
        st = lib.kata_mg_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(state), _ptr(z),
                                     B, H, dk, dv, int(g), code, _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_mg_decode_step")
    return out


def kata_quadratic_forward(q, k, v, out=None, stream=None):
    """out[B,H,T,dv] = causal KATA forward of q, k [B,H,T,dk] and v [B,H,T,dv] in
    the quadratic (flash-attention-style) form: no state, no workspace."""
    import torch

    lib = load_library()
    B, H, T, dk = q.shape
    dev = q.device
    dv = v.shape[-1]
    _check(q, "q", (B, H, T, dk), device=dev)
    _check(k, "k", (B, H, T, dk), q.dtype, device=dev)
    _check(v, "v", (B, H, T, dv), q.dtype, device=dev)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", (B, H, T, dv), q.dtype, device=dev)
    with _on_device(dev):
        st = lib.kata_quadratic_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, dk, dv,
                                        code, _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_quadratic_forward")
    return out


def kata_decode_step(q, k, v, state, z, out=None, stream=None):
    """One recurrent step, in place on (state, z); q, k [B,H,dk], v [B,H,dv]."""
    import torch

    lib = load_library()
    B, H, dk = q.shape
    dev = q.device
    dv = v.shape[-1]
    _check(q, "q", (B, H, dk), device=dev)
    _check(k, "k", (B, H, dk), q.dtype, device=dev)
    _check(v, "v", (B, H, dv), q.dtype, device=dev)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", (B, H, dv), q.dtype, device=dev)
    _check(state, "state", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z, "z", (B, H, dk, dk), torch.float32, device=dev)
    with _on_device(dev):
        st = lib.kata_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(state), _ptr(z),
                                  B, H, dk, dv, code, _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_decode_step")
    return out


def packed_rows(d: int) -> int:
    """Rows of the packed state layout: the pairs i <= j."""
    return d * (d + 1) // 2


def kata_decode_step_packed(q, k, v, state_p, z_p, out=None, stream=None):
    """kata_decode_step on the packed layout: state_p [B,H,R,dv], z_p [B,H,R],
    R = dk(dk+1)/2, updated in place."""
    import torch

    lib = load_library()
    B, H, dk = q.shape
    dev = q.device
    dv = v.shape[-1]
    R = packed_rows(dk)
    _check(q, "q", (B, H, dk), device=dev)
    _check(k, "k", (B, H, dk), q.dtype, device=dev)
    _check(v, "v", (B, H, dv), q.dtype, device=dev)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", (B, H, dv), q.dtype, device=dev)
    _check(state_p, "state_p", (B, H, R, dv), torch.float32, device=dev)
    _check(z_p, "z_p", (B, H, R), torch.float32, device=dev)
    with _on_device(dev):
        st = lib.kata_decode_step_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(state_p),
                                         _ptr(z_p), B, H, dk, dv, code,
                                         _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_decode_step_packed")
    return out


def kata_state_pack(state, z, state_p=None, z_p=None, stream=None):
    """Dense (state [B,H,dk*dk,dv], z [B,H,dk,dk]) -> packed (state_p, z_p)."""
    import torch

    lib = load_library()
    B, H, dd, dv = state.shape
    dev = state.device
    dk = z.shape[-1]
    R = packed_rows(dk)
    _check(state, "state", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z, "z", (B, H, dk, dk), torch.float32, device=dev)
    if state_p is None:
        state_p = torch.empty((B, H, R, dv), dtype=torch.float32, device=state.device)
    if z_p is None:
        z_p = torch.empty((B, H, R), dtype=torch.float32, device=state.device)
    _check(state_p, "state_p", (B, H, R, dv), torch.float32, device=dev)
    _check(z_p, "z_p", (B, H, R), torch.float32, device=dev)
    with _on_device(dev):
        st = lib.kata_state_pack(_ptr(state), _ptr(z), _ptr(state_p), _ptr(z_p), B, H, dk, dv,
                                 _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_state_pack")
    return state_p, z_p


def kata_state_unpack(state_p, z_p, state=None, z=None, stream=None):
    """Packed (state_p [B,H,R,dv], z_p [B,H,R]) -> dense (state, z)."""
    import torch

    lib = load_library()
    B, H, R, dv = state_p.shape
    dev = state_p.device
    dk = next(d for d in (16, 32, 64) if packed_rows(d) == R) if R in (136, 528, 2080) else 0
    if dk == 0:
        raise KataError(KATA_ERR_UNSUPPORTED, f"no supported head size has {R} packed rows")
    _check(state_p, "state_p", (B, H, R, dv), torch.float32, device=dev)
    _check(z_p, "z_p", (B, H, R), torch.float32, device=dev)
    if state is None:
        state = torch.empty((B, H, dk * dk, dv), dtype=torch.float32, device=state_p.device)
    if z is None:
        z = torch.empty((B, H, dk, dk), dtype=torch.float32, device=state_p.device)
    _check(state, "state", (B, H, dk * dk, dv), torch.float32, device=dev)
    _check(z, "z", (B, H, dk, dk), torch.float32, device=dev)
    with _on_device(dev):
        st = lib.kata_state_unpack(_ptr(state_p), _ptr(z_p), _ptr(state), _ptr(z), B, H, dk, dv,
                                   _stream_handle(stream, dev))
    if st != KATA_OK:
        raise KataError(st, "kata_state_unpack")
    return state, z


def kata_get_device_status(stream=None) -> int:
    """Synchronises `stream` (default: the current device's current stream) and
    returns and clears the status word of the stream's device."""
    import torch

    dev = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    with _on_device(dev):
        return int(load_library().kata_get_device_status(_stream_handle(stream, dev)))
