"""KATA kernelized linear attention (rank-one PSD features), causal forward and
recurrent decode on NVIDIA B200 (sm_100a).

The compute path is libkata.so (hand-written CUDA kernels behind the C ABI in
include/kata.h); ``binding`` marshals torch CUDA tensors into it.
"""
from .binding import (  # noqa: F401
    KataError,
    kata_chunked_forward,
    kata_chunked_forward_from_state,
    kata_chunked_forward_host,
    kata_chunked_forward_host_buffer_bytes,
    kata_chunked_forward_noalloc,
    kata_chunked_forward_workspace_bytes,
    kata_chunked_state,
    kata_decode_step,
    kata_decode_step_packed,
    kata_get_device_status,
    kata_mg_chunked_forward,
    kata_mg_chunked_forward_workspace_bytes,
    kata_mg_decode_step,
    kata_quadratic_forward,
    kata_state_pack,
    kata_state_unpack,
    kata_status_string,
    kata_version,
    load_library,
)
