"""Sequence-sharded KATA forward: one long sequence split into contiguous
blocks, one block per rank, ranks in sequence order.

The chunked-state form makes the state after any prefix an additive summary
(gist.science summary of "Kernelized Linear Attention: Breaking the Capacity
Wall with Symmetric Cones", 2.3: chunk states combined by an associative
scan).  The same scan one level up shards a sequence over ranks:

1. every rank computes its block's own total state (S_r, Z_r) with
   kata_chunked_state, into one flat fp32 buffer [S_r | Z_r];
2. one all-gather of those buffers (the only data-path exchange; NCCL over
   NVLink, 8 MiB + 128 KiB per rank for 8 heads of d = 64);
3. rank r runs kata_chunked_forward_from_state on its block with the first r
   gathered totals as inputs: the library sums them while it scans its own
   segments, so the exclusive prefix over ranks costs no extra pass.  The
   block's per-segment states, built in step 1, stay in the workspace and
   are reused (KATA_REUSE_SEGMENT_STATES) instead of being built again.

Rank r's optional state output is the state after its block's last token
(the last rank's is the whole sequence's).  Every step runs in libkata's
kernels; torch supplies the buffers and torch.distributed the all-gather.
"""
from __future__ import annotations

from . import binding


class LibkataOps:
    """The library calls a block needs (the default; tests of the multi-rank
    orchestration substitute their own)."""

    @staticmethod
    def workspace(k, v, C):
        import torch

        B, H, T, dk = k.shape
        code = binding.KATA_BF16 if k.dtype == torch.bfloat16 else binding.KATA_F32
        n = binding.kata_chunked_forward_workspace_bytes(B, H, T, dk, v.shape[-1], C, code)
        return torch.empty(max(n, 256), dtype=torch.uint8, device=k.device)

    @staticmethod
    def chunked_state(k, v, C, state_out, z_out, workspace):
        binding.kata_chunked_state(k, v, C=C, state_out=state_out, z_out=z_out,
                                   workspace=workspace)

    @staticmethod
    def forward_from_state(q, k, v, state_in, z_in, C, out, state_out, z_out, workspace, reuse):
        binding.kata_chunked_forward_from_state(q, k, v, state_in, z_in, C=C, out=out,
                                                state_out=state_out, z_out=z_out,
                                                workspace=workspace, reuse_segment_states=reuse)


def state_numel(B, H, dk, dv):
    """(floats of S, floats of Z) of one block's state."""
    return B * H * dk * dk * dv, B * H * dk * dk


def block_state(k, v, C=64, ops=LibkataOps, workspace=None):
    """This block's total state as one flat fp32 buffer [S | Z].  `workspace`
    (from ops.workspace) then holds the block's per-segment states for
    block_forward(..., reuse=True)."""
    import torch

    B, H, _, dk = k.shape
    dv = v.shape[-1]
    ns, nz = state_numel(B, H, dk, dv)
    flat = torch.empty(ns + nz, dtype=torch.float32, device=k.device)
    if workspace is None:
        workspace = ops.workspace(k, v, C)
    ops.chunked_state(k, v, C, flat[:ns].view(B, H, dk * dk, dv), flat[ns:].view(B, H, dk, dk),
                      workspace)
    return flat


def gathered_views(gathered, n, B, H, dk, dv):
    """The first n states of a gathered [world, |S| + |Z|] buffer, as strided
    stacks S [n, B, H, dk*dk, dv] and Z [n, B, H, dk, dk] (no copy)."""
    ns, nz = state_numel(B, H, dk, dv)
    row = gathered.stride(0)
    s = gathered.as_strided((n, B, H, dk * dk, dv), (row, H * dk * dk * dv, dk * dk * dv, dv, 1),
                            gathered.storage_offset())
    z = gathered.as_strided((n, B, H, dk, dk), (row, H * dk * dk, dk * dk, dk, 1),
                            gathered.storage_offset() + ns)
    return s, z


def block_forward(q, k, v, gathered, rank, C=64, out=None, state_out=None, z_out=None,
                  ops=LibkataOps, workspace=None, reuse=False):
    """Outputs of block `rank`, starting from the sum of the totals of blocks
    0 .. rank-1 (rows of `gathered`).  reuse: `workspace` is the one
    block_state filled for these k, v, untouched since."""
    import torch

    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    if workspace is None:
        workspace, reuse = ops.workspace(k, v, C), False
    s_in, z_in = gathered_views(gathered, rank, B, H, dk, dv)
    ops.forward_from_state(q, k, v, s_in, z_in, C, out, state_out, z_out, workspace, reuse)
    return out


def sequence_sharded_forward(q, k, v, C=64, group=None, out=None, state_out=None, z_out=None,
                             ops=LibkataOps):
    """This rank's block of the causal forward of one sequence sharded over the
    ranks of `group` in rank order (q, k, v [B, H, T_r, d] are this rank's
    tokens; blocks may differ in length).  Runs on the current CUDA stream."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ws = ops.workspace(k, v, C)
    flat = block_state(k, v, C, ops, ws)
    gathered = torch.empty(world * flat.numel(), dtype=flat.dtype, device=flat.device)
    dist.all_gather_into_tensor(gathered, flat, group=group)
    return block_forward(q, k, v, gathered.view(world, flat.numel()), rank, C, out, state_out,
                         z_out, ops, ws, reuse=True)
