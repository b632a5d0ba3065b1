"""Sequence-sharded forward: the multi-rank orchestration on CPU (gloo; no GPU).

`kernelized_linear_attention_fwd_b200.sharded` splits one sequence into
contiguous blocks, one per rank: each rank computes its block's total state,
the ranks all-gather those totals, and rank r continues its forward from the
sum of the totals of ranks 0 .. r-1.  Here the two library calls are replaced
by oracle-backed stand-ins (the state by direct summation, the forward from a
given state as token-by-token decode steps), so what is tested is the host
logic: the gather layout, the strided views into the gathered buffer, and
that rank r starts from exactly the earlier ranks' totals.  Concatenated over
ranks, the outputs must equal the oracle's quadratic forward of the whole
sequence, and each rank's state output the oracle's state after its block.
The GPU path itself is tested in tests/test_from_state_gpu.py.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleOps:
    """fp64 oracle stand-ins for kata_chunked_state and
    kata_chunked_forward_from_state, on CPU tensors.  The workspace records the
    keys the state call saw, so a forward told to reuse it checks that it got
    the workspace of its own block's state call."""

    @staticmethod
    def workspace(k, v, C):
        return {"keys": None}

    @staticmethod
    def chunked_state(k, v, C, state_out, z_out, workspace):
        workspace["keys"] = k
        from oracle import oracle

        S, Z = oracle.state(k.double().numpy(), v.double().numpy())
        state_out.copy_(torch.from_numpy(S))
        z_out.copy_(torch.from_numpy(Z))

    @staticmethod
    def forward_from_state(q, k, v, state_in, z_in, C, out, state_out, z_out, workspace, reuse):
        from oracle import oracle

        assert not reuse or workspace["keys"] is k  # reused only for the same block

        B, H, T, dk = q.shape
        dv = v.shape[-1]
        BH = B * H
        S = state_in.double().sum(0).reshape(BH, dk * dk, dv).numpy()
        Z = z_in.double().sum(0).reshape(BH, dk, dk).numpy()
        qn, kn, vn = (x.double().reshape(BH, T, -1).numpy() for x in (q, k, v))
        for t in range(T):
            y, S, Z, _ = oracle.decode_step(qn[:, t], kn[:, t], vn[:, t], S, Z)
            out[:, :, t] = torch.from_numpy(y.reshape(B, H, dv))
        if state_out is not None:
            state_out.copy_(torch.from_numpy(S.reshape(B, H, dk * dk, dv)))
            z_out.copy_(torch.from_numpy(Z.reshape(B, H, dk, dk)))


def _worker(rank, world, port, bounds, results):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from kernelized_linear_attention_fwd_b200 import inputs, sharded

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = inputs.make_qkv(1, 2, bounds[-1], 4, 4, "f32", seed=5)
        lo, hi = bounds[rank], bounds[rank + 1]
        blk = [torch.from_numpy(np.ascontiguousarray(x[:, :, lo:hi])) for x in (q, k, v)]
        so = torch.empty((1, 2, 16, 4), dtype=torch.float32)
        zo = torch.empty((1, 2, 4, 4), dtype=torch.float32)
        out = sharded.sequence_sharded_forward(*blk, C=16, state_out=so, z_out=zo,
                                               ops=OracleOps)
        results[rank] = (out.numpy(), so.numpy(), zo.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bounds", [(0, 40, 96), (0, 33, 34, 90)])
def test_ranks_continue_from_the_earlier_ranks_totals(oracle_mod, bounds):
    world = len(bounds) - 1
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, _free_port(), bounds, results), nprocs=world, join=True)
        res = dict(results)
    sys.path.insert(0, ROOT)
    from kernelized_linear_attention_fwd_b200 import inputs

    T = bounds[-1]
    q, k, v = (inputs.widen(x, "f32") for x in inputs.make_qkv(1, 2, T, 4, 4, "f32", seed=5))
    yref = oracle_mod.forward(q, k, v)
    y = np.concatenate([res[r][0] for r in range(world)], axis=2)
    np.testing.assert_allclose(y, yref, rtol=0, atol=1e-5 * np.abs(yref).max())
    for r in range(world):
        S, Z = oracle_mod.state(k, v, n=bounds[r + 1])
        np.testing.assert_allclose(res[r][1], S, rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(res[r][2], Z, rtol=1e-5, atol=1e-5)


def test_gathered_views_pick_rows_without_copy():
    from kernelized_linear_attention_fwd_b200 import sharded

    B, H, dk, dv = 2, 3, 4, 4
    ns, nz = sharded.state_numel(B, H, dk, dv)
    g = torch.arange(4 * (ns + nz), dtype=torch.float32).view(4, ns + nz)
    s, z = sharded.gathered_views(g, 3, B, H, dk, dv)
    assert s.shape == (3, B, H, dk * dk, dv) and z.shape == (3, B, H, dk, dk)
    for m in range(3):
        assert torch.equal(s[m].reshape(-1), g[m, :ns])
        assert torch.equal(z[m].reshape(-1), g[m, ns:])
        assert s[m].is_contiguous() and z[m].is_contiguous()
    assert s.data_ptr() == g.data_ptr() and s.stride(0) == z.stride(0) == ns + nz
    s0, z0 = sharded.gathered_views(g, 0, B, H, dk, dv)
    assert s0.shape[0] == 0 and z0.shape[0] == 0
