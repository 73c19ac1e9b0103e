"""Ring attention's schedule on CPU: gloo ranks, fp64 stand-ins for the kernels.

The ring algorithm (exact_io_aware_51_b200.ring) is the same code the GPUs
run; here its transport is torch.distributed over gloo and the per-chunk
kernels are replaced by plain fp64 stand-ins written below from the
definitions (chunk attention via the oracle, the pair backward with the global
LSE, the merge and the sums).  What is checked is the decomposition: the
assembled outputs and gradients of all ranks equal the oracle on the whole
sequence, for 1, 2 and 3 ranks, with and without the causal mask, including
grouped K/V heads.
"""

from __future__ import annotations

import math
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class Fp64Ops:
    """Test stand-ins for the library's kernels (fp64 torch / oracle on CPU)."""

    acc_dtype = torch.float64

    def fwd(self, q, k, v, causal, scale):
        import oracle
        o, lse = oracle.forward(q, k, v, scale, causal)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def bwd(self, q, k, v, o, do, lse, causal, scale):
        # one chunk pair's gradients with the row's global LSE and O
        G = q.shape[2] // k.shape[2]
        kk, vv = k.repeat_interleave(G, dim=2), v.repeat_interleave(G, dim=2)
        s = scale * torch.einsum("bqhd,bkhd->bhqk", q, kk)
        if causal:
            n = s.shape[-1]
            s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), -math.inf)
        p = torch.exp(s - lse[..., None])
        dv = torch.einsum("bhqk,bqhd->bkhd", p, do)
        dp = torch.einsum("bqhd,bkhd->bhqk", do, vv)
        dvec = (do * o).sum(-1).permute(0, 2, 1)[..., None]
        ds = p * (dp - dvec)
        dq = scale * torch.einsum("bhqk,bkhd->bqhd", ds, kk)
        dk = scale * torch.einsum("bhqk,bqhd->bkhd", ds, q)
        B, N, Hkv, d = k.shape
        return dq, dk.reshape(B, N, Hkv, G, d).sum(3), dv.reshape(B, N, Hkv, G, d).sum(3)

    def merge(self, o_acc, lse_acc, o_part, lse_part, init):
        if init:
            o_acc.copy_(o_part)
            lse_acc.copy_(lse_part)
            return
        m = torch.maximum(lse_acc, lse_part)
        wa, wb = torch.exp(lse_acc - m), torch.exp(lse_part - m)
        wa_, wb_ = wa.permute(0, 2, 1)[..., None], wb.permute(0, 2, 1)[..., None]
        o_acc.copy_((wa_ * o_acc + wb_ * o_part) / (wa_ + wb_))
        lse_acc.copy_(m + torch.log(wa + wb))

    def accumulate(self, acc, part, init):
        if init:
            acc.copy_(part)
        else:
            acc.add_(part)

    def cast(self, x):
        return x.clone()


def _worker(rank, world, port, causal, H, Hkv, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from exact_io_aware_51_b200 import ring as R
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(0)
        B, N, d = 1, 60, 8
        q = torch.randn(B, N, H, d, generator=g, dtype=torch.float64)
        k = torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64)
        v = torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64)
        do = torch.randn(B, N, H, d, generator=g, dtype=torch.float64)
        c = N // world
        sl = slice(rank * c, (rank + 1) * c)
        args = [t[:, sl].contiguous() for t in (q, k, v)]
        ops = Fp64Ops()
        o, lse = R.ring_forward(*args, causal=causal, scale=0.37, ops=ops, ring=R.DistRing())
        dq, dk, dv = R.ring_backward(*args, o, do[:, sl].contiguous(), lse, causal=causal, scale=0.37, ops=ops,
                                     ring=R.DistRing())
        q_out.put((rank, o.numpy(), lse.numpy(), dq.numpy(), dk.numpy(), dv.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _reference(causal, H, Hkv):
    import oracle
    g = torch.Generator().manual_seed(0)
    B, N, d = 1, 60, 8
    q = torch.randn(B, N, H, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, N, Hkv, d, generator=g, dtype=torch.float64)
    do = torch.randn(B, N, H, d, generator=g, dtype=torch.float64)
    o, lse = oracle.forward(q, k, v, 0.37, causal)
    dq, dk, dv = oracle.backward(q, k, v, do, 0.37, causal)
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 2)])
def test_ring_attention_equals_full_attention(world, causal, H, Hkv):
    ctx = mp.get_context("spawn")
    qo = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, H, Hkv, qo)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(qo.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    o = np.concatenate([r[1] for r in res], axis=1)
    lse = np.concatenate([r[2] for r in res], axis=2)
    dq, dk, dv = (np.concatenate([r[i] for r in res], axis=1) for i in (3, 4, 5))
    ro, rl, rq, rk, rv = _reference(causal, H, Hkv)
    for got, ref in ((o, ro), (lse, rl), (dq, rq), (dk, rk), (dv, rv)):
        assert np.max(np.abs(got - ref)) < 1e-10
