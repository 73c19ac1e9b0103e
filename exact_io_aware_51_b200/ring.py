"""Ring attention: exact attention over a sequence split across ranks.

"Flash Attention" (Ultralytics glossary), "Flash Attention и смежные понятия"
(ring attention): a very long sequence is split between devices; each device
computes blockwise attention for its own part while the key/value blocks are
passed around a ring.

Rank r of W holds the r-th chunk of the sequence: q, k, v (and, for the
backward, o, do, lse) of shape [B, N/W, heads, d].  At step s it works on the
key/value chunk c = (r - s) mod W that the ring has brought to it:

* forward: the kernels compute exact attention of q against chunk c alone
  (causal masking: c < r sees every key, c == r is the causal diagonal, c > r is
  skipped) and `merge_partial` folds that partial (O_c, LSE_c) into the running
  result with the online softmax's correction;
* backward: with the final O and LSE of the whole row, the gradients of one
  chunk pair are the ordinary recomputed backward of that pair (P = exp(S - LSE)
  uses the global LSE, D = rowsum(dO * O) the global O), so dQ sums the pair
  gradients locally and dK, dV travel around the ring with their chunk and are
  summed in fp32 on the way back to the chunk's owner.

The transport is torch.distributed point-to-point (NCCL between GPUs); the
next chunk's exchange is started before the current chunk's kernels and
finished after them, so the transfer overlaps the compute.  Every arithmetic
step runs in the library's kernels (attention, merge, fp32 accumulation, cast).
"""

from __future__ import annotations

import dataclasses

import torch


class DistRing:
    """Ring transport over torch.distributed (default group): send to rank + 1, receive from rank - 1."""

    def __init__(self):
        import torch.distributed as dist
        self.dist = dist
        self.rank = dist.get_rank()
        self.world = dist.get_world_size()

    def exchange(self, tensors):
        """Start sending `tensors` to the next rank and receiving the same shapes from the
        previous one; returns a handle whose wait() gives the received tensors."""
        d = self.dist
        nxt, prv = (self.rank + 1) % self.world, (self.rank - 1) % self.world
        recv = [torch.empty_like(t) for t in tensors]
        ops = [d.P2POp(d.isend, t.contiguous(), nxt) for t in tensors]
        ops += [d.P2POp(d.irecv, t, prv) for t in recv]
        reqs = d.batch_isend_irecv(ops)
        return _Pending(reqs, recv)


class _Pending:
    def __init__(self, reqs, recv):
        self.reqs, self.recv = reqs, recv

    def wait(self):
        for rq in self.reqs:
            rq.wait()
        return self.recv


@dataclasses.dataclass
class KernelOps:
    """The library's kernels, as the ring algorithm calls them."""

    acc_dtype: torch.dtype = torch.float32  # running output and gradient sums

    def fwd(self, q, k, v, causal, scale):
        from . import fwd
        return fwd(q, k, v, causal=causal, scale=scale)

    def bwd(self, q, k, v, o, do, lse, causal, scale):
        from . import bwd
        return bwd(q, k, v, o, do, lse, causal=causal, scale=scale)

    def merge(self, o_acc, lse_acc, o_part, lse_part, init):
        from . import merge_partial
        merge_partial(o_acc, lse_acc, o_part, lse_part, init=init)

    def accumulate(self, acc, part, init):
        from . import accumulate
        accumulate(acc, part, init=init)

    def cast(self, x):
        from . import cast_bf16
        return cast_bf16(x)


def _visible(causal: bool, c: int, r: int) -> bool:
    return not (causal and c > r)


def ring_forward(q, k, v, *, causal: bool = False, scale: float | None = None, ring=None, ops=None):
    """Forward of rank ring.rank: returns (o [B, Nc, H, d] bf16, lse [B, H, Nc] fp32) of its query chunk."""
    ring = ring if ring is not None else DistRing()
    ops = ops if ops is not None else KernelOps()
    W, r = ring.world, ring.rank
    B, Nc, H, d = q.shape
    o_acc = torch.empty((B, Nc, H, d), dtype=ops.acc_dtype, device=q.device)
    lse_acc = torch.empty((B, H, Nc), dtype=ops.acc_dtype, device=q.device)
    kv = (k, v)
    first = True
    for s in range(W):
        c = (r - s) % W
        pending = ring.exchange(kv) if s + 1 < W else None  # the next chunk travels while this one computes
        if _visible(causal, c, r):
            o_p, lse_p = ops.fwd(q, kv[0], kv[1], causal and c == r, scale)
            ops.merge(o_acc, lse_acc, o_p, lse_p, first)
            first = False
        if pending is not None:
            kv = tuple(pending.wait())
    return ops.cast(o_acc), lse_acc


def ring_backward(q, k, v, o, do, lse, *, causal: bool = False, scale: float | None = None, ring=None, ops=None):
    """Backward of rank ring.rank given its chunk's final o and lse: returns (dq, dk, dv) of its chunks (bf16)."""
    ring = ring if ring is not None else DistRing()
    ops = ops if ops is not None else KernelOps()
    W, r = ring.world, ring.rank
    dq_acc = torch.empty(q.shape, dtype=ops.acc_dtype, device=q.device)
    dk_acc = torch.empty(k.shape, dtype=ops.acc_dtype, device=k.device)
    dv_acc = torch.empty(v.shape, dtype=ops.acc_dtype, device=v.device)
    kv = (k, v)
    dq_first = True
    for s in range(W):
        c = (r - s) % W
        pending_kv = ring.exchange(kv) if s + 1 < W else None
        if _visible(causal, c, r):
            dq_p, dk_p, dv_p = ops.bwd(q, kv[0], kv[1], o, do, lse, causal and c == r, scale)
            ops.accumulate(dq_acc, dq_p, dq_first)
            dq_first = False
            # step 0 is always the rank's own chunk (visible), so its owner starts the sums
            ops.accumulate(dk_acc, dk_p, s == 0)
            ops.accumulate(dv_acc, dv_p, s == 0)
        # chunk c's gradient sums follow chunk c; after W hops they are back with the owner
        dk_acc, dv_acc = ring.exchange((dk_acc, dv_acc)).wait() if W > 1 else (dk_acc, dv_acc)
        if pending_kv is not None:
            kv = tuple(pending_kv.wait())
    return ops.cast(dq_acc), ops.cast(dk_acc), ops.cast(dv_acc)
