"""Ring attention with the library's kernels on one GPU, W ranks emulated.

The ring algorithm runs unchanged (exact_io_aware_51_b200.ring with the
library's kernels: chunk attention, merge, fp32 sums, casts); only the
transport differs: W Python threads stand in for W ranks and hand each other
their chunks through queues on the same device.  The assembled outputs and
gradients are compared with the fp64 oracle on the whole sequence.  The
point-to-point transport itself is covered on CPU by tests/test_ring_cpu.py.
"""

from __future__ import annotations

import math
import queue
import threading

import numpy as np
import pytest
import torch

import exact_io_aware_51_b200 as fa
import oracle
from exact_io_aware_51_b200 import inputs as I
from exact_io_aware_51_b200 import ring as R
from tests.helpers import TOL_BF16_REL, TOL_LSE, abs_err, need_gpu, rel_err


class ThreadRing:
    """One rank's end of an in-process ring (test transport).

    Like point-to-point messages, the i-th exchange a rank starts receives the
    i-th message its left neighbour sent, whatever order the waits come in."""

    def __init__(self, rank, world, inboxes):
        self.rank, self.world, self.inboxes = rank, world, inboxes
        self.sent = self.posted = 0
        self.early = {}

    def exchange(self, tensors):
        torch.cuda.synchronize()  # the tensors handed on are complete
        self.inboxes[(self.rank + 1) % self.world].put((self.sent, list(tensors)))
        self.sent += 1
        self.posted += 1
        return _Handle(self, self.posted - 1)

    def receive(self, seq):
        while seq not in self.early:
            k, ts = self.inboxes[self.rank].get(timeout=120)
            self.early[k] = ts
        return self.early.pop(seq)


class _Handle:
    def __init__(self, ring, seq):
        self.ring, self.seq = ring, seq

    def wait(self):
        return self.ring.receive(self.seq)


def _run_ranks(world, fn):
    inboxes = [queue.Queue() for _ in range(world)]
    out, errs = [None] * world, []

    def body(r):
        try:
            out[r] = fn(r, ThreadRing(r, world, inboxes))
        except Exception as e:  # noqa: BLE001 - reported below
            errs.append(e)

    ts = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(timeout=300)
    if errs:
        raise errs[0]
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_forward_backward_match_full_attention(world, causal):
    need_gpu()
    B, N, H, Hkv, d = 1, 1024, 4, 2, 128
    sc = float(np.float32(1.0 / math.sqrt(d)))
    q, k, v, do = I.make_inputs(B, N, H, d, seed=world + 10 * causal, kv_heads=Hkv)
    c = N // world

    def rank_fn(r, ring):
        sl = slice(r * c, (r + 1) * c)
        qr, kr, vr, dor = (t[:, sl].contiguous().cuda() for t in (q, k, v, do))
        o, lse = R.ring_forward(qr, kr, vr, causal=causal, scale=sc, ring=ring)
        dq, dk, dv = R.ring_backward(qr, kr, vr, o, dor, lse, causal=causal, scale=sc, ring=ring)
        torch.cuda.synchronize()
        return [t.cpu() for t in (o, lse, dq, dk, dv)]

    res = _run_ranks(world, rank_fn)
    o, dq, dk, dv = (torch.cat([r[i] for r in res], dim=1) for i in (0, 2, 3, 4))
    lse = torch.cat([r[1] for r in res], dim=2)
    ro, rl = oracle.forward(q, k, v, sc, causal)
    rq, rk, rv = oracle.backward(q, k, v, do, sc, causal)
    assert rel_err(o, ro) <= TOL_BF16_REL
    assert abs_err(lse, rl) <= TOL_LSE
    for g, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert rel_err(g, ref) <= TOL_BF16_REL
    assert fa.last_device_status()[0] == 0


@pytest.mark.gpu
def test_merge_of_two_key_halves_equals_one_pass():
    """fa_merge_partial: merging a partial with itself is attention over the same keys
    twice (O unchanged, LSE + ln 2), which is also what one forward pass over the
    doubled key set gives."""
    need_gpu()
    B, N, H, d = 2, 512, 3, 64
    q, k, v, _ = (t.cuda() if t is not None else None for t in I.make_inputs(B, N, H, d, seed=3, with_do=False))
    # a single pass over both halves of the keys: queries attend to the concatenation
    o_full, l_full = fa.fwd(torch.cat([q, q], 1), torch.cat([k, k], 1), torch.cat([v, v], 1))
    o1, l1 = fa.fwd(q, k, v)
    o_acc = torch.empty(o1.shape, dtype=torch.float32, device="cuda")
    l_acc = torch.empty_like(l1)
    out = torch.empty_like(o1)
    fa.merge_partial(o_acc, l_acc, o1, l1, init=True)
    fa.merge_partial(o_acc, l_acc, o1, l1, o_out=out)
    torch.cuda.synchronize()
    # the same keys twice: O unchanged, LSE + ln 2
    assert rel_err(o_acc.cpu(), o1.float().cpu()) <= 1e-6
    assert abs_err(l_acc.cpu(), (l1 + math.log(2.0)).cpu()) <= 1e-5
    assert torch.equal(out, fa.cast_bf16(o_acc))
    # the single forward over the doubled key set (its first N query rows)
    assert rel_err(o_full[:, :N].float().cpu(), o_acc.cpu()) <= TOL_BF16_REL
