"""Split backward walks on small grids: dK, dV summed over several CTAs.

When a problem gives fewer than three waves of key-tile CTAs, the backward
splits each key tile's (query head, query tile) walk over up to 8 CTAs that
add fp32 partial dK, dV into accumulators; a convert kernel writes the bf16
results.  These tests take shapes that split (checked through the workspace
size), compare with the fp64 oracle, and check that a workspace without the
accumulators gives the same result without splitting.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import exact_io_aware_51_b200 as fa
import oracle
from exact_io_aware_51_b200 import inputs as I
from tests.helpers import TOL_BF16_REL, need_gpu, rel_err


def _splits(B, H, Hkv, N, d):
    full = fa.bwd_workspace_size(B, H, N, d, kv_heads=Hkv)
    base = B * N * H * d * 4 + 2 * B * H * ((N + 127) // 128 * 128) * 4
    return full > base + 1024


CASES = [  # (B, H, Hkv, N, d, kw): all split
    (1, 4, 4, 4096, 128, {}),
    (1, 4, 4, 4096, 128, {"causal": True}),
    (1, 8, 2, 2048, 128, {"window": (300, 0)}),
    (1, 4, 4, 4096, 64, {}),
    (1, 8, 1, 2048, 64, {"causal": True}),
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,Hkv,N,d,kw", CASES, ids=lambda x: str(x))
def test_split_backward_matches_oracle(B, H, Hkv, N, d, kw):
    need_gpu()
    assert _splits(B, H, Hkv, N, d)
    sc = float(np.float32(1.0 / math.sqrt(d)))
    q, k, v, do = I.make_inputs(B, N, H, d, seed=N + H + d, kv_heads=Hkv)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, scale=sc, **kw)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, scale=sc, **kw)
    torch.cuda.synchronize()
    assert fa.last_device_status()[0] == 0
    causal = kw.get("causal", False)
    window = kw.get("window")
    heads = [(0, 0), (0, H - 1)]
    G = H // Hkv
    # dK, dV of a K/V head need every query head of its group
    kv_heads = sorted({h // G for (_, h) in heads})
    all_heads = [(0, h) for g in kv_heads for h in range(g * G, (g + 1) * G)]
    rq, rk, rv = oracle.backward(q, k, v, do, sc, causal, heads=all_heads, window=window)
    for (_, h) in heads:
        assert rel_err(dq[0, :, h].cpu(), rq[0, :, h]) <= TOL_BF16_REL
    for g in kv_heads:
        assert rel_err(dk[0, :, g].cpu(), rk[0, :, g]) <= TOL_BF16_REL
        assert rel_err(dv[0, :, g].cpu(), rv[0, :, g]) <= TOL_BF16_REL


@pytest.mark.gpu
def test_split_and_unsplit_agree():
    """A workspace without the dK / dV accumulators runs unsplit; both results agree
    to fp32 summation order and one bf16 rounding."""
    need_gpu()
    B, H, Hkv, N, d = 1, 8, 2, 2048, 128
    q, k, v, do = (t.cuda() for t in I.make_inputs(B, N, H, d, seed=3, kv_heads=Hkv))
    o, lse = fa.fwd(q, k, v)
    full = fa.bwd_workspace_size(B, H, N, d, kv_heads=Hkv)
    base = B * N * H * d * 4 + 2 * B * H * N * 4
    assert full > base
    split = fa.bwd(q, k, v, o, do, lse, workspace=torch.empty(full, dtype=torch.uint8, device="cuda"))
    plain = fa.bwd(q, k, v, o, do, lse, workspace=torch.empty(base, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    for a_, b_ in zip(split, plain):
        assert rel_err(a_.cpu(), b_.cpu()) <= 1e-2


@pytest.mark.gpu
def test_split_blocksparse():
    need_gpu()
    B, H, N, d = 1, 4, 4096, 128
    nb = N // 128
    m = (np.random.default_rng(5).random((nb, nb)) < 0.5).astype(np.uint8)
    m[np.arange(nb), np.arange(nb)] = 1
    assert _splits(B, H, H, N, d)
    sc = float(np.float32(1.0 / math.sqrt(d)))
    q, k, v, do = I.make_inputs(B, N, H, d, seed=8)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    md = torch.from_numpy(m).cuda()
    o, lse = fa.fwd(qd, kd, vd, scale=sc, block_mask=md)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, scale=sc, block_mask=md)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.backward(q, k, v, do, sc, False, heads=[(0, 2)], block_mask=m)
    for g_, r_ in ((dq, rq), (dk, rk), (dv, rv)):
        assert rel_err(g_[0, :, 2].cpu(), r_[0, :, 2]) <= TOL_BF16_REL
