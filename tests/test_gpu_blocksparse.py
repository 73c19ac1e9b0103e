"""Block-sparse attention parity: the CUDA path against the fp64 oracle.

"Flash Attention" (Ultralytics glossary), "Flash Attention и смежные понятия":
sparse attention scores only chosen query/key pairs, and the block-sparse form
skips the empty blocks.  The mask is 0/1 over 128 x 128 blocks (shared by all
heads or one per query head); masks are drawn at random with fixed seeds and
include rows of blocks that see nothing (O = 0, LSE = -inf, dQ = 0) and key
blocks no query sees (dK = dV = 0).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import exact_io_aware_51_b200 as fa
import oracle
from exact_io_aware_51_b200 import inputs as I
from tests.helpers import TOL_BF16_REL, TOL_F32_O, TOL_LSE, abs_err, need_gpu, rel_err


def _scale(d):
    return float(np.float32(1.0 / math.sqrt(d)))


def _mask(nb, heads, density, seed, empty_row=None, empty_col=None):
    m = (np.random.default_rng(seed).random((heads, nb, nb)) < density).astype(np.uint8)
    if empty_row is not None:
        m[:, empty_row, :] = 0
    if empty_col is not None:
        m[:, :, empty_col] = 0
    return m if heads > 1 else m[0]


def _lse_close(got, ref):
    """LSE within the bound, rows with no visible key -inf on both sides."""
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    both_inf = np.isneginf(got) & np.isneginf(ref)
    with np.errstate(invalid="ignore"):
        close = np.abs(got - ref) <= TOL_LSE
    return bool(np.all(both_inf | close))


@pytest.mark.gpu
@pytest.mark.parametrize("n,d", [(200, 64), (384, 128), (700, 128), (1000, 64)])
@pytest.mark.parametrize("heads_mask", [1, 3])
def test_blocksparse_forward(n, d, heads_mask):
    need_gpu()
    nb = (n + 127) // 128
    m = _mask(nb, heads_mask, 0.5, n + heads_mask, empty_row=nb // 2)
    q, k, v, _ = I.make_inputs(2, n, 3, d, seed=n, with_do=False)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), scale=_scale(d), block_mask=torch.from_numpy(m).cuda())
    torch.cuda.synchronize()
    ro, rl = oracle.forward(q, k, v, _scale(d), False, block_mask=m)
    assert rel_err(o.cpu(), ro) <= TOL_BF16_REL
    assert _lse_close(lse.cpu(), rl)


@pytest.mark.gpu
@pytest.mark.parametrize("n,d", [(256, 64), (333, 128), (700, 64)])
@pytest.mark.parametrize("heads_mask", [1, 2])
def test_blocksparse_forward_fp32(n, d, heads_mask):
    """The exact fp32 forward under a block mask: every element within 1e-5,
    including a block row that sees nothing (O = 0, LSE = -inf)."""
    need_gpu()
    nb = (n + 127) // 128
    m = _mask(nb, heads_mask, 0.5, 7 * n + heads_mask, empty_row=nb - 1)
    q, k, v, _ = I.make_inputs(1, n, 2, d, seed=n + 1, dtype="fp32", with_do=False)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), scale=_scale(d), block_mask=torch.from_numpy(m).cuda())
    torch.cuda.synchronize()
    ro, rl = oracle.forward(q, k, v, _scale(d), False, block_mask=m)
    assert abs_err(o.cpu(), ro) <= TOL_F32_O
    assert _lse_close(lse.cpu(), rl)
    assert fa.last_device_status()[0] == 0


@pytest.mark.gpu
@pytest.mark.parametrize("n", [384, 640])
@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_backward(n, causal):
    need_gpu()
    nb = (n + 127) // 128
    m = _mask(nb, 1, 0.6, 7 * n + causal)
    m[np.arange(nb), np.arange(nb)] = 1  # keep the diagonal so causal rows see their own key
    m[:, 1] = 0  # ... except in key block 1, which no query block sees
    sc = _scale(128)
    q, k, v, do = I.make_inputs(2, n, 2, 128, seed=n + 5)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    md = torch.from_numpy(m).cuda()
    o, lse = fa.fwd(qd, kd, vd, causal=causal, scale=sc, block_mask=md)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=sc, block_mask=md)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.backward(q, k, v, do, sc, causal, block_mask=m)
    assert rel_err(dq.cpu(), rq) <= TOL_BF16_REL
    assert rel_err(dk.cpu(), rk) <= TOL_BF16_REL
    assert rel_err(dv.cpu(), rv) <= TOL_BF16_REL
    # key block 1 is seen by no query: its gradients are exactly zero
    assert torch.count_nonzero(dk[:, 128:256]) == 0 and torch.count_nonzero(dv[:, 128:256]) == 0
    assert fa.last_device_status()[0] == 0


@pytest.mark.gpu
def test_blocksparse_per_head_masks_with_gqa_and_window():
    need_gpu()
    n, H, Hkv = 512, 4, 2
    nb = n // 128
    m = _mask(nb, H, 0.5, 3)
    m[:, np.arange(nb), np.arange(nb)] = 1
    sc = _scale(128)
    q, k, v, do = I.make_inputs(1, n, H, 128, seed=9, kv_heads=Hkv)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    md = torch.from_numpy(m).cuda()
    win = (300, 40)
    o, lse = fa.fwd(qd, kd, vd, scale=sc, window=win, block_mask=md)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, scale=sc, window=win, block_mask=md)
    torch.cuda.synchronize()
    ro, rl = oracle.forward(q, k, v, sc, False, window=win, block_mask=m)
    rq, rk, rv = oracle.backward(q, k, v, do, sc, False, window=win, block_mask=m)
    assert rel_err(o.cpu(), ro) <= TOL_BF16_REL and _lse_close(lse.cpu(), rl)
    for g, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert rel_err(g.cpu(), r) <= TOL_BF16_REL


@pytest.mark.gpu
def test_all_ones_mask_equals_dense_bitwise():
    need_gpu()
    n = 1000
    q, k, v, _ = I.make_inputs(1, n, 4, 128, seed=13, with_do=False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ones = torch.ones((8, 8), dtype=torch.uint8, device="cuda")
    o1, l1 = fa.fwd(qd, kd, vd)
    o2, l2 = fa.fwd(qd, kd, vd, block_mask=ones)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.gpu
def test_blocksparse_n16384_skips_work():
    """A 10 % block mask at B1 H16 N16384: sampled rows match the oracle, and the
    forward takes well under a quarter of the dense forward's time."""
    need_gpu()
    n, H = 16384, 16
    nb = n // 128
    m = _mask(nb, 1, 0.1, 21)
    m[np.arange(nb), np.arange(nb)] = 1
    q, k, v, _ = I.make_inputs(1, n, H, 128, seed=22, with_do=False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    md = torch.from_numpy(m).cuda()
    o, lse = fa.fwd(qd, kd, vd, block_mask=md)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(1).choice(n, 200, replace=False))
    from tests.helpers import f64
    ro, rl = oracle.forward_rows_head(f64(q[0, :, 5]), f64(k[0, :, 5]), f64(v[0, :, 5]), rows, _scale(128), False,
                                      block_mask=m)
    assert rel_err(o[0, rows, 5].cpu(), ro) <= TOL_BF16_REL
    assert _lse_close(lse[0, 5, rows].cpu(), rl)

    def t_ms(fn):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(5):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / 5
    dense = t_ms(lambda: fa.fwd(qd, kd, vd))
    sparse = t_ms(lambda: fa.fwd(qd, kd, vd, block_mask=md))
    assert sparse < 0.25 * dense, (sparse, dense)
