"""Sliding-window attention parity: the CUDA path against the fp64 oracle.

"Flash Attention" (karlkratz.de), section "Sliding Window Attention": each
position attends to a fixed neighbourhood, and blocks wholly outside it are
skipped.  Key j is visible to query i when i - left <= j <= i + right; the
page's 4096-token window (Mistral 7B) is (4095, 0).  Windows are chosen to put
the edge inside a tile, on a tile boundary, one past it, and to cover open
sides, a zero-width window and grouped K/V heads.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import exact_io_aware_51_b200 as fa
import oracle
from exact_io_aware_51_b200 import inputs as I
from tests.helpers import TOL_BF16_REL, TOL_F32_O, TOL_LSE, abs_err, f64, need_gpu, rel_err


def _scale(d):
    return float(np.float32(1.0 / math.sqrt(d)))


FWD_WINDOWS = [(0, 0), (1, 0), (63, 0), (127, 0), (128, 0), (129, 5), (300, 300), (None, 64), (64, None),
               (0, 129)]


@pytest.mark.gpu
@pytest.mark.parametrize("window", FWD_WINDOWS, ids=str)
@pytest.mark.parametrize("n,d", [(200, 64), (384, 128), (700, 128)])
def test_window_forward_small(window, n, d):
    need_gpu()
    q, k, v, _ = I.make_inputs(2, n, 3, d, seed=n + d, with_do=False)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), scale=_scale(d), window=window)
    torch.cuda.synchronize()
    ro, rl = oracle.forward(q, k, v, _scale(d), False, window=window)
    assert rel_err(o.cpu(), ro) <= TOL_BF16_REL
    assert abs_err(lse.cpu(), rl) <= TOL_LSE


@pytest.mark.gpu
@pytest.mark.parametrize("window", [(0, 0), (37, 0), (128, 3), (None, 100)], ids=str)
def test_window_forward_fp32(window):
    need_gpu()
    q, k, v, _ = I.make_inputs(1, 333, 2, 64, seed=4, dtype="fp32", with_do=False)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), scale=_scale(64), window=window)
    torch.cuda.synchronize()
    ro, rl = oracle.forward(q, k, v, _scale(64), False, window=window)
    assert abs_err(o.cpu(), ro) <= TOL_F32_O
    assert abs_err(lse.cpu(), rl) <= TOL_LSE


BWD_WINDOWS = [(0, 0), (100, 0), (127, 0), (128, 0), (129, 17), (None, 200), (255, 255), (0, 300)]


@pytest.mark.gpu
@pytest.mark.parametrize("window", BWD_WINDOWS, ids=str)
@pytest.mark.parametrize("n", [333, 640])
def test_window_backward_small(window, n):
    need_gpu()
    sc = _scale(128)
    q, k, v, do = I.make_inputs(2, n, 2, 128, seed=3 * n + 1)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, scale=sc, window=window)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, scale=sc, window=window)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.backward(q, k, v, do, sc, False, window=window)
    assert rel_err(dq.cpu(), rq) <= TOL_BF16_REL
    assert rel_err(dk.cpu(), rk) <= TOL_BF16_REL
    assert rel_err(dv.cpu(), rv) <= TOL_BF16_REL
    assert fa.last_device_status()[0] == 0


@pytest.mark.gpu
def test_window_with_grouped_heads_and_causal_flag():
    """causal=True with window (200, None) is the window (200, 0); K/V heads grouped 2:1."""
    need_gpu()
    sc = _scale(128)
    q, k, v, do = I.make_inputs(1, 512, 4, 128, seed=8, kv_heads=2)
    qd, kd, vd = (t.cuda().requires_grad_() for t in (q, k, v))
    dod = do.cuda()
    out = fa.attention(qd, kd, vd, causal=True, scale=sc, window=(200, None))
    out.backward(dod)
    torch.cuda.synchronize()
    ro, _ = oracle.forward(q, k, v, sc, False, window=(200, 0))
    rq, rk, rv = oracle.backward(q, k, v, do, sc, False, window=(200, 0))
    assert rel_err(out.detach().cpu(), ro) <= TOL_BF16_REL
    for g, r in ((qd.grad, rq), (kd.grad, rk), (vd.grad, rv)):
        assert rel_err(g.cpu(), r) <= TOL_BF16_REL


@pytest.mark.gpu
def test_open_window_equals_unmasked_and_causal_bitwise():
    """(-1, -1) and (-1, 0) run the same tiles and masks as the plain passes."""
    need_gpu()
    q, k, v, _ = I.make_inputs(1, 1000, 4, 128, seed=12, with_do=False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    for causal, window in ((False, (None, None)), (True, (None, 0))):
        o1, l1 = fa.fwd(qd, kd, vd, causal=causal)
        o2, l2 = fa.fwd(qd, kd, vd, window=window)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.gpu
def test_window_4096_at_n32768_sampled_rows():
    """The page's configuration: 4096-token window over 32768 tokens (rows sampled
    across the sequence, including the first window's growing rows)."""
    need_gpu()
    n, d, window = 32768, 128, (4095, 0)
    q, k, v, _ = I.make_inputs(1, n, 4, d, seed=21, with_do=False)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), window=window)
    torch.cuda.synchronize()
    o, lse = o.cpu(), lse.cpu()
    rows = np.unique(np.concatenate([np.arange(0, 130), np.arange(4090, 4230),
                                     np.random.default_rng(0).integers(0, n, 200), np.arange(n - 130, n)]))
    for h in (0, 3):
        ro, rl = oracle.forward_rows_head(f64(q[0, :, h]), f64(k[0, :, h]), f64(v[0, :, h]), rows, _scale(d),
                                          False, window=window)
        assert rel_err(o[0, rows, h], ro) <= TOL_BF16_REL
        assert abs_err(lse[0, h, rows], rl) <= TOL_LSE


@pytest.mark.gpu
def test_window_backward_n8192_whole_head():
    need_gpu()
    n, window = 8192, (1023, 0)
    sc = _scale(128)
    q, k, v, do = I.make_inputs(1, n, 2, 128, seed=22)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, scale=sc, window=window)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, scale=sc, window=window)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.backward(q, k, v, do, sc, False, heads=[(0, 1)], window=window)
    assert rel_err(dq[0, :, 1].cpu(), rq[0, :, 1]) <= TOL_BF16_REL
    assert rel_err(dk[0, :, 1].cpu(), rk[0, :, 1]) <= TOL_BF16_REL
    assert rel_err(dv[0, :, 1].cpu(), rv[0, :, 1]) <= TOL_BF16_REL


def _time_ms(fn, reps=5):
    fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / reps


@pytest.mark.gpu
def test_window_skips_blocks_outside_it():
    """Blocks outside the window are not computed: with the page's 4096-token
    window at N = 32768 (12 % of the block grid visible) the forward takes well
    under a quarter of the unmasked forward's time."""
    need_gpu()
    q, k, v, _ = I.make_inputs(1, 32768, 16, 128, seed=23, with_do=False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    full = _time_ms(lambda: fa.fwd(qd, kd, vd))
    win = _time_ms(lambda: fa.fwd(qd, kd, vd, window=(4095, 0)))
    assert win < 0.25 * full, (win, full)
