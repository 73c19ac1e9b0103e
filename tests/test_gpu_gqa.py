"""Grouped-query attention parity: the CUDA path against the fp64 oracle.

"Flash Attention" (karlkratz.de), section "Grouped Query Attention": several
query heads share one K/V head (64 query heads on 8 K/V heads in the page's
example).  Query head h reads K/V head h // (H / Hkv).  The forward of each
query head is the ordinary forward with its group's K and V; the gradient of a
shared K/V head is the sum over its query heads, which the backward kernel
accumulates inside one CTA per (key tile, K/V head).
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


def _fwd(q, k, v, causal):
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=_scale(q.shape[-1]))
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


@pytest.mark.gpu
@pytest.mark.parametrize("H,Hkv", [(4, 1), (4, 2), (6, 3), (8, 8)])
@pytest.mark.parametrize("n,d", [(1, 64), (200, 64), (384, 128), (333, 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_forward_small(H, Hkv, n, d, causal):
    need_gpu()
    q, k, v, _ = I.make_inputs(2, n, H, d, seed=H * 100 + Hkv + n, with_do=False, kv_heads=Hkv)
    o, lse = _fwd(q, k, v, causal)
    ro, rl = oracle.forward(q, k, v, _scale(d), causal)
    assert rel_err(o, ro) <= TOL_BF16_REL
    assert abs_err(lse, rl) <= TOL_LSE


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_forward_fp32(causal):
    need_gpu()
    q, k, v, _ = I.make_inputs(1, 300, 6, 64, seed=9, dtype="fp32", with_do=False, kv_heads=2)
    o, lse = _fwd(q, k, v, causal)
    ro, rl = oracle.forward(q, k, v, _scale(64), causal)
    assert abs_err(o, ro) <= TOL_F32_O
    assert abs_err(lse, rl) <= TOL_LSE


@pytest.mark.gpu
@pytest.mark.parametrize("H,Hkv", [(4, 1), (4, 2), (6, 3)])
@pytest.mark.parametrize("n", [1, 128, 333, 640])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_backward_small(H, Hkv, n, causal):
    need_gpu()
    sc = _scale(128)
    q, k, v, do = I.make_inputs(2, n, H, 128, seed=7 * H + Hkv + n, kv_heads=Hkv)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=causal, scale=sc)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=sc)
    torch.cuda.synchronize()
    assert dk.shape == k.shape and dv.shape == v.shape
    rq, rk, rv = oracle.backward(q, k, v, do, sc, causal)
    assert rel_err(dq.cpu(), rq) <= TOL_BF16_REL
    assert rel_err(dk.cpu(), rk) <= TOL_BF16_REL
    assert rel_err(dv.cpu(), rv) <= TOL_BF16_REL
    assert fa.last_device_status()[0] == 0


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_h64_kv8_n4096_groups(causal):
    """The pages' head grouping at N = 4096: a whole K/V group (the first one
    without the mask, the last one with it) against the oracle."""
    need_gpu()
    w = I.BF16_GQA_H64_KV8
    sc = _scale(w.d)
    q, k, v, do = I.workload_inputs(w)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=causal, scale=sc)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=sc)
    torch.cuda.synchronize()
    o, dq, dk, dv = o.cpu(), dq.cpu(), dk.cpu(), dv.cpu()
    G = w.H // w.Hkv
    for g in ((w.Hkv - 1,) if causal else (0,)):
        heads = [(0, h) for h in range(g * G, (g + 1) * G)]
        ro, _ = oracle.forward(q, k, v, sc, causal, heads=heads)
        rq, rk, rv = oracle.backward(q, k, v, do, sc, causal, heads=heads)
        hs = slice(g * G, (g + 1) * G)
        assert rel_err(o[:, :, hs], ro[:, :, hs]) <= TOL_BF16_REL, ("o", g)
        assert rel_err(dq[:, :, hs], rq[:, :, hs]) <= TOL_BF16_REL, ("dq", g)
        assert rel_err(dk[:, :, g], rk[:, :, g]) <= TOL_BF16_REL, ("dk", g)
        assert rel_err(dv[:, :, g], rv[:, :, g]) <= TOL_BF16_REL, ("dv", g)


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_forward_equals_multi_head_on_repeated_kv(causal):
    """Each query head does the same arithmetic whether its K/V head is shared or
    copied, so the forward on repeated K/V heads is bitwise the same."""
    need_gpu()
    q, k, v, _ = I.make_inputs(1, 2048, 16, 128, seed=31, with_do=False, kv_heads=4)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = fa.fwd(qd, kd, vd, causal=causal)
    o2, l2 = fa.fwd(qd, kd.repeat_interleave(4, dim=2).contiguous(), vd.repeat_interleave(4, dim=2).contiguous(),
                    causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)


@pytest.mark.gpu
def test_gqa_backward_sums_match_multi_head_gradients():
    """dK, dV of a shared head equal the group sums of the multi-head gradients on
    repeated K/V (up to fp32 summation order and one bf16 rounding)."""
    need_gpu()
    q, k, v, do = I.make_inputs(1, 1024, 8, 128, seed=32, kv_heads=2)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse)
    kr, vr = (t.repeat_interleave(4, dim=2).contiguous() for t in (kd, vd))
    o2, lse2 = fa.fwd(qd, kr, vr)
    dq2, dk2, dv2 = fa.bwd(qd, kr, vr, o2, dod, lse2)
    torch.cuda.synchronize()
    assert rel_err(dq.cpu(), dq2.cpu()) <= 1e-2
    dk_sum = dk2.float().view(1, 1024, 2, 4, 128).sum(3)
    dv_sum = dv2.float().view(1, 1024, 2, 4, 128).sum(3)
    assert rel_err(dk.cpu(), dk_sum.cpu()) <= 1e-2
    assert rel_err(dv.cpu(), dv_sum.cpu()) <= 1e-2


@pytest.mark.gpu
def test_gqa_autograd():
    need_gpu()
    q, k, v, do = I.make_inputs(1, 256, 4, 128, seed=33, kv_heads=1)
    qd, kd, vd = (t.cuda().requires_grad_() for t in (q, k, v))
    out = fa.attention(qd, kd, vd, causal=True)
    out.backward(do.cuda())
    sc = _scale(128)
    rq, rk, rv = oracle.backward(q, k, v, do, sc, True)
    assert kd.grad.shape == k.shape
    for g, r in ((qd.grad, rq), (kd.grad, rk), (vd.grad, rv)):
        assert rel_err(g.cpu(), r) <= TOL_BF16_REL
    assert np.isfinite(f64(out)).all()
