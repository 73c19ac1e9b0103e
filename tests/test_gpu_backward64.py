"""Backward parity at head dimension 64: dQ, dK, dV against the fp64 oracle.

The d = 64 backward kernel has its own layout (dQ in TMEM columns of its own,
computed non-transposed and staged through a swizzled tile); these tests give
it the edge cases and masks the d = 128 kernel gets.  Tolerance as for every
bf16 result: max|d| / max|ref| <= 2e-2.
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

D = 64


def _scale():
    return float(np.float32(1.0 / math.sqrt(D)))


def _run(q, k, v, do, **kw):
    sc = _scale()
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, scale=sc, **kw)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, scale=sc, **kw)
    torch.cuda.synchronize()
    assert fa.last_device_status()[0] == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


def _check(got, ref):
    for g, r, name in zip(got, ref, ("dq", "dk", "dv")):
        assert torch.isfinite(g.float()).all(), name
        assert rel_err(g, r) <= TOL_BF16_REL, name


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 64, 128, 200, 384, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd64_small(n, causal):
    need_gpu()
    q, k, v, do = I.make_inputs(2, n, 3, D, seed=n + 64)
    got = _run(q, k, v, do, causal=causal)
    _check(got, oracle.backward(q, k, v, do, _scale(), causal))


@pytest.mark.gpu
def test_bwd64_b4_h16_n1024_causal_heads():
    need_gpu()
    q, k, v, do = I.make_inputs(4, 1024, 16, D, seed=5)
    dq, dk, dv = _run(q, k, v, do, causal=True)
    heads = [(0, 0), (1, 7), (3, 15)]
    rq, rk, rv = oracle.backward(q, k, v, do, _scale(), True, heads=heads)
    for (b, h) in heads:
        assert rel_err(dq[b, :, h], rq[b, :, h]) <= TOL_BF16_REL
        assert rel_err(dk[b, :, h], rk[b, :, h]) <= TOL_BF16_REL
        assert rel_err(dv[b, :, h], rv[b, :, h]) <= TOL_BF16_REL


@pytest.mark.gpu
@pytest.mark.parametrize("window", [(100, 0), (129, 17)], ids=str)
def test_bwd64_window_and_gqa(window):
    need_gpu()
    q, k, v, do = I.make_inputs(1, 640, 4, D, seed=11, kv_heads=2)
    got = _run(q, k, v, do, window=window)
    _check(got, oracle.backward(q, k, v, do, _scale(), False, window=window))


@pytest.mark.gpu
def test_bwd64_blocksparse():
    need_gpu()
    n = 512
    m = (np.random.default_rng(2).random((4, 4)) < 0.6).astype(np.uint8)
    m[np.arange(4), np.arange(4)] = 1
    q, k, v, do = I.make_inputs(1, n, 2, D, seed=12)
    got = _run(q, k, v, do, block_mask=torch.from_numpy(m).cuda())
    _check(got, oracle.backward(q, k, v, do, _scale(), False, block_mask=m))


@pytest.mark.gpu
def test_bwd64_b1_h32_n16384_heads():
    """The bench sweep's d = 64 workload at full size: the whole problem on the GPU,
    two whole heads (first and last) against the oracle."""
    need_gpu()
    q, k, v, do = I.workload_inputs(I.BF16_FWDBWD_N16K_D64)
    dq, dk, dv = _run(q, k, v, do, causal=False)
    sc = _scale()
    f64 = lambda t: t.float().numpy().astype(np.float64)
    for h in (0, 31):
        rq, rk, rv, _ = oracle.backward_head(*(f64(t[0, :, h]) for t in (q, k, v, do)), sc, False)
        for g, r, name in ((dq[0, :, h], rq, "dq"), (dk[0, :, h], rk, "dk"), (dv[0, :, h], rv, "dv")):
            assert torch.isfinite(g.float()).all(), (h, name)
            assert rel_err(g, r) <= TOL_BF16_REL, (h, name)
