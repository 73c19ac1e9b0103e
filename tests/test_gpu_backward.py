"""Backward parity: dQ, dK, dV from the CUDA path against the fp64 oracle.

The oracle recomputes P from Q, K, V and forms dV = P^T dO, dS = P (dP - D),
dQ = scale dS K, dK = scale dS^T Q in float64 on the same bf16 inputs.  A key
row of dK/dV needs every query, so large problems are checked on whole heads
chosen across the batch and head range.  Tolerance: max|d| / max|ref| <= 2e-2.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import exact_io_aware_51_b200 as fa
import oracle
from exact_io_aware_51_b200 import inputs as I
from tests.helpers import TOL_BF16_REL, f64, need_gpu, rel_err


def _scale(d):
    return float(np.float32(1.0 / math.sqrt(d)))


def _run(q, k, v, do, causal):
    sc = _scale(q.shape[-1])
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=causal, scale=sc)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=sc)
    torch.cuda.synchronize()
    return dq.cpu(), dk.cpu(), dv.cpu()


def _check_heads(q, k, v, do, causal, heads):
    sc = _scale(q.shape[-1])
    dq, dk, dv = _run(q, k, v, do, causal)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    for (b, h) in heads:
        rq, rk, rv, _ = oracle.backward_head(*(f64(t[b, :, h]) for t in (q, k, v, do)), sc, causal)
        assert rel_err(dq[b, :, h], rq) <= TOL_BF16_REL, ("dq", b, h)
        assert rel_err(dk[b, :, h], rk) <= TOL_BF16_REL, ("dk", b, h)
        assert rel_err(dv[b, :, h], rv) <= TOL_BF16_REL, ("dv", b, h)


def _all(B, H):
    return [(b, h) for b in range(B) for h in range(H)]


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 64, 128, 200, 384, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_small(n, causal):
    need_gpu()
    q, k, v, do = I.make_inputs(2, n, 3, 128, seed=n + 17)
    _check_heads(q, k, v, do, causal, _all(2, 3))


@pytest.mark.gpu
def test_bwd_b2_h16_n4096_d128_causal():
    need_gpu()
    q, k, v, do = I.workload_inputs(I.BF16_FWDBWD_N4K)
    _check_heads(q, k, v, do, True, [(0, 0), (1, 15), (0, 9), (1, 4)])


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_b1_h32_n16384_d128_kspike(causal):
    need_gpu()
    q, k, v, do = I.workload_inputs(I.BF16_FWDBWD_N16K)
    _check_heads(q, k, v, do, causal, [(0, 0), (0, 31)])


@pytest.mark.gpu
def test_bwd_scores_growing_along_keys():
    """A key component that grows along the sequence makes the row maxima large
    and uneven (the LSE spans tens of units); K keeps a random part comparable to
    the ramp so dQ = dS K is not a cancellation of a large common K offset (bf16
    dS could not resolve that)."""
    need_gpu()
    B, N, H, d = 1, 768, 2, 128
    g = torch.Generator().manual_seed(4)
    u = torch.randn(d, generator=g)
    u = u / u.norm()
    ramp = torch.linspace(0.0, 12.0, N).view(1, N, 1, 1)
    q = (torch.randn(B, N, H, d, generator=g) + 2.0 * u).to(torch.bfloat16)
    k = (torch.randn(B, N, H, d, generator=g) + ramp * u).to(torch.bfloat16)
    v = torch.randn(B, N, H, d, generator=g).to(torch.bfloat16)
    do = torch.randn(B, N, H, d, generator=g).to(torch.bfloat16)
    for causal in (False, True):
        _check_heads(q, k, v, do, causal, _all(B, H))


@pytest.mark.gpu
def test_autograd_function_matches_oracle():
    need_gpu()
    q, k, v, do = I.make_inputs(1, 300, 2, 128, seed=21)
    qd, kd, vd = (t.cuda().requires_grad_(True) for t in (q, k, v))
    o = fa.attention(qd, kd, vd, causal=True)
    o.backward(do.cuda())
    torch.cuda.synchronize()
    sc = _scale(128)
    for h in range(2):
        rq, rk, rv, _ = oracle.backward_head(*(f64(t[0, :, h]) for t in (q, k, v, do)), sc, True)
        assert rel_err(qd.grad[0, :, h].cpu(), rq) <= TOL_BF16_REL
        assert rel_err(kd.grad[0, :, h].cpu(), rk) <= TOL_BF16_REL
        assert rel_err(vd.grad[0, :, h].cpu(), rv) <= TOL_BF16_REL


@pytest.mark.gpu
def test_bwd_refuses_what_it_does_not_implement():
    """The fp32 backward is not implemented: refused, nothing computed."""
    need_gpu()
    q = torch.zeros(1, 128, 1, 64, dtype=torch.float32, device="cuda")
    lse = torch.zeros(1, 1, 128, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.bwd(q, q, q, q, q, lse)
    assert e.value.status == -2
