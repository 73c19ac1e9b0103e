"""Forward parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small problems are compared element by element over every (b, h); large ones
on every row of a few heads, or on sampled query rows (a row of O and its LSE
depend only on that query, so the oracle computes them one by one).
Tolerances: fp32 inputs max|dO| <= 1e-5 absolute; bf16 inputs
max|dO| / max|O| <= 2e-2; LSE within 1e-3 (natural log) in both cases.
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


def _run(q, k, v, causal, scale):
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _check_all_heads(q, k, v, causal, fp32=False):
    d = q.shape[-1]
    sc = _scale(d)
    o, lse = _run(q, k, v, causal, sc)
    o_ref, l_ref = oracle.forward(q, k, v, sc, causal)
    assert np.isfinite(f64(o)).all() and np.isfinite(f64(lse)).all()
    if fp32:
        assert abs_err(o, o_ref) <= TOL_F32_O
    else:
        assert rel_err(o, o_ref) <= TOL_BF16_REL
    assert abs_err(lse, l_ref) <= TOL_LSE
    return o, lse


def _check_sampled(q, k, v, causal, heads, nrows=256, seed=0):
    d = q.shape[-1]
    N = q.shape[1]
    sc = _scale(d)
    o, lse = _run(q, k, v, causal, sc)
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([rng.choice(N, size=min(nrows, N), replace=False), [0, N - 1]]))
    for (b, h) in heads:
        qh, kh, vh = (f64(t[b, :, h]) for t in (q, k, v))
        o_ref, l_ref = oracle.forward_rows_head(qh, kh, vh, rows, sc, causal)
        got = f64(o[b, rows, h])
        assert np.isfinite(got).all()
        assert rel_err(got, o_ref) <= TOL_BF16_REL, (b, h)
        assert abs_err(lse[b, h, rows], l_ref) <= TOL_LSE, (b, h)


# ----------------------------------------------------------------------------
# fp32 path
# ----------------------------------------------------------------------------

@pytest.mark.gpu
def test_fp32_b1_h1_n256_d64():
    need_gpu()
    q, k, v, _ = I.workload_inputs(I.FP32_SMALL)
    _check_all_heads(q, k, v, False, fp32=True)


@pytest.mark.gpu
@pytest.mark.parametrize("n,d,causal", [(256, 64, True), (200, 64, False), (333, 128, True), (1, 64, False),
                                        (130, 128, False)])
def test_fp32_other_shapes(n, d, causal):
    need_gpu()
    q, k, v, _ = I.make_inputs(2, n, 3, d, seed=n + d, dtype="fp32", with_do=False)
    _check_all_heads(q, k, v, causal, fp32=True)


# ----------------------------------------------------------------------------
# bf16 tensor-core path: small shapes, every element
# ----------------------------------------------------------------------------

SMALL = [(n, d, c) for n in (1, 64, 128, 129, 200, 256, 384, 1000) for d in (64, 128) for c in (False, True)]


@pytest.mark.gpu
@pytest.mark.parametrize("n,d,causal", SMALL)
def test_bf16_small(n, d, causal):
    need_gpu()
    q, k, v, _ = I.make_inputs(2, n, 3, d, seed=7 * n + d, with_do=False)
    _check_all_heads(q, k, v, causal)


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_bf16_b4_h16_n1024_d64(causal):
    need_gpu()
    q, k, v, _ = I.workload_inputs(I.BF16_FWD_N1K, with_do=False)
    _check_all_heads(q, k, v, causal)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("top", [24.0, 48.0])
def test_bf16_growing_row_maximum(d, causal, top):
    """Scores grow along the keys so the running maximum moves by many times the
    lazy-rescale threshold over a row: with top = 24 by about 8.6 (d = 64) to 12
    (d = 128) log2 units per key tile, so the kept maximum trails and moves every
    tile or two; with top = 48 by 17 to 24 per tile, so it moves on every tile.
    The oracle handles both exactly."""
    need_gpu()
    B, N, H = 1, 1024, 2
    q = torch.full((B, N, H, d), 0.25)
    ramp = torch.linspace(0.0, top, N).view(1, N, 1, 1)
    g = torch.Generator().manual_seed(3)
    k = (ramp + 0.05 * torch.randn(B, N, H, d, generator=g)).to(torch.bfloat16)
    v = torch.randn(B, N, H, d, generator=g).to(torch.bfloat16)
    _check_all_heads(q.to(torch.bfloat16), k, v, causal)


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_bf16_large_magnitude_scores(causal):
    """Inputs scaled by 8: many probabilities underflow to zero, none may be NaN."""
    need_gpu()
    q, k, v, _ = I.make_inputs(1, 512, 4, 128, seed=11, with_do=False)
    q = (q.float() * 8).to(torch.bfloat16)
    k = (k.float() * 8).to(torch.bfloat16)
    _check_all_heads(q, k, v, causal)


@pytest.mark.gpu
def test_bf16_permuting_keys_and_values_leaves_output_unchanged():
    """Non-causal attention is invariant to a joint permutation of K and V rows
    (up to the accumulation order): a property that holds at any size."""
    need_gpu()
    q, k, v, _ = I.make_inputs(1, 2048, 2, 128, seed=5, with_do=False)
    perm = torch.randperm(2048, generator=torch.Generator().manual_seed(9))
    o1, l1 = _run(q, k, v, False, _scale(128))
    o2, l2 = _run(q, k[:, perm].contiguous(), v[:, perm].contiguous(), False, _scale(128))
    assert rel_err(o2, o1) <= TOL_BF16_REL
    assert abs_err(l2, l1) <= TOL_LSE


@pytest.mark.gpu
def test_bf16_forward_is_deterministic():
    need_gpu()
    q, k, v, _ = I.make_inputs(2, 1000, 4, 128, seed=1, with_do=False)
    for causal in (False, True):
        o1, l1 = _run(q, k, v, causal, _scale(128))
        o2, l2 = _run(q, k, v, causal, _scale(128))
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.gpu
def test_empty_problems_are_no_ops():
    need_gpu()
    for shape in ((0, 128, 2, 64), (2, 0, 2, 64), (2, 128, 0, 128)):
        q = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        o, lse = fa.fwd(q, q, q)
        torch.cuda.synchronize()
        assert o.shape == shape and lse.shape == (shape[0], shape[2], shape[1])


# ----------------------------------------------------------------------------
# bf16: the full-size workloads (sampled rows / heads)
# ----------------------------------------------------------------------------

@pytest.mark.gpu
@pytest.mark.parametrize("w", I.SWEEP, ids=lambda w: w.name)
@pytest.mark.parametrize("causal", [False, True])
def test_bf16_sweep_sampled_rows(w, causal):
    need_gpu()
    q, k, v, _ = I.workload_inputs(w, with_do=False)
    heads = [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 3)]
    _check_sampled(q, k, v, causal, heads)


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_bf16_n16k_kspike_forward_sampled_rows(causal):
    need_gpu()
    q, k, v, _ = I.workload_inputs(I.BF16_FWDBWD_N16K, with_do=False)
    _check_sampled(q, k, v, causal, [(0, 0), (0, 13), (0, 31)], nrows=512)


# The bf16 forward takes one query tile per CTA (two CTAs per SM) when a query row
# sees at most 768 keys on average, two tiles per CTA otherwise.  Each case sits on
# one side of that rule: non-causal N = 768 / 769, causal N = 1535 / 1536, and a
# window of 767 keys on a longer sequence (one tile) against 769 (two).
@pytest.mark.gpu
@pytest.mark.parametrize("n,causal,window", [(768, False, None), (769, False, None), (1535, True, None),
                                             (1536, True, None), (2000, False, (700, 66)),
                                             (2000, False, (700, 68))],
                         ids=["n768", "n769", "causal1535", "causal1536", "window767", "window769"])
@pytest.mark.parametrize("d", [64, 128])
def test_bf16_one_and_two_tiles_per_cta(n, causal, window, d):
    need_gpu()
    q, k, v, _ = I.make_inputs(1, n, 3, d, seed=n + d, with_do=False, kv_heads=1)
    sc = _scale(d)
    kw = {"window": window} if window else {"causal": causal}
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), scale=sc, **kw)
    torch.cuda.synchronize()
    assert fa.last_device_status()[0] == 0
    o_ref, l_ref = oracle.forward(q, k, v, sc, causal, **({"window": window} if window else {}))
    assert np.isfinite(f64(o)).all()
    assert rel_err(o.cpu(), o_ref) <= TOL_BF16_REL
    assert abs_err(lse.cpu(), l_ref) <= TOL_LSE
