"""FP8 forward parity: e4m3 Q, K, V against the fp64 oracle on the dequantised inputs.

"Flash Attention" (karlkratz.de), "Versionen" (FlashAttention-3 runs attention
with FP8 inputs).  The oracle computes exact attention of x = scale_x * code
for each input; the kernel differs from it only by rounding the probabilities
to e4m3 before P V (the row sums use the unrounded values) and by the bf16
output.  The bound checked element by element follows from that rounding:

    P_ij >= 2^-10: the scaled probability is a normal e4m3 number, relative
                   error <= 2^-4;
    P_ij <  2^-10: absolute error <= 2^-10 / l' <= 2^-14 in units of P, where
                   l' >= 2^4 is the kernel's scaled row sum;

so |dO_ik| <= 2^-4 sum_j P_ij |v_jk| + 2^-14 sum_{j: P_ij < 2^-10} |v_jk|
            + 2^-8 |O_ik| (bf16 output) + 1e-5 (fp32 arithmetic).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import exact_io_aware_51_b200 as fa
import oracle
from exact_io_aware_51_b200 import inputs as I
from tests.helpers import TOL_LSE, abs_err, f64, need_gpu

E4M3_MAX = 448.0


def _quantise(x: torch.Tensor):
    """Per-tensor e4m3 codes and scale (input preparation for the tests, not part of the method)."""
    amax = float(x.float().abs().max())
    s = amax / E4M3_MAX if amax > 0 else 1.0
    codes = (x.float() / s).to(torch.float8_e4m3fn)
    return codes, s


def _fp8_inputs(B, N, H, Hkv, seed, spike_frac=0.0):
    q, k, v, _ = I.make_inputs(B, N, H, 128, seed=seed, dtype="fp32", with_do=False, kv_heads=Hkv,
                               spike_frac=spike_frac)
    (cq, sq), (ck, sk), (cv, sv) = (_quantise(t) for t in (q, k, v))
    deq = [c.double() * s for c, s in ((cq, sq), (ck, sk), (cv, sv))]
    return (cq, ck, cv), (sq, sk, sv), deq


def _bound(qd, kd, vd, scale, causal, window, rows=None, block_mask=None):
    """Per-element error bound of the e4m3 probabilities (see the module docstring), one head."""
    if rows is None:
        rows = np.arange(qd.shape[0])
    s = oracle.scores_head(qd[rows], kd, scale, False)
    hidden = oracle.hidden_keys(rows, kd.shape[0], causal, window, block_mask)
    s = np.where(hidden, -np.inf, s)
    p, _ = oracle.probs_head(s)
    av = np.abs(vd)
    o = p @ vd
    small = (p < 2.0 ** -10) & ~hidden
    return 2.0 ** -4 * (p @ av) + 2.0 ** -14 * (small @ av) + 2.0 ** -8 * np.abs(o) + 1e-5


def _check(B, N, H, Hkv, causal=False, window=None, seed=0, heads=None, rows=None, spike_frac=0.0):
    (cq, ck, cv), (sq, sk, sv), (dq, dk, dv) = _fp8_inputs(B, N, H, Hkv, seed, spike_frac)
    scale = float(np.float32(1.0 / math.sqrt(128)))
    o, lse = fa.fwd_fp8(cq.cuda(), ck.cuda(), cv.cuda(), sq, sk, sv, causal=causal, scale=scale, window=window)
    torch.cuda.synchronize()
    assert fa.last_device_status()[0] == 0
    o, lse = f64(o), f64(lse)
    assert np.isfinite(o).all()
    G = H // Hkv
    worst = 0.0
    for (b, h) in (heads or [(b, h) for b in range(B) for h in range(H)]):
        g = h // G
        qh, kh, vh = dq[b, :, h].numpy(), dk[b, :, g].numpy(), dv[b, :, g].numpy()
        r = np.arange(N) if rows is None else rows
        win = window if not causal else ((None, 0) if window is None else (window[0], 0))
        ro, rl = oracle.forward_rows_head(qh, kh, vh, r, scale, False, window=win)
        bound = _bound(qh, kh, vh, scale, False, win, rows=r)
        err = np.abs(o[b, r, h] - ro)
        assert (err <= bound).all(), (b, h, float(np.max(err - bound)))
        assert abs_err(lse[b, h, r], rl) <= TOL_LSE
        worst = max(worst, float(np.max(err) / max(np.max(np.abs(ro)), 1e-30)))
    return worst


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 128, 200, 384, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_small(n, causal):
    need_gpu()
    _check(2, n, 3, 3, causal=causal, seed=n)


@pytest.mark.gpu
@pytest.mark.parametrize("window", [(0, 0), (127, 0), (300, 64)], ids=str)
def test_fp8_window_and_gqa(window):
    need_gpu()
    _check(1, 700, 4, 2, window=window, seed=5)


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_b1_h32_n16384_sampled_rows(causal):
    """The long-sequence workload with the K-row spike, 2 heads x 256 sampled rows."""
    need_gpu()
    rows = np.sort(np.random.default_rng(3).choice(16384, 256, replace=False))
    _check(1, 16384, 32, 32, causal=causal, seed=0, heads=[(0, 0), (0, 31)], rows=rows, spike_frac=0.01)


@pytest.mark.gpu
def test_fp8_refuses_other_head_dims():
    need_gpu()
    x = torch.zeros(1, 128, 1, 64, dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(fa.FAError):
        fa.fwd_fp8(x, x, x, 1.0, 1.0, 1.0)


@pytest.mark.gpu
@pytest.mark.parametrize("n,H,Hkv,heads_mask", [(384, 2, 2, 1), (700, 4, 2, 4), (1000, 2, 1, 1)])
def test_fp8_blocksparse(n, H, Hkv, heads_mask):
    """The 8-bit forward under a 0/1 mask over 128 x 128 blocks (one shared or one
    per query head, with an empty block row): every element within the e4m3
    bound of the oracle on the dequantised inputs; empty rows O = 0, LSE = -inf."""
    need_gpu()
    nb = (n + 127) // 128
    m = (np.random.default_rng(n + H).random((heads_mask, nb, nb)) < 0.5).astype(np.uint8)
    m[:, nb // 2, :] = 0
    mask = m[0] if heads_mask == 1 else m
    (cq, ck, cv), (sq, sk, sv), (dq, dk, dv) = _fp8_inputs(1, n, H, Hkv, seed=n)
    scale = float(np.float32(1.0 / math.sqrt(128)))
    o, lse = fa.fwd_fp8(cq.cuda(), ck.cuda(), cv.cuda(), sq, sk, sv, scale=scale,
                        block_mask=torch.from_numpy(mask).cuda())
    torch.cuda.synchronize()
    assert fa.last_device_status()[0] == 0
    o, lse = f64(o), f64(lse)
    G = H // Hkv
    for h in range(H):
        mh = mask if heads_mask == 1 else mask[h]
        qh, kh, vh = dq[0, :, h].numpy(), dk[0, :, h // G].numpy(), dv[0, :, h // G].numpy()
        rows = np.arange(n)
        ro, rl = oracle.forward_rows_head(qh, kh, vh, rows, scale, False, block_mask=mh)
        bound = _bound(qh, kh, vh, scale, False, None, rows=rows, block_mask=mh)
        assert (np.abs(o[0, :, h] - ro) <= bound).all(), h
        both_inf = np.isneginf(lse[0, h]) & np.isneginf(rl)
        with np.errstate(invalid="ignore"):
            assert np.all(both_inf | (np.abs(lse[0, h] - rl) <= TOL_LSE)), h
