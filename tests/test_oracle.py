"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these re-type the oracle's formulas; each compares it with something
independent of it: closed-form outputs, invariants, the pages' worked example,
central finite differences, or a library routine on a special case.  The
mutation tests at the end plant plausible mistakes in copies of the oracle and
check that at least one pin catches each.
"""

from __future__ import annotations

import json
import math
import pathlib

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A

GOLDEN = pathlib.Path(__file__).parent / "golden"


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------------------
# Pin functions.  Each takes the two oracle entry points it exercises so that
# the mutation tests can run the same checks against planted mistakes.
# ---------------------------------------------------------------------------

def pin_rows_sum_to_one(probs_fn=A.probs_head, scores_fn=A.scores_head):
    """P >= 0 and each row of P sums to 1 (definition of the row softmax)."""
    worst = 0.0
    for causal in (False, True):
        q, k = _rand((37, 8), 1), _rand((37, 8), 2)
        p, _ = probs_fn(scores_fn(q, k, 0.35, causal))
        if np.any(p < 0):
            return math.inf
        worst = max(worst, float(np.max(np.abs(p.sum(axis=1) - 1.0))))
        if causal:
            # hidden keys (j > i) carry exactly zero weight
            worst = max(worst, float(np.max(np.abs(np.triu(p, 1)))))
    return worst


def pin_constant_scores(fwd=A.forward_head):
    """Q = 0 gives equal scores: O_i = mean of the visible V_j, LSE_i = ln(#visible)."""
    n, d = 23, 5
    v = _rand((n, d), 3)
    k = _rand((n, d), 4)
    q = np.zeros((n, d))
    worst = 0.0
    o, lse = fwd(q, k, v, 0.7, False)
    worst = max(worst, np.max(np.abs(o - v.mean(axis=0))), np.max(np.abs(lse - math.log(n))))
    o, lse = fwd(q, k, v, 0.7, True)
    counts = np.arange(1, n + 1)
    want = np.cumsum(v, axis=0) / counts[:, None]
    worst = max(worst, np.max(np.abs(o - want)), np.max(np.abs(lse - np.log(counts))))
    # all key rows equal: the score of row i is the constant c_i = scale*<q_i, k>
    q = _rand((n, d), 5)
    krow = _rand((1, d), 6)
    kk = np.repeat(krow, n, axis=0)
    o, lse = fwd(q, kk, v, 0.3, False)
    c = 0.3 * (q @ krow[0])
    worst = max(worst, np.max(np.abs(o - v.mean(axis=0))), np.max(np.abs(lse - (c + math.log(n)))))
    return float(worst)


def pin_dominant_key(fwd=A.forward_head):
    """One key scores t, all others 0: O_i = (e^t v_* + sum_{others} v_j) / (e^t + #others)."""
    n = d = 12
    t = 9.0
    k = np.eye(n, d)                      # orthonormal keys
    v = _rand((n, d), 7)
    star = (np.arange(n) * 5 + 3) % n     # a different target key per query
    q = t * k[star]                       # <q_i, k_j> = t if j == star_i else 0
    worst = 0.0
    o, lse = fwd(q, k, v, 1.0, False)
    for i in range(n):
        num = math.exp(t) * v[star[i]] + (v.sum(axis=0) - v[star[i]])
        den = math.exp(t) + (n - 1)
        worst = max(worst, np.max(np.abs(o[i] - num / den)), abs(lse[i] - math.log(den)))
    # causal: only keys j <= i are visible
    star_c = np.array([(i * 7) % (i + 1) for i in range(n)])
    q = t * k[star_c]
    o, lse = fwd(q, k, v, 1.0, True)
    for i in range(n):
        vis = v[: i + 1]
        num = math.exp(t) * v[star_c[i]] + (vis.sum(axis=0) - v[star_c[i]])
        den = math.exp(t) + i
        worst = max(worst, np.max(np.abs(o[i] - num / den)), abs(lse[i] - math.log(den)))
    return float(worst)


def pin_permutation(fwd=A.forward_head):
    """Non-causal attention does not depend on the order of the (k_j, v_j) pairs."""
    q, k, v = _rand((19, 6), 8), _rand((31, 6), 9), _rand((31, 4), 10)
    perm = np.random.default_rng(11).permutation(31)
    o1, l1 = fwd(q, k, v, 0.4, False)
    o2, l2 = fwd(q, k[perm], v[perm], 0.4, False)
    return float(max(np.max(np.abs(o1 - o2)), np.max(np.abs(l1 - l2))))


def pin_blocked_equals_full(fwd=A.forward_head, blocked=A.blocked_forward_head):
    """The pages' online-softmax recurrence equals the full softmax (exact in fp64)."""
    worst = 0.0
    n, d = 70, 8
    q, k, v = _rand((n, d), 12), 3 * _rand((n, d), 13), _rand((n, d), 14)
    for causal in (False, True):
        o, lse = fwd(q, k, v, 0.5, causal)
        for block in (1, 7, 16, 32, 256):
            for tau in (0.0, 2.0, math.log(256.0)):
                ob, lb = blocked(q, k, v, 0.5, causal, block, tau)
                worst = max(worst, np.max(np.abs(ob - o)), np.max(np.abs(lb - lse)))
    return float(worst)


def pin_finite_differences(fwd=A.forward_head, bwd=A.backward_head, causal=False):
    """Central differences of L = sum(dO * O) against (dQ, dK, dV)."""
    n, d = 6, 3
    q, k, v, do = (_rand((n, d), s) for s in (20, 21, 22, 23))
    scale = 0.8
    dq, dk, dv, _ = bwd(q, k, v, do, scale, causal)
    h = 1e-6
    worst = 0.0
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for idx in np.ndindex(n, d):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            lp = float(np.sum(do * fwd(*args, scale, causal)[0]))
            args[which][idx] -= 2 * h
            lm = float(np.sum(do * fwd(*args, scale, causal)[0]))
            fd = (lp - lm) / (2 * h)
            worst = max(worst, abs(fd - grad[idx]) / (1.0 + abs(fd)))
    return float(worst)


def pin_d_identity(bwd=A.backward_head):
    """D_i = sum_k dO_ik O_ik equals sum_j P_ij dP_ij with dP = dO V^T."""
    n, d = 17, 4
    q, k, v, do = (_rand((n, d), s) for s in (30, 31, 32, 33))
    worst = 0.0
    for causal in (False, True):
        _, _, _, dvec = bwd(q, k, v, do, 0.6, causal)
        p, _ = A.probs_head(A.scores_head(q, k, 0.6, causal))
        other = np.sum(p * (do @ v.T), axis=1)
        worst = max(worst, float(np.max(np.abs(dvec - other))))
    return worst


def pin_autograd(bwd=A.backward_head, fwd=A.forward_head):
    """torch.autograd in float64 on CPU (a library routine) agrees with the oracle."""
    worst = 0.0
    for causal in (False, True):
        n, d = 21, 5
        q, k, v, do = (_rand((n, d), s) for s in (40, 41, 42, 43))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        mask = None
        if causal:
            mask = torch.ones(n, n, dtype=torch.bool).tril()
        out = torch.nn.functional.scaled_dot_product_attention(
            tq[None, None], tk[None, None], tv[None, None], attn_mask=mask, scale=0.45)[0, 0]
        out.backward(torch.tensor(do))
        o, _ = fwd(q, k, v, 0.45, causal)
        dq, dk, dv, _ = bwd(q, k, v, do, 0.45, causal)
        worst = max(worst, float(np.max(np.abs(o - out.detach().numpy()))))
        for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            worst = max(worst, float(np.max(np.abs(a - b.numpy()))))
    return worst


def _gqa_case(seed, B=2, N=19, H=6, Hkv=2, d=4):
    q = _rand((B, N, H, d), seed)
    k = _rand((B, N, Hkv, d), seed + 1)
    v = _rand((B, N, Hkv, d), seed + 2)
    do = _rand((B, N, H, d), seed + 3)
    return q, k, v, do


def pin_gqa_torch(fwd=A.forward, bwd=A.backward):
    """Grouped-query attention against torch's SDPA with enable_gqa (fp64, CPU, autograd).

    torch repeats each K/V head over H / Hkv consecutive query heads, the
    grouping read from "Flash Attention" (karlkratz.de), "Grouped Query Attention".
    """
    worst = 0.0
    for causal in (False, True):
        for H, Hkv in ((6, 2), (6, 1), (4, 4)):
            q, k, v, do = _gqa_case(60 + H + Hkv, H=H, Hkv=Hkv)
            tq, tk, tv = (torch.tensor(x.transpose(0, 2, 1, 3), requires_grad=True) for x in (q, k, v))
            out = torch.nn.functional.scaled_dot_product_attention(
                tq, tk, tv, is_causal=causal, scale=0.6, enable_gqa=True)
            out.backward(torch.tensor(do.transpose(0, 2, 1, 3)))
            o, _ = fwd(q, k, v, 0.6, causal)
            dq, dk, dv = bwd(q, k, v, do, 0.6, causal)
            pairs = ((o, out.detach()), (dq, tq.grad), (dk, tk.grad), (dv, tv.grad))
            for a, b in pairs:
                worst = max(worst, float(np.max(np.abs(a - b.numpy().transpose(0, 2, 1, 3)))))
    return worst


def pin_gqa_finite_differences(bwd=A.backward, causal=True):
    """dK, dV of a shared K/V head by central differences of L = sum(O * dO) over all query heads."""
    q, k, v, do = _gqa_case(70, B=1, N=9, H=6, Hkv=2, d=3)
    dq, dk, dv = bwd(q, k, v, do, 0.8, causal)

    def loss(kk, vv):
        o, _ = A.forward(q, kk, vv, 0.8, causal)
        return float(np.sum(o * do))

    eps = 1e-6
    worst = 0.0
    for (n, g, c) in ((0, 0, 0), (4, 1, 2), (8, 0, 1), (3, 1, 0)):
        for which, grad in (("k", dk), ("v", dv)):
            kp, km = k.copy(), k.copy()
            vp, vm = v.copy(), v.copy()
            if which == "k":
                kp[0, n, g, c] += eps
                km[0, n, g, c] -= eps
            else:
                vp[0, n, g, c] += eps
                vm[0, n, g, c] -= eps
            fd = (loss(kp, vp) - loss(km, vm)) / (2 * eps)
            worst = max(worst, abs(fd - grad[0, n, g, c]))
    return worst


WINDOWS = ((0, 0), (1, 0), (3, 2), (0, 4), (None, 0), (5, None), (None, None), (2, 40))


def pin_window_rowwise(fwd=A.forward_head):
    """Sliding window: each row is ordinary softmax attention over the slice of
    keys k[i-left : i+right+1] (the neighbourhood itself, no mask involved)."""
    n, d = 23, 4
    q, k, v = _rand((n, d), 90), _rand((n, d), 91), _rand((n, 3), 92)
    worst = 0.0
    for window in WINDOWS:
        o, lse = fwd(q, k, v, 0.7, False, window)
        left, right = window
        for i in range(n):
            lo = 0 if left is None else max(0, i - left)
            hi = n if right is None else min(n, i + right + 1)
            s = 0.7 * (k[lo:hi] @ q[i])
            e = np.exp(s - s.max())
            worst = max(worst, float(np.max(np.abs(o[i] - e @ v[lo:hi] / e.sum()))),
                        abs(lse[i] - (s.max() + math.log(e.sum()))))
    return worst


def pin_window_zero_width(fwd=A.forward_head):
    """Window (0, 0) leaves one key per row: O_i = v_i and LSE_i = scale <q_i, k_i>."""
    n, d = 11, 5
    q, k, v = _rand((n, d), 93), _rand((n, d), 94), _rand((n, d), 95)
    o, lse = fwd(q, k, v, 0.3, False, (0, 0))
    return float(max(np.max(np.abs(o - v)), np.max(np.abs(lse - 0.3 * np.sum(q * k, axis=1)))))


def pin_window_finite_differences(bwd=A.backward_head, window=(2, 1)):
    """Central differences of L = sum(dO * O) under a sliding window."""
    n, d = 7, 3
    q, k, v, do = (_rand((n, d), s) for s in (96, 97, 98, 99))
    dq, dk, dv, _ = bwd(q, k, v, do, 0.8, False, window)
    h = 1e-6
    worst = 0.0
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for idx in np.ndindex(n, d):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            lp = float(np.sum(do * A.forward_head(*args, 0.8, False, window)[0]))
            args[which][idx] -= 2 * h
            lm = float(np.sum(do * A.forward_head(*args, 0.8, False, window)[0]))
            worst = max(worst, abs((lp - lm) / (2 * h) - grad[idx]))
    return worst


def window_skipped_block_fraction(n, window, block, hidden=A.hidden_keys):
    """Fraction of the n x n grid of block x block tiles in which every key is hidden."""
    skipped = 0
    for r0 in range(0, n, block):
        h = hidden(np.arange(r0, min(n, r0 + block)), n, False, window)
        visible_cols = ~np.all(h, axis=0)
        per_tile = visible_cols.reshape(-1, block).any(axis=1)
        skipped += int(np.sum(~per_tile))
    nb = n // block
    return skipped / (nb * nb)


BLOCK_MASKS = (
    np.array([[1, 0, 1], [0, 1, 0], [1, 1, 1]]),
    np.array([[0, 0, 1], [1, 0, 0], [0, 1, 1]]),
    np.array([[1, 1, 1], [0, 0, 0], [1, 0, 1]]),   # middle row block sees nothing
)


def pin_blocksparse_rowwise(fwd=A.forward_head):
    """Block-sparse mask over 128 x 128 blocks: each row is ordinary softmax
    attention over the keys gathered from its visible blocks (no mask involved);
    a row with no visible block gets O = 0 and LSE = -inf."""
    n, d = 300, 4
    q, k, v = 0.3 * _rand((n, d), 110), 0.3 * _rand((n, d), 111), _rand((n, 3), 112)
    worst = 0.0
    for bm in BLOCK_MASKS:
        o, lse = fwd(q, k, v, 0.7, False, None, bm)
        for i in range(n):
            idx = np.concatenate([np.arange(128 * c, min(n, 128 * c + 128)) for c in range(3) if bm[i // 128, c]]
                                 + [np.zeros(0, dtype=int)]).astype(int)
            if idx.size == 0:
                if not (np.all(o[i] == 0) and lse[i] == -np.inf):
                    return math.inf
                continue
            s_ = 0.7 * (k[idx] @ q[i])
            e = np.exp(s_ - s_.max())
            worst = max(worst, float(np.max(np.abs(o[i] - e @ v[idx] / e.sum()))),
                        abs(lse[i] - (s_.max() + math.log(e.sum()))))
    return worst


def pin_blocksparse_finite_differences(bwd=A.backward_head):
    """Central differences of L = sum(dO * O) under a block mask, on sampled entries."""
    n, d = 300, 3
    q, k, v, do = (0.3 * _rand((n, d), s) for s in (113, 114, 115, 116))
    bm = BLOCK_MASKS[0]
    dq, dk, dv, _ = bwd(q, k, v, do, 0.8, True, None, bm)
    h = 1e-6
    worst = 0.0
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for idx in ((0, 0), (17, 2), (130, 1), (200, 0), (299, 2), (256, 1)):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            lp = float(np.sum(do * A.forward_head(*args, 0.8, True, None, bm)[0]))
            args[which][idx] -= 2 * h
            lm = float(np.sum(do * A.forward_head(*args, 0.8, True, None, bm)[0]))
            worst = max(worst, abs((lp - lm) / (2 * h) - grad[idx]))
    return worst


# ---------------------------------------------------------------------------
# The pins themselves
# ---------------------------------------------------------------------------

def test_rows_sum_to_one():
    assert pin_rows_sum_to_one() < 1e-14


def test_constant_scores_closed_form():
    assert pin_constant_scores() < 1e-12


def test_dominant_key_closed_form():
    assert pin_dominant_key() < 1e-12


def test_permutation_invariance():
    assert pin_permutation() < 1e-13


def test_blocked_online_softmax_equals_full():
    assert pin_blocked_equals_full() < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_backward_finite_differences(causal):
    assert pin_finite_differences(causal=causal) < 1e-7


def test_d_identity():
    assert pin_d_identity() < 1e-12


def test_autograd_cross_check():
    assert pin_autograd() < 1e-12


def test_rows_subset_matches_definition_on_those_rows():
    n, d = 40, 8
    q, k, v = _rand((n, d), 50), _rand((n, d), 51), _rand((n, d), 52)
    rows = [0, 5, 17, 39]
    for causal in (False, True):
        # the full-row closed form for query 0 under causal masking: only key 0
        o_r, l_r = A.forward_rows_head(q, k, v, rows, 0.3, causal)
        if causal:
            assert np.max(np.abs(o_r[0] - v[0])) < 1e-15
            assert abs(l_r[0] - 0.3 * float(q[0] @ k[0])) < 1e-14
        o, l = A.forward_head(q, k, v, 0.3, causal)
        assert np.max(np.abs(o_r - o[rows])) < 1e-13
        assert np.max(np.abs(l_r - l[rows])) < 1e-13


def test_batched_layout_maps_heads():
    """[B, N, H, d] inputs and [B, H, N] LSE: a zero-query head reduces to mean(V)."""
    B, N, H, d = 2, 9, 3, 4
    g = np.random.default_rng(60)
    Q, K, V = (g.standard_normal((B, N, H, d)) for _ in range(3))
    Q[1, :, 2] = 0.0
    O, LSE = oracle.forward(Q, K, V, 0.5, False)
    assert np.max(np.abs(O[1, :, 2] - V[1, :, 2].mean(axis=0))) < 1e-13
    assert np.max(np.abs(LSE[1, 2] - math.log(N))) < 1e-13
    # the other heads are untouched by head (1, 2)'s inputs
    Q2 = Q.copy()
    Q2[1, :, 2] = 5.0
    O2, _ = oracle.forward(Q2, K, V, 0.5, False)
    mask = np.ones((B, H), bool)
    mask[1, 2] = False
    for b in range(B):
        for h in range(H):
            if mask[b, h]:
                assert np.array_equal(O[b, :, h], O2[b, :, h])
    dQ, dK, dV = oracle.backward(Q, K, V, np.ones_like(Q), 0.5, False)
    # with dO = 1 and Q = 0 on head (1,2): dV_j = sum_i P_ij = N * (1/N) = 1
    assert np.max(np.abs(dV[1, :, 2] - 1.0)) < 1e-13


def test_fully_masked_row_is_zero_with_minus_inf_lse():
    s = np.array([[-np.inf, -np.inf], [0.0, -np.inf]])
    p, lse = A.probs_head(s)
    assert np.all(p[0] == 0) and lse[0] == -np.inf
    assert p[1, 0] == 1.0 and lse[1] == 0.0


def test_pages_demo_fp32_error_magnitude():
    """The pages' fp32 demonstration: blocked vs full differ by ~4.3e-07."""
    g = json.loads((GOLDEN / "online_softmax_demo.json").read_text())
    n, d, block = g["n"], g["d"], g["block"]
    torch.manual_seed(g["seed"])
    q, k, v = (t.numpy() for t in torch.randn(3, n, d).unbind(0))
    scale = 1.0 / math.sqrt(d)
    ob, _ = A.blocked_forward_head(q, k, v, np.float32(scale), False, block, 0.0, dtype=np.float32)
    assert ob.dtype == np.float32
    # full fp32 standard attention through torch's own softmax (library routine)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    full = (torch.softmax(tq @ tk.T / math.sqrt(d), dim=-1) @ tv).numpy()
    diff = float(np.max(np.abs(ob - full)))
    printed = g["printed_max_abs_diff"]
    assert printed / 10 <= diff <= printed * 10, diff
    # in fp64 the same recurrence is exact to rounding of fp64
    o64, _ = A.forward_head(q, k, v, scale, False)
    ob64, _ = A.blocked_forward_head(q, k, v, scale, False, block, 0.0)
    assert float(np.max(np.abs(ob64 - o64))) < 1e-12
    # and both fp32 results sit within fp32 rounding of the fp64 truth
    assert float(np.max(np.abs(full - o64))) < 10 * printed


def test_memory_arithmetic_of_the_score_matrix():
    """The pages' sizes for the materialised score matrix that the kernel avoids."""
    g = json.loads((GOLDEN / "memory_arithmetic.json").read_text())
    c = {x["what"]: x for x in g["cases"]}
    assert 4096 ** 2 >= c["score entries at N=4096"]["entries_at_least"]
    e8k = 8192 ** 2
    assert abs(e8k - 67e6) / 67e6 < 0.01
    assert abs(e8k * 2 / 2 ** 20 - 128) < 1e-9
    assert e8k * 2 * 32 / 2 ** 30 >= 4
    assert 256 * 256 * 2 / 1024 == 128
    assert 16384 ** 2 * 2 / 2 ** 20 == 512
    # the oracle really materialises N x N per head
    s = A.scores_head(np.zeros((64, 4)), np.zeros((64, 4)), 1.0, False)
    assert s.shape == (64, 64)


# ---------------------------------------------------------------------------
# Mutation tests: plausible mistakes planted in copies of the oracle.
# ---------------------------------------------------------------------------

def _mut_fwd(kind):
    def fwd(q, k, v, scale, causal):
        q, k, v = (np.asarray(x, float) for x in (q, k, v))
        sc = scale
        if kind == "no_scale":
            sc = 1.0
        s = sc * (q @ k.T)
        if kind == "transposed_scores":
            s = s.T
        if causal:
            hidden = np.arange(k.shape[0])[None, :] > np.arange(q.shape[0])[:, None]
            if kind == "mask_direction":
                hidden = hidden.T
            if kind == "mask_diagonal":
                hidden = np.arange(k.shape[0])[None, :] >= np.arange(q.shape[0])[:, None]
            s = np.where(hidden, -np.inf, s)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        if kind == "sum_over_columns":
            l = e.sum(axis=0, keepdims=True).T
        p = e / l
        lse = m[:, 0] + np.log(l[:, 0])
        if kind == "lse_base2":
            lse = m[:, 0] + np.log2(l[:, 0])
        if kind == "lse_drops_max":
            lse = np.log(l[:, 0])
        out = p @ v
        if kind == "values_are_keys":
            out = p @ k[:, : v.shape[1]]
        return out, lse
    return fwd


def _mut_bwd(kind):
    def bwd(q, k, v, do, scale, causal):
        q, k, v, do = (np.asarray(x, float) for x in (q, k, v, do))
        p, _ = A.probs_head(A.scores_head(q, k, scale, causal))
        o = p @ v
        dv = p.T @ do
        if kind == "dv_untransposed":
            dv = p @ do
        dp = do @ v.T
        dvec = np.sum(do * o, axis=1)
        ds = p * (dp - dvec[:, None])
        if kind == "ds_sign":
            ds = p * (dp + dvec[:, None])
        if kind == "ds_drops_d":
            ds = p * dp
        dq = scale * (ds @ k)
        dk = scale * (ds.T @ q)
        if kind == "dk_no_scale":
            dk = ds.T @ q
        if kind == "dq_uses_v":
            dq = scale * (ds @ v)
        return dq, dk, dv, dvec
    return bwd


def _caught(pin, impl, tol=1e-9):
    """A pin catches a mutant when it reports a large residual or cannot run at all."""
    try:
        return not (pin(impl) <= tol)
    except (ValueError, IndexError, FloatingPointError):
        return True


@pytest.mark.parametrize("kind", ["no_scale", "transposed_scores", "mask_direction", "mask_diagonal",
                                  "sum_over_columns", "lse_base2", "lse_drops_max", "values_are_keys"])
def test_forward_mutants_are_caught(kind):
    f = _mut_fwd(kind)
    fails = [
        _caught(pin_constant_scores, f),
        _caught(pin_dominant_key, f),
        _caught(pin_permutation, f),
        _caught(pin_blocked_equals_full, f),
        _caught(lambda g: pin_autograd(fwd=g), f),
    ]
    assert any(fails), kind


@pytest.mark.parametrize("kind", ["dv_untransposed", "ds_sign", "ds_drops_d", "dk_no_scale", "dq_uses_v"])
def test_backward_mutants_are_caught(kind):
    b = _mut_bwd(kind)
    fails = [_caught(lambda g, c=c: pin_finite_differences(bwd=g, causal=c), b) for c in (False, True)]
    assert any(fails), kind


def test_gqa_matches_torch_enable_gqa():
    assert pin_gqa_torch() < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_shared_head_gradient_finite_differences(causal):
    assert pin_gqa_finite_differences(causal=causal) < 1e-7


def test_gqa_with_equal_head_counts_is_multi_head():
    q, k, v, do = _gqa_case(80, H=3, Hkv=3)
    o, lse = A.forward(q, k, v, 0.5, True)
    for h in range(3):
        oh, lh = A.forward_head(q[1, :, h], k[1, :, h], v[1, :, h], 0.5, True)
        assert np.array_equal(o[1, :, h], oh) and np.array_equal(lse[1, h], lh)
    with pytest.raises(ValueError):
        A.kv_head(0, 6, 4)


def _mut_gqa_fwd(interleaved):
    def fwd(Q, K, V, scale, causal):
        b_, n_, h_, _ = Q.shape
        hkv = K.shape[2]
        O = np.zeros(Q.shape[:3] + (V.shape[3],))
        for b in range(b_):
            for h in range(h_):
                g = h % hkv if interleaved else A.kv_head(h, h_, hkv)
                O[b, :, h], _ = A.forward_head(Q[b, :, h], K[b, :, g], V[b, :, g], scale, causal)
        return O, None
    return fwd


def _mut_gqa_bwd(kind):
    def bwd(Q, K, V, dO, scale, causal):
        h_, hkv = Q.shape[2], K.shape[2]
        dQ, dK, dV = np.zeros(Q.shape), np.zeros(K.shape), np.zeros(V.shape)
        for b in range(Q.shape[0]):
            for h in range(h_):
                g = A.kv_head(h, h_, hkv)
                dq, dk, dv, _ = A.backward_head(Q[b, :, h], K[b, :, g], V[b, :, g], dO[b, :, h], scale, causal)
                dQ[b, :, h] = dq
                if kind == "last_head_wins":
                    dK[b, :, g], dV[b, :, g] = dk, dv
                elif kind == "group_mean":
                    dK[b, :, g] += dk / (h_ // hkv)
                    dV[b, :, g] += dv / (h_ // hkv)
        return dQ, dK, dV
    return bwd


def test_gqa_mutants_are_caught():
    # interleaved grouping (h % Hkv) instead of consecutive groups
    assert _caught(lambda g: pin_gqa_torch(fwd=g), _mut_gqa_fwd(True))
    assert not _caught(lambda g: pin_gqa_torch(fwd=g), _mut_gqa_fwd(False))
    for kind in ("last_head_wins", "group_mean"):
        b = _mut_gqa_bwd(kind)
        assert _caught(lambda g: pin_gqa_finite_differences(bwd=g), b, tol=1e-7), kind
        assert _caught(lambda g: pin_gqa_torch(bwd=g), b), kind


def test_window_rows_equal_attention_over_their_neighbourhood():
    assert pin_window_rowwise() < 1e-12


def test_window_zero_width_closed_form():
    assert pin_window_zero_width() < 1e-12


def test_window_special_cases_reduce_to_full_and_causal():
    q, k, v = _rand((19, 4), 100), _rand((19, 4), 101), _rand((19, 4), 102)
    full = A.forward_head(q, k, v, 0.5, False)
    causal = A.forward_head(q, k, v, 0.5, True)
    for a, b in zip(A.forward_head(q, k, v, 0.5, False, (None, None)), full):
        assert np.array_equal(a, b)
    for a, b in zip(A.forward_head(q, k, v, 0.5, False, (None, 0)), causal):
        assert np.array_equal(a, b)
    # a window wider than the sequence hides nothing
    for a, b in zip(A.forward_head(q, k, v, 0.5, True, (100, 100)), causal):
        assert np.array_equal(a, b)


def test_window_backward_finite_differences():
    for window in ((2, 1), (0, 3), (None, 0), (1, None)):
        assert pin_window_finite_differences(window=window) < 1e-7, window


def test_window_skips_the_pages_share_of_blocks():
    """The page: a 4096-token window over 32768 tokens leaves up to 87 % of the
    blocks uncomputed.  With the (4095, 0) reading and 128 x 128 blocks the
    mask hides 87.9 % of the full block grid."""
    g = json.loads((GOLDEN / "sliding_window_blocks.json").read_text())
    w = g["window_tokens"]
    frac = window_skipped_block_fraction(g["N"], (w - 1, 0), g["block"])
    assert g["skipped_fraction_stated"] <= frac < g["skipped_fraction_stated"] + 0.01


def _mut_window(kind):
    def hidden(rows, nk, causal, window=None):
        if window is not None and kind == "left_off_by_one":
            left, right = window
            window = (None if left is None else left + 1, right)
        if window is not None and kind == "swapped_sides":
            window = (window[1], window[0])
        return A.hidden_keys(rows, nk, causal, window)

    def fwd(q, k, v, scale, causal, window=None):
        s = scale * (np.asarray(q) @ np.asarray(k).T)
        s = np.where(hidden(np.arange(s.shape[0]), s.shape[1], causal, window), -np.inf, s)
        p, lse = A.probs_head(s)
        return p @ v, lse
    return fwd, hidden


@pytest.mark.parametrize("kind", ["left_off_by_one", "swapped_sides"])
def test_window_mutants_are_caught(kind):
    fwd, hidden = _mut_window(kind)
    assert _caught(pin_window_rowwise, fwd)
    if kind == "left_off_by_one":
        frac = window_skipped_block_fraction(32768, (4095, 0), 128, hidden=hidden)
        assert not (0.87 <= frac < 0.88) or _caught(pin_window_zero_width, fwd)


def test_blocksparse_rows_equal_attention_over_their_blocks():
    assert pin_blocksparse_rowwise() < 1e-12


def test_blocksparse_special_cases():
    n = 300
    q, k, v = _rand((n, 4), 120), _rand((n, 4), 121), _rand((n, 4), 122)
    full = A.forward_head(q, k, v, 0.5, False)
    causal = A.forward_head(q, k, v, 0.5, True)
    ones = np.ones((3, 3), dtype=np.uint8)
    for a, b in zip(A.forward_head(q, k, v, 0.5, False, None, ones), full):
        assert np.array_equal(a, b)
    # block-lower-triangular mask on top of the causal mask hides nothing more
    tril = np.tril(ones)
    for a, b in zip(A.forward_head(q, k, v, 0.5, True, None, tril), causal):
        assert np.array_equal(a, b)


def test_blocksparse_backward_finite_differences():
    assert pin_blocksparse_finite_differences() < 1e-7


def test_blocksparse_mutants_are_caught():
    def transposed_mask(q, k, v, scale, causal, window=None, block_mask=None):
        return A.forward_head(q, k, v, scale, causal, window, None if block_mask is None else block_mask.T)
    assert _caught(pin_blocksparse_rowwise, transposed_mask)

    def dense(q, k, v, scale, causal, window=None, block_mask=None):
        return A.forward_head(q, k, v, scale, causal, window, None)
    assert _caught(pin_blocksparse_rowwise, dense)



# ---------------------------------------------------------------------------
# Paged KV cache, one decode step ("Flash Attention" (Ultralytics glossary),
# "Flash Attention и смежные понятия", PagedAttention)
# ---------------------------------------------------------------------------

def _paged_case(seed, lens, H=6, Hkv=2, d=5, P=4, spare=3):
    """Contiguous per-sequence K/V, and a pool holding them in shuffled pages.

    The pool is built here by slicing each sequence into page-sized chunks and
    storing chunk c of sequence b at page perm[first page of b + c]; every pool
    row that holds no cached position is NaN, so reading one poisons the result.
    """
    rng = np.random.default_rng(seed)
    B = len(lens)
    q = rng.standard_normal((B, H, d))
    ks = [rng.standard_normal((n, Hkv, d)) for n in lens]
    vs = [rng.standard_normal((n, Hkv, d)) for n in lens]
    npages = [-(-n // P) for n in lens]
    total = sum(npages) + spare
    perm = rng.permutation(total)
    kc = np.full((total, P, Hkv, d), np.nan)
    vc = np.full((total, P, Hkv, d), np.nan)
    table = np.full((B, max(npages + [1]) + 1), -7, dtype=np.int64)
    first = 0
    for b, n in enumerate(lens):
        for c in range(npages[b]):
            page = perm[first + c]
            table[b, c] = page
            rows = slice(c * P, min(n, (c + 1) * P))
            kc[page, : rows.stop - rows.start] = ks[b][rows]
            vc[page, : rows.stop - rows.start] = vs[b][rows]
        first += npages[b]
    return q, ks, vs, kc, vc, table, np.asarray(lens)


def pin_paged_sdpa(decode=A.decode_paged):
    """One decode step against torch SDPA (fp64, CPU, enable_gqa) on each sequence's contiguous K/V."""
    worst = 0.0
    for seed, lens, H, Hkv, P in ((1, [7, 1, 12, 4], 6, 2, 4), (2, [9, 16, 3], 4, 4, 8), (3, [5, 11], 6, 1, 3)):
        q, ks, vs, kc, vc, table, lens_a = _paged_case(seed, lens, H=H, Hkv=Hkv, P=P)
        o, lse = decode(q, kc, vc, table, lens_a, 0.7)
        for b, n in enumerate(lens):
            tq = torch.tensor(q[b][:, None, :])            # [H, 1, d]
            tk = torch.tensor(ks[b].transpose(1, 0, 2))     # [Hkv, n, d]
            tv = torch.tensor(vs[b].transpose(1, 0, 2))
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.7, enable_gqa=True)
            s = 0.7 * torch.einsum("hd,hnd->hn", tq[:, 0], tk.repeat_interleave(H // Hkv, 0))
            ref_lse = torch.logsumexp(s, dim=1)
            err = max(float(np.max(np.abs(o[b] - ref[:, 0].numpy()))), float(np.max(np.abs(lse[b] - ref_lse.numpy()))))
            worst = max(worst, err if np.isfinite(err) else math.inf)
    return worst


def pin_paged_special_cases(decode=A.decode_paged):
    """Closed forms: one cached position gives O = v_0, LSE = scale <q, k_0>; none gives O = 0, LSE = -inf."""
    q, ks, vs, kc, vc, table, lens = _paged_case(4, [1, 0, 1], H=4, Hkv=2, P=4)
    o, lse = decode(q, kc, vc, table, lens, 0.9)
    worst = 0.0
    for b in (0, 2):
        for h in range(4):
            g = h // 2
            worst = max(worst, float(np.max(np.abs(o[b, h] - vs[b][0, g]))),
                        abs(float(lse[b, h]) - 0.9 * float(q[b, h] @ ks[b][0, g])))
    ok_empty = np.all(o[1] == 0.0) and np.all(np.isneginf(lse[1]))
    return worst if ok_empty and np.isfinite(worst) else math.inf


def test_paged_decode_matches_sdpa_on_contiguous_rows():
    assert pin_paged_sdpa() < 1e-12


def test_paged_decode_special_cases():
    assert pin_paged_special_cases() < 1e-12


def test_paged_decode_with_an_identity_table_is_the_plain_forward():
    """Pages laid out in order reduce the gather to slicing the flattened pool."""
    rng = np.random.default_rng(9)
    P, n, Hkv, H, d = 4, 10, 2, 4, 3
    kc = rng.standard_normal((3, P, Hkv, d))
    vc = rng.standard_normal((3, P, Hkv, d))
    q = rng.standard_normal((1, H, d))
    o, lse = A.decode_paged(q, kc, vc, np.arange(3)[None, :], np.array([n]), 0.4)
    kf, vf = kc.reshape(-1, Hkv, d)[:n], vc.reshape(-1, Hkv, d)[:n]
    for h in range(H):
        oh, lh = A.forward_head(q[0, h][None, :], kf[:, h // 2], vf[:, h // 2], 0.4, False)
        assert np.allclose(o[0, h], oh[0], rtol=0, atol=1e-14) and abs(lse[0, h] - lh[0]) < 1e-14


def _mut_paged(kind):
    def decode(Q, Kc, Vc, table, lens, scale):
        nb, nh, _ = Q.shape
        hkv, P = Kc.shape[2], Kc.shape[1]
        O = np.zeros(Q.shape)
        LSE = np.full((nb, nh), -np.inf)
        for b in range(nb):
            n = int(lens[b]) + (1 if kind == "one_row_too_many" else 0)
            if n == 0:
                continue
            row = table[(b + 1) % nb] if kind == "wrong_sequence" else table[b]
            if kind == "page_slot_swapped":
                idx = [(row[j % P], j // P) for j in range(n)]
            else:
                idx = [(row[j // P], j % P) for j in range(n)]
            kr = np.stack([Kc[p, s] for p, s in idx])
            vr = np.stack([Vc[p, s] for p, s in idx])
            for h in range(nh):
                g = h % hkv if kind == "interleaved_heads" else A.kv_head(h, nh, hkv)
                o, l = A.forward_rows_head(Q[b, h][None, :], kr[:, g], vr[:, g], [0], scale, False)
                O[b, h], LSE[b, h] = o[0], l[0]
        return O, LSE
    return decode


@pytest.mark.parametrize("kind", ["page_slot_swapped", "one_row_too_many", "wrong_sequence", "interleaved_heads"])
def test_paged_decode_mutants_are_caught(kind):
    with np.errstate(invalid="ignore", over="ignore"):
        try:
            worst = pin_paged_sdpa(decode=_mut_paged(kind))
        except (IndexError, ValueError):
            worst = math.inf  # the mistake reads outside the pool or table
    assert worst > 1e-6
    assert pin_paged_sdpa(decode=_mut_paged("none")) < 1e-12


def test_paged_decode_randomised_tables():
    """Random batches, page sizes, lengths and page orders (seeded): the paged
    oracle equals torch SDPA on each sequence's contiguous rows."""
    rng = np.random.default_rng(2024)
    for trial in range(12):
        B = int(rng.integers(1, 5))
        Hkv = int(rng.choice([1, 2, 3]))
        H = Hkv * int(rng.choice([1, 2, 4]))
        P = int(rng.choice([1, 2, 3, 5, 8]))
        lens = [int(x) for x in rng.integers(0, 23, size=B)]
        if max(lens) == 0:
            lens[0] = 1
        q, ks, vs, kc, vc, table, lens_a = _paged_case(100 + trial, lens, H=H, Hkv=Hkv, d=4, P=P,
                                                         spare=int(rng.integers(0, 4)))
        o, lse = A.decode_paged(q, kc, vc, table, lens_a, 0.8)
        for b, n in enumerate(lens):
            if n == 0:
                assert np.all(o[b] == 0) and np.all(np.isneginf(lse[b]))
                continue
            tq = torch.tensor(q[b][:, None, :])
            tk = torch.tensor(ks[b].transpose(1, 0, 2))
            tv = torch.tensor(vs[b].transpose(1, 0, 2))
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.8, enable_gqa=True)
            assert np.max(np.abs(o[b] - ref[:, 0].numpy())) < 1e-12
