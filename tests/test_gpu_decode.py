"""One decode step over a paged KV cache: the CUDA kernel against the fp64 oracle.

The pool's pages are handed out to the sequences in a shuffled order (the
seeded generator in exact_io_aware_51_b200.inputs), so consecutive positions of
a sequence live in unrelated pages.  Pool rows that hold no cached position are
set to NaN in most cases: the kernel must never let one reach an output.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import exact_io_aware_51_b200 as fa
import oracle
from exact_io_aware_51_b200 import inputs as I
from tests.helpers import TOL_BF16_REL, TOL_LSE, abs_err, need_gpu, rel_err


def _poison_unused(k, v, table, lens, page_size):
    """NaN in every pool row that is not a cached position of some sequence."""
    used = torch.zeros(k.shape[0], page_size, dtype=torch.bool)
    for b, n in enumerate(lens):
        for j in range(n):
            used[int(table[b, j // page_size]), j % page_size] = True
    k = k.clone()
    v = v.clone()
    k[~used] = float("nan")
    v[~used] = float("nan")
    return k, v


def _run(B, H, Hkv, d, P, lens, seed, poison=True, spare=2, workspace="auto", max_pages=None):
    q, k, v, table, sl = I.make_paged_decode(B, H, Hkv, d, P, lens, seed=seed, spare_pages=spare,
                                             max_pages=max_pages)
    if poison:
        k, v = _poison_unused(k, v, table, lens, P)
    sc = float(np.float32(1.0 / math.sqrt(d)))
    dev = [t.cuda() for t in (q, k, v, table, sl)]
    ws = None
    if workspace == "none":
        ws = torch.empty(1, dtype=torch.uint8, device="cuda")
    o, lse = fa.decode_paged(*dev, scale=sc, workspace=ws)
    torch.cuda.synchronize()
    assert fa.last_device_status()[0] == 0
    ro, rl = oracle.decode_paged(q, k, v, table, sl, sc)
    return o.cpu(), lse.cpu(), ro, rl


def _check(o, lse, ro, rl, lens):
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))
            continue
        assert rel_err(o[b], ro[b]) <= TOL_BF16_REL, b
        assert abs_err(lse[b], rl[b]) <= TOL_LSE, b


CASES = [
    # B, H, Hkv, d, page_size, sequence lengths
    (4, 8, 2, 128, 16, [1, 17, 64, 200]),
    (3, 16, 16, 64, 8, [0, 65, 130]),
    (2, 32, 1, 128, 64, [300, 129]),       # 32 query heads on one K/V head: two head groups
    (2, 64, 8, 128, 256, [1000, 513]),
    (2, 32, 2, 64, 32, [63, 777]),         # 16 query heads per K/V head
    (1, 4, 4, 64, 4096, [5000]),           # a page longer than a tile
    (5, 12, 4, 128, 128, [128, 129, 0, 255, 1]),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}H{c[1]}kv{c[2]}d{c[3]}P{c[4]}" for c in CASES])
def test_decode_matches_oracle(case):
    need_gpu()
    B, H, Hkv, d, P, lens = case
    o, lse, ro, rl = _run(B, H, Hkv, d, P, lens, seed=sum(lens) % 97)
    _check(o, lse, ro, rl, lens)


@pytest.mark.gpu
def test_decode_split_and_unsplit_agree_with_the_oracle():
    """A long sequence in a small batch is split into key chunks (merged from fp32
    partials) when the workspace allows; without one it runs as one chunk."""
    need_gpu()
    lens = [9000, 3, 4100]
    B, H, Hkv, d, P = 3, 8, 2, 128, 16
    assert fa.decode_workspace_size(B, H, Hkv, d, P, (9000 + P - 1) // P) > 0
    o1, l1, ro, rl = _run(B, H, Hkv, d, P, lens, seed=4)
    o2, l2, _, _ = _run(B, H, Hkv, d, P, lens, seed=4, workspace="none")
    _check(o1, l1, ro, rl, lens)
    _check(o2, l2, ro, rl, lens)


@pytest.mark.gpu
def test_decode_is_deterministic():
    need_gpu()
    q, k, v, table, sl = (t.cuda() for t in I.make_paged_decode(4, 16, 4, 128, 16, [700, 64, 1, 2000], seed=8))
    a = fa.decode_paged(q, k, v, table, sl)
    b = fa.decode_paged(q, k, v, table, sl)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.gpu
def test_decode_full_size_sampled_sequences():
    """The measured workload (64 sequences, 64 query heads on 8 K/V heads, d 128,
    16-token pages, lengths 512..8192): six sequences against the oracle."""
    need_gpu()
    lens = I.decode_lengths(64, 512, 8192, seed=21)
    q, k, v, table, sl = I.make_paged_decode(64, 64, 8, 128, 16, lens, seed=21)
    o, lse = fa.decode_paged(*(t.cuda() for t in (q, k, v, table, sl)))
    torch.cuda.synchronize()
    assert fa.last_device_status()[0] == 0
    pick = [0, 7, 21, 33, 50, 63]
    sc = float(np.float32(1.0 / math.sqrt(128)))
    ro, rl = oracle.decode_paged(q[pick], k, v, table[pick], sl[pick], sc)
    _check(o[pick].cpu(), lse[pick].cpu(), ro, rl, [lens[i] for i in pick])


@pytest.mark.gpu
@pytest.mark.parametrize("what", ["page_index", "length"])
def test_decode_reports_out_of_range_device_inputs(what):
    """A page index outside the pool, or a length beyond the table, is caught by the
    kernel before any load: that sequence's rows come back empty, the others are
    exact, and the status word reports FA_ERR_DEVICE_INPUT (-9)."""
    need_gpu()
    lens = [100, 50, 80]
    B, H, Hkv, d, P = 3, 8, 2, 64, 16
    q, k, v, table, sl = I.make_paged_decode(B, H, Hkv, d, P, lens, seed=12)
    sc = float(np.float32(1.0 / math.sqrt(d)))
    ro, rl = oracle.decode_paged(q, k, v, table, sl, sc)
    if what == "page_index":
        table[1, 2] = k.shape[0] + 5
    else:
        sl[1] = table.shape[1] * P + 1
    fa.last_device_status()  # clear
    o, lse = fa.decode_paged(*(t.cuda() for t in (q, k, v, table, sl)), scale=sc)
    rc, detail = fa.last_device_status()
    assert rc == -9 and detail & 0x2000
    o, lse = o.cpu(), lse.cpu()
    assert torch.all(o[1] == 0) and torch.all(torch.isneginf(lse[1]))
    _check(o[[0, 2]], lse[[0, 2]], ro[[0, 2]], rl[[0, 2]], [lens[0], lens[2]])
