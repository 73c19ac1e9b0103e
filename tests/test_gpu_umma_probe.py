"""One tcgen05 MMA tile per operand layout the kernels use, against a CPU matmul.

The probe places A [128][K] and B [N][K] in shared memory with the 128-byte
swizzle (or A in tensor memory), issues the MMAs from one thread and reads D
back from tensor memory.  The reference is a float64 matmul of the same bf16
values; bf16 products are exact in fp32, so only the accumulation order differs.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_io_aware_51_b200 as fa
from tests.helpers import need_gpu, rel_err

# (N, K, a_mn_major, b_mn_major, a_tmem): the forward's S = Q K^T (128x128x128 and
# 128x128x64), P V with P in TMEM (N = d), and the backward's S^T / dP^T
# (N = 64), dV / dK (K = 64, B MN-major) and dQ^T (both MN-major).
CASES = [
    (128, 128, 0, 0, 0),
    (128, 64, 0, 0, 0),
    (64, 128, 0, 0, 0),
    (128, 128, 0, 1, 1),
    (64, 128, 0, 1, 1),
    (128, 64, 0, 1, 0),
    (64, 128, 1, 1, 0),
    (128, 128, 1, 0, 0),
]


@pytest.mark.gpu
@pytest.mark.parametrize("n,k,a_mn,b_mn,a_tmem", CASES)
def test_umma_tile(n, k, a_mn, b_mn, a_tmem):
    need_gpu()
    g = torch.Generator().manual_seed(n * 1000 + k * 10 + a_mn * 4 + b_mn * 2 + a_tmem)
    a = torch.randn(128, k, generator=g).to(torch.bfloat16)
    b = torch.randn(n, k, generator=g).to(torch.bfloat16)
    d = fa.debug_umma(a.cuda(), b.cuda(), a_mn, b_mn, a_tmem)
    torch.cuda.synchronize()
    ref = a.double().numpy() @ b.double().numpy().T
    assert rel_err(d.cpu(), ref) < 1e-5


# 8-bit MMA (e4m3, K = 128): S = Q K^T (both K-major), O += P V with P in TMEM and
# V stored [keys][d] (B MN-major), and MN-major B from shared memory.
F8_CASES = [(128, 0, 0), (64, 0, 0), (128, 1, 1), (128, 1, 0), (64, 1, 1)]


@pytest.mark.gpu
@pytest.mark.parametrize("n,b_mn,a_tmem", F8_CASES)
def test_umma_tile_e4m3(n, b_mn, a_tmem):
    need_gpu()
    g = torch.Generator().manual_seed(n * 10 + b_mn * 2 + a_tmem)
    a = (torch.randn(128, 128, generator=g) * 4).to(torch.float8_e4m3fn)
    b = (torch.randn(n, 128, generator=g) * 4).to(torch.float8_e4m3fn)
    d = fa.debug_umma_f8(a.view(torch.uint8).cuda(), b.view(torch.uint8).cuda(), b_mn, a_tmem)
    torch.cuda.synchronize()
    # e4m3 values and their products are exact; the tensor core's fp32 accumulation
    # of 8-bit products may keep fewer mantissa bits than an fp32 add, so the
    # bound is 1e-3 (a wrong operand layout gives errors of order 1)
    ref = a.double().numpy() @ b.double().numpy().T
    assert rel_err(d.cpu(), ref) < 1e-3


# Two-CTA tile (cta_group::2, M = 256 over a cluster of two CTAs, each holding
# half of A's rows and half of B's rows): the forms a paired kernel would use for
# S = Q K^T (both K-major), P V with P in each CTA's TMEM and V's feature halves
# N-contiguous, and an MN-major B from shared memory.
TWO_CTA_CASES = [(128, 0, 0), (64, 0, 0), (128, 1, 1), (128, 1, 0)]


@pytest.mark.gpu
@pytest.mark.parametrize("k,b_mn,a_tmem", TWO_CTA_CASES)
def test_umma_tile_two_cta(k, b_mn, a_tmem):
    need_gpu()
    g = torch.Generator().manual_seed(7000 + k * 10 + b_mn * 2 + a_tmem)
    a = torch.randn(256, k, generator=g).to(torch.bfloat16)
    b = torch.randn(128, k, generator=g).to(torch.bfloat16)
    d = fa.debug_umma_2cta(a.cuda(), b.cuda(), b_mn, a_tmem)
    torch.cuda.synchronize()
    ref = a.double().numpy() @ b.double().numpy().T
    assert rel_err(d.cpu(), ref) < 1e-5


# Tensor-pipe rate (mode, n, traffic kind): the bare pipe for each MMA form the kernels
# could use, then a 128 x 128 x 16 stream under each kind of concurrent traffic.
RATE_CASES = ([(0, n, 0) for n in (64, 128, 256)] + [(1, n, 0) for n in (64, 128, 256)]
              + [(2, n, 0) for n in (128, 256)]
              + [(0, 128, k) for k in range(1, 15)] + [(1, 128, k) for k in (3, 4, 5, 6, 9)])


@pytest.mark.gpu
def test_mma_rate_table():
    """Clocks per MMA on every SM at once, and what concurrent traffic gets.

    Pins what the kernels' design rests on: a 128 x 128 x 16 MMA takes about 64
    SM clocks whether B alone or both operands come from shared memory, N = 256 and
    the CTA pair give no more per SM, N = 64 costs more per unit of work, and while
    MMAs with both operands in shared memory run, shared-memory reads by the LSU
    and by bulk copies are starved while stores, TMEM traffic and L1 loads are not.
    The issuing thread competes for its SMSP's issue slots: ALU-bound warps there
    (not elsewhere) slow the MMA stream; two issuers on two SMSPs, or one converged
    warp issuing through elect.sync, recover it.
    `-s` prints the table (one JSON line per case)."""
    need_gpu()
    import json
    rows = {}
    for mode, n, kind in RATE_CASES:
        r = fa.debug_mma_rate(mode, n, kind)
        rows[(mode, n, kind)] = r
        print(json.dumps(r))
    unit = lambda m, n, k=0: rows[(m, n, k)]["clk_per_128x128x16"]
    traffic = lambda m, k: rows[(m, 128, k)]["traffic_bytes_per_clk"]
    for m, n in ((0, 128), (0, 256), (1, 128), (1, 256), (2, 128), (2, 256)):
        assert unit(m, n) < 72.0, (m, n, unit(m, n))
    assert unit(0, 64) > 1.2 * unit(0, 128)
    for k in (1, 2, 3, 8):  # TMEM loads / stores, shared stores, L1 loads: the MMAs keep their rate
        assert unit(0, 128, k) < 72.0, (k, unit(0, 128, k))
    # shared-memory reads next to MMAs reading both operands from shared memory vs. B only
    assert traffic(0, 4) < 0.5 * traffic(1, 4), (traffic(0, 4), traffic(1, 4))
    assert traffic(0, 6) < 0.5 * traffic(1, 6), (traffic(0, 6), traffic(1, 6))
    # issue slots: one ALU-bound warp on the issuing thread's SMSP slows the MMAs more than
    # three on the other SMSPs, and a second issuer on another SMSP wins the rate back
    assert unit(0, 128, 11) > 1.3 * unit(0, 128, 12), (unit(0, 128, 11), unit(0, 128, 12))
    assert unit(0, 128, 12) < 72.0, unit(0, 128, 12)
    assert unit(0, 128, 13) < 0.8 * unit(0, 128, 10), (unit(0, 128, 13), unit(0, 128, 10))
    # and a converged warp issuing through elect.sync keeps its slots where a lone lane does not
    assert unit(0, 128, 14) < 0.8 * unit(0, 128, 11), (unit(0, 128, 14), unit(0, 128, 11))
