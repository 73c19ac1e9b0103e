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
