"""fa_bwd_static_scratch: the backward for callers that cannot allocate.

Some callers cannot allocate device memory when they run the backward pass
(their device memory is laid out once at start-up, or a cudaMalloc mid-run
could synchronise the device or fail under memory pressure).  For them the
library offers a backward whose scratch is an array compiled into the library.
These tests call it through the C ABI and compare it with fa_bwd (the caller
passes a workspace there) on the same inputs, twice in a row, so the second
call runs on the scratch the first one left behind.

The file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test.  It passes on its own in a
fresh process (the first call on the device does the one-time set-up) and
after the other tests.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import exact_io_aware_51_b200 as fa
from exact_io_aware_51_b200 import inputs as I
from tests.helpers import TOL_BF16_REL, need_gpu, rel_err

FA_ERR_TOO_LARGE = -8


def _static_bwd(q, k, v, o, do, lse, causal, scale):
    B, N, H, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = fa.lib().fa_bwd_static_scratch(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
        dk.data_ptr(), dv.data_ptr(), B, H, N, d, scale, int(causal), fa.FA_BF16,
        torch.cuda.current_stream().cuda_stream)
    assert rc == 0, fa.status_string(rc)
    return dq, dk, dv


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_static_scratch_backward_matches_fa_bwd_twice(causal):
    need_gpu()
    B, N, H, d = 1, 2048, 8, 128  # 8.1 MiB of scratch, well inside the array
    scale = float(np.float32(1.0 / math.sqrt(d)))
    q, k, v, do = (t.cuda() for t in I.make_inputs(B, N, H, d, seed=77))
    o, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
    ref = fa.bwd(q, k, v, o, do, lse, causal=causal, scale=scale)
    for _ in range(2):
        got = _static_bwd(q, k, v, o, do, lse, causal, scale)
        torch.cuda.synchronize()
        for g, r in zip(got, ref):
            assert torch.isfinite(g.float()).all()
            assert rel_err(g.cpu(), r.cpu()) <= TOL_BF16_REL
    assert fa.last_device_status()[0] == 0


@pytest.mark.gpu
def test_static_scratch_refuses_problems_beyond_its_size():
    need_gpu()
    # B1 H32 N16384 d128 needs a 256 MiB workspace: refused before any GPU work
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(16, device="cuda")
    rc = fa.lib().fa_bwd_static_scratch(*([t.data_ptr()] * 5), lse.data_ptr(), *([t.data_ptr()] * 3),
                                        1, 32, 16384, 128, 0.088, 0, fa.FA_BF16, None)
    assert rc == FA_ERR_TOO_LARGE
