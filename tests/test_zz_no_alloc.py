"""fa_bwd_static_scratch: the backward for callers that cannot allocate.

Some callers cannot allocate device memory when they run the backward pass
(their device memory is laid out once at start-up, or a cudaMalloc mid-run
could synchronise the device or fail under memory pressure).  For them the
library offers a backward whose scratch is an array compiled into the library.
These tests call it through the C ABI and compare it with fa_bwd (the caller
passes a workspace there) on the same inputs, twice in a row, so the second
call runs on the scratch the first one left behind; one whole head of each
gradient is also compared with the fp64 oracle.  A problem of another shape
run after a larger one that used the split-walk accumulators checks that no
call reads what an earlier one left in the shared array.

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
import oracle
from exact_io_aware_51_b200 import inputs as I
from tests.helpers import TOL_BF16_REL, f64, need_gpu, rel_err

FA_ERR_TOO_LARGE = -8
SCRATCH_BYTES = 64 << 20


def _static_bwd(q, k, v, o, do, lse, causal, scale):
    B, N, H, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = fa.lib().fa_bwd_static_scratch(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
        dk.data_ptr(), dv.data_ptr(), B, H, N, d, scale, int(causal), fa.FA_BF16,
        torch.cuda.current_stream().cuda_stream)
    assert rc == 0, fa.status_string(rc)
    return dq, dk, dv


def _problem(B, N, H, d, causal, seed):
    scale = float(np.float32(1.0 / math.sqrt(d)))
    host = I.make_inputs(B, N, H, d, seed=seed)
    q, k, v, do = (t.cuda() for t in host)
    o, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
    return host, (q, k, v, o, do, lse), scale


def _same_as_fa_bwd(dev, causal, scale):
    q, k, v, o, do, lse = dev
    ref = fa.bwd(q, k, v, o, do, lse, causal=causal, scale=scale)
    got = _static_bwd(q, k, v, o, do, lse, causal, scale)
    torch.cuda.synchronize()
    for g, r in zip(got, ref):
        assert torch.isfinite(g.float()).all()
        assert rel_err(g.cpu(), r.cpu()) <= TOL_BF16_REL
    return got


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_static_scratch_backward_matches_fa_bwd_and_oracle_twice(causal):
    need_gpu()
    # 8.1 MiB of base scratch; causal walks of this shape split in two, which
    # adds 16 MiB of fp32 dK / dV accumulators from the same array
    B, N, H, d = 1, 2048, 8, 128
    host, dev, scale = _problem(B, N, H, d, causal, seed=77)
    for _ in range(2):
        got = _same_as_fa_bwd(dev, causal, scale)
    # one whole head against the fp64 oracle
    h = 5
    rq, rk, rv, _ = oracle.backward_head(*(f64(t[0, :, h]) for t in host), scale, causal)
    for g, r in zip(got, (rq, rk, rv)):
        assert rel_err(g[0, :, h].cpu(), r) <= TOL_BF16_REL
    assert fa.last_device_status()[0] == 0


@pytest.mark.gpu
def test_static_scratch_other_shape_after_a_larger_split_problem():
    need_gpu()
    # a causal problem whose walks split (dK / dV accumulators in the array) ...
    _, dev, scale = _problem(1, 2048, 8, 128, True, seed=3)
    _same_as_fa_bwd(dev, True, scale)
    # ... then a smaller unsplit one of another shape with a ragged N: its
    # preprocess must rewrite everything its main kernel reads
    host, dev, scale = _problem(2, 1000, 3, 128, False, seed=4)
    got = _same_as_fa_bwd(dev, False, scale)
    rq, rk, rv, _ = oracle.backward_head(*(f64(t[1, :, 2]) for t in host), scale, False)
    for g, r in zip(got, (rq, rk, rv)):
        assert rel_err(g[1, :, 2].cpu(), r) <= TOL_BF16_REL
    assert fa.last_device_status()[0] == 0


@pytest.mark.gpu
def test_static_scratch_runs_unsplit_when_only_the_base_fits():
    need_gpu()
    # B1 H4 N12288 d128 causal: the base workspace (24 MiB) fits the array, the
    # split-walk accumulators (48 MiB more) do not; the call runs unsplit
    B, N, H, d = 1, 12288, 4, 128
    full = fa.bwd_workspace_size(B, H, N, d)
    assert full > SCRATCH_BYTES > B * N * H * d * 4
    _, dev, scale = _problem(B, N, H, d, True, seed=5)
    _same_as_fa_bwd(dev, True, scale)
    assert fa.last_device_status()[0] == 0


@pytest.mark.gpu
def test_static_scratch_refuses_problems_beyond_its_size():
    need_gpu()
    # B1 H32 N16384 d128 needs a 256 MiB base workspace: refused before any GPU work
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(16, device="cuda")
    rc = fa.lib().fa_bwd_static_scratch(*([t.data_ptr()] * 5), lse.data_ptr(), *([t.data_ptr()] * 3),
                                        1, 32, 16384, 128, 0.088, 0, fa.FA_BF16, None)
    assert rc == FA_ERR_TOO_LARGE
