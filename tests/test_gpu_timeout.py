"""Bounded waits: a wait that can never complete ends with an error, not a hang.

The library's test knob makes the forward's first key-tile barrier expect 16
bytes that never arrive.  Every wait in the kernel is bounded, so the launch
gives up after the wait limit, releases its tensor memory and records the
failure in the device status word; the context stays usable and the next
launch is correct.  No fault, trap or endless loop is involved.
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


@pytest.mark.gpu
def test_expired_wait_reports_status_and_context_survives():
    need_gpu()
    q, k, v, _ = I.make_inputs(1, 512, 2, 128, seed=2, with_do=False)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    assert fa.last_device_status()[0] == 0
    fa.set_wait_limit_ms(200)
    fa.debug_inject(1)
    try:
        fa.fwd(qd, kd, vd)
        rc, detail = fa.last_device_status()
    finally:
        fa.debug_inject(0)
        fa.set_wait_limit_ms(0)
    assert rc == -7, rc
    assert detail & 0x1000, hex(detail)
    # the status word was cleared and the next launch is normal and correct
    sc = float(np.float32(1 / math.sqrt(128)))
    o, lse = fa.fwd(qd, kd, vd, scale=sc)
    assert fa.last_device_status()[0] == 0
    for h in range(2):
        o_ref, _ = oracle.forward_head(*(f64(t[0, :, h]) for t in (q, k, v)), sc, False)
        assert rel_err(o[0, :, h].cpu(), o_ref) <= TOL_BF16_REL
