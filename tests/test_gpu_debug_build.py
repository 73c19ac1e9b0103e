"""The checking build (libfa_debug.so, compiled with FA_DEBUG).

Its kernels check, before each load or store, that the row, head and batch
coordinates and the per-row LSE / D ranges lie inside their tensors; a failed
check records FA_ERR_DEVICE_CHECK (0x4000 | check id) in the status word and
skips the access, so nothing traps or faults.  These tests run it in a child
process (the binding loads it when FA_LIBRARY names it):

* on small forward and backward problems it gives the oracle's results with a
  clean status word;
* a host-side knob moves the forward's first key-tile row past N; the loader's
  check refuses the load, the launch reports the check (not a fault), and the
  next launch is correct.

The product library ignores that knob.
"""

from __future__ import annotations

import os
import subprocess
import sys
import textwrap

import pytest

from tests.helpers import need_gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import math, sys
    import numpy as np, torch
    sys.path.insert(0, ROOT)
    import exact_io_aware_51_b200 as fa
    import oracle
    from exact_io_aware_51_b200 import inputs as I
    assert fa.lib_path().name == "libfa_debug.so"

    def rel(x, ref):
        x = x.float().cpu().numpy().astype(np.float64)
        return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-6))

    for (B, N, H, d, causal) in ((2, 200, 3, 128, False), (1, 333, 2, 128, True), (2, 129, 2, 64, True)):
        sc = float(np.float32(1.0 / math.sqrt(d)))
        q, k, v, do = I.make_inputs(B, N, H, d, seed=N + d)
        qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
        o, lse = fa.fwd(qd, kd, vd, causal=causal, scale=sc)
        dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=sc)
        torch.cuda.synchronize()
        rc, detail = fa.last_device_status()
        assert rc == 0, (rc, hex(detail))
        for b in range(B):
            for h in range(H):
                args = [t[b, :, h].float().numpy().astype(np.float64) for t in (q, k, v, do)]
                o_ref, _ = oracle.forward_head(*args[:3], sc, causal)
                rq, rk, rv, _ = oracle.backward_head(*args, sc, causal)
                for got, ref in ((o[b, :, h], o_ref), (dq[b, :, h], rq), (dk[b, :, h], rk), (dv[b, :, h], rv)):
                    assert rel(got, ref) <= 2e-2

    # the 8-bit forward: its loads pass the same checks
    q, k, v, _ = I.make_inputs(1, 384, 2, 128, seed=9, with_do=False)
    q8, k8, v8 = (t.cuda().to(torch.float8_e4m3fn) for t in (q, k, v))
    sc = float(np.float32(1.0 / math.sqrt(128)))
    o8, _ = fa.fwd_fp8(q8, k8, v8, 1.0, 1.0, 1.0, scale=sc)
    torch.cuda.synchronize()
    assert fa.last_device_status()[0] == 0
    ro, _ = oracle.forward(*(t.float().cpu() for t in (q8, k8, v8)), sc, False)
    assert float(np.max(np.abs(o8.float().cpu().numpy() - ro))) <= 2.0 ** -4 * float(np.max(np.abs(ro))) + 2e-2

    # a key row past N: the loader's check refuses it, the waits for it expire
    q, k, v, _ = I.make_inputs(1, 512, 2, 128, seed=2, with_do=False)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    fa.set_wait_limit_ms(200)
    fa.debug_inject(2)
    try:
        fa.fwd(qd, kd, vd)
        rc, detail = fa.last_device_status()
    finally:
        fa.debug_inject(0)
        fa.set_wait_limit_ms(0)
    assert rc == -10, (rc, hex(detail))
    assert detail == 0x4000 | 0x02, hex(detail)
    sc = float(np.float32(1.0 / math.sqrt(128)))
    o, _ = fa.fwd(qd, kd, vd, scale=sc)
    assert fa.last_device_status()[0] == 0
    o_ref, _ = oracle.forward_head(*(t[0, :, 1].float().numpy().astype(np.float64) for t in (q, k, v)), sc, False)
    assert rel(o[0, :, 1], o_ref) <= 2e-2
    print("checking build ok")
""")


@pytest.mark.gpu
def test_checking_build_matches_oracle_and_reports_a_refused_access():
    need_gpu()
    env = dict(os.environ, FA_LIBRARY="libfa_debug.so")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD], capture_output=True, text=True,
                       env=env, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "checking build ok" in r.stdout


@pytest.mark.gpu
def test_product_library_ignores_the_checking_knob():
    need_gpu()
    import torch

    import exact_io_aware_51_b200 as fa
    from exact_io_aware_51_b200 import inputs as I
    assert fa.lib_path().name == "libfa.so"
    q, k, v, _ = I.make_inputs(1, 256, 1, 128, seed=3, with_do=False)
    fa.debug_inject(2)
    try:
        fa.fwd(q.cuda(), k.cuda(), v.cuda())
        torch.cuda.synchronize()
        assert fa.last_device_status()[0] == 0
    finally:
        fa.debug_inject(0)
