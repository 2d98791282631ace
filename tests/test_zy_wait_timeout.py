"""Bounded device waits that run out, and the unwind after them.

Every mbarrier wait between the warps of the tensor-core kernels (statistics,
covariance norm, routing, fused attention) is bounded.  A wait that runs out records
PISA_ERR_TIMEOUT in the device error word, the CTA lets the copies and MMAs it
already issued complete, frees its tensor memory and exits.  Here the limit is
set to 1 ns through pisa_set_wait_limit, so the first wait that has to spin
gives up: nothing faults or hangs, the host reads the status, and the same
process then runs a normal forward that matches the oracle.  The routing call
runs on valid statistics; its selections are then undefined (the timed-out
CTAs skip the top-k), and the fused call uses the selections computed before.

Collected after the other GPU tests (and before the no-allocation entry
point's file), so that a run stopping at the first failure has run them.
"""

import numpy as np
import pytest
import torch

from workloads import small_config
from parity_util import assert_output_close, inputs, oracle_head, to_device

pytestmark = pytest.mark.gpu

CFG = small_config("wait_timeout", L=4096, d=128, block=128, heads=4, keep_ratio=0.2, seed=34)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def test_short_wait_limit_times_out_each_kernel_then_context_stays_usable(lib):
    q, k, v = inputs(CFG)
    qd, kd, vd = (to_device(x, CFG.dtype) for x in (q, k, v))
    B = CFG.block
    kk = lib.keep_count(CFG.L, B, CFG.keep_ratio)
    # valid intermediate inputs at the default limit
    qbar, kbar, vsum, hbar = lib.block_stats(qd, kd, vd, B)
    M = lib.cov_norm(kd, vd, B, kbar, vsum, hbar)
    sel = lib.select(qbar, kbar, M, CFG.L, B, kk)
    torch.cuda.synchronize()
    assert lib.device_status() == lib.PISA_OK

    stages = {
        "statistics": lambda: lib.block_stats(qd, kd, vd, B),
        "covariance norm": lambda: lib.cov_norm(kd, vd, B, kbar, vsum, hbar),
        "routing": lambda: lib.select(qbar, kbar, M, CFG.L, B, kk),
        "fused attention": lambda: lib.attn_fwd_with_sel(qd, kd, vd, B, kbar, vsum, hbar, sel),
    }
    try:
        lib.set_wait_limit(1)
        for name, run in stages.items():
            run()  # the call itself is accepted: the timeout happens on the device
            torch.cuda.synchronize()
            assert lib.device_status(reset=True) == lib.PISA_ERR_TIMEOUT, name
    finally:
        lib.set_wait_limit(0)
    assert lib.device_status() == lib.PISA_OK

    out = lib.attn_fwd(qd, kd, vd, B, CFG.keep_ratio)
    torch.cuda.synchronize()
    assert lib.device_status() == lib.PISA_OK
    got = out.float().cpu().numpy()
    for h in range(CFG.heads):
        r = oracle_head(q[0, h], k[0, h], v[0, h], B, kk)
        assert_output_close(got[0, h], r["out"], CFG.dtype, f"after timeout, head {h}")
