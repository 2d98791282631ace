"""Bounded device waits that run out, and the unwind after them.

Every mbarrier wait between the warps of the tensor-core kernels (statistics,
covariance norm, routing, fused attention) is bounded.  A wait that runs out records
PISA_ERR_TIMEOUT in the device error word, the CTA lets the copies and MMAs it
already issued complete, frees its tensor memory and exits.  Here the limit is
set to 1 ns through pisa_set_wait_limit, so the first wait that has to spin
gives up: nothing faults or hangs, the host reads the status, and the same
process then runs a normal forward that matches the oracle.  The timed-out
calls' results are undefined (the routing call's CTAs skip the top-k); the
fused call uses selections computed before, at the default limit.

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
# the calls that time out run on a larger shape: many CTAs and thousands of
# waits, so that some wait certainly spans a tick of the GPU's global timer
# (its resolution is coarser than the 1 ns limit)
BIG = small_config("wait_timeout_big", L=16384, d=128, block=128, heads=8, keep_ratio=0.2, seed=35)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def test_short_wait_limit_times_out_each_kernel_then_context_stays_usable(lib):
    # valid intermediate inputs at the default limit
    bq, bk, bv = (to_device(x, BIG.dtype) for x in inputs(BIG, redraws={}))
    B = BIG.block
    bkk = lib.keep_count(BIG.L, B, BIG.keep_ratio)
    qbar, kbar, vsum, hbar = lib.block_stats(bq, bk, bv, B)
    M = lib.cov_norm(bk, bv, B, kbar, vsum, hbar)
    sel = lib.select(qbar, kbar, M, BIG.L, B, bkk)
    # the routing call gets its own statistics with many key blocks (1024 per
    # head, 16 heads: 512 CTAs of 16 staged tiles), seeded noise: only its
    # status is checked
    gen = torch.Generator(device="cuda").manual_seed(7)
    rnb, rheads = 1024, 16
    rq = torch.randn(1, rheads, rnb, 128, device="cuda", generator=gen)
    rk = torch.randn(1, rheads, rnb, 128, device="cuda", generator=gen)
    rM = torch.rand(1, rheads, rnb, device="cuda", generator=gen)
    rL = rnb * 128
    rkk = lib.keep_count(rL, 128, 0.1)
    torch.cuda.synchronize()
    assert lib.device_status() == lib.PISA_OK

    stages = {
        "statistics": lambda: lib.block_stats(bq, bk, bv, B),
        "covariance norm": lambda: lib.cov_norm(bk, bv, B, kbar, vsum, hbar),
        "routing": lambda: lib.select(rq, rk, rM, rL, 128, rkk),
        "fused attention": lambda: lib.attn_fwd_with_sel(bq, bk, bv, B, kbar, vsum, hbar, sel),
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

    q, k, v = inputs(CFG)
    qd, kd, vd = (to_device(x, CFG.dtype) for x in (q, k, v))
    kk = lib.keep_count(CFG.L, CFG.block, CFG.keep_ratio)
    out = lib.attn_fwd(qd, kd, vd, CFG.block, CFG.keep_ratio)
    torch.cuda.synchronize()
    assert lib.device_status() == lib.PISA_OK
    got = out.float().cpu().numpy()
    for h in range(CFG.heads):
        r = oracle_head(q[0, h], k[0, h], v[0, h], CFG.block, kk)
        assert_output_close(got[0, h], r["out"], CFG.dtype, f"after timeout, head {h}")
