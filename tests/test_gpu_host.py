"""GPU parity of the host-buffer entry point, pisa_attn_fwd_host: chunks of
(batch, head) slices are copied in, run through the whole forward and copied
back, with the copies overlapping the compute.  Compared against the device
entry point on the same inputs and against the fp64 oracle."""

import numpy as np
import pytest
import torch

from workloads import small_config
from parity_util import TOL, assert_output_close, inputs, oracle_head, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def _host(x: np.ndarray, dtype: str, pinned: bool) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t.clone()
    return t.pin_memory() if pinned else t


CASES = [
    # 2*3 = 6 slices in chunks of 4: one full chunk and a ragged one of 2
    (small_config("host_bf16_b128", batch=2, heads=3, L=700, d=128, block=128, keep_ratio=0.3, seed=41), 4),
    # 5 slices one at a time (every chunk reuses a staging slot two chunks later)
    (small_config("host_bf16_b64", heads=5, L=640, d=128, block=64, keep_ratio=0.25, seed=42), 1),
    (small_config("host_fp32_d64", dtype="fp32", heads=3, L=500, d=64, block=64, keep_ratio=0.3, seed=43), 2),
]


@pytest.mark.parametrize("cfg,chunk", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_host_entry_point_matches_device_path_and_oracle(lib, cfg, chunk):
    q, k, v = inputs(cfg)
    B = cfg.block
    kk = lib.keep_count(cfg.L, B, cfg.keep_ratio)
    qh, kh, vh = (_host(x, cfg.dtype, True) for x in (q, k, v))
    out = lib.attn_fwd_host(qh, kh, vh, B, cfg.keep_ratio, chunk=chunk)
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    got = out.float().numpy()
    # the same slices through the device entry point, one launch per chunk shape
    qd, kd, vd = (to_device(x, cfg.dtype) for x in (q, k, v))
    dev = lib.attn_fwd(qd, kd, vd, B, cfg.keep_ratio).float().cpu().numpy()
    # per-chunk launches group Hbar's fixed-order partial sums differently, so
    # the two paths may differ in the last bits of a few outputs
    tol_abs, _ = TOL[cfg.dtype]
    diff = np.abs(got - dev)
    assert diff.max() <= tol_abs, f"host vs device path: max-abs {diff.max():.3e}"
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            r = oracle_head(q[b, h], k[b, h], v[b, h], B, kk)
            assert_output_close(got[b, h], r["out"], cfg.dtype, f"{cfg.name}[{b},{h}]")


def test_single_chunk_is_bit_identical_to_device_path(lib):
    cfg = small_config("host_single", heads=4, L=1000, d=128, block=128, keep_ratio=0.2, seed=44)
    q, k, v = inputs(cfg)
    qh, kh, vh = (_host(x, cfg.dtype, True) for x in (q, k, v))
    out = lib.attn_fwd_host(qh, kh, vh, cfg.block, cfg.keep_ratio, chunk=cfg.heads)
    qd, kd, vd = (to_device(x, cfg.dtype) for x in (q, k, v))
    dev = lib.attn_fwd(qd, kd, vd, cfg.block, cfg.keep_ratio)
    torch.cuda.synchronize()
    assert torch.equal(out, dev.cpu())


def test_pageable_buffers_and_repeat_calls(lib):
    cfg = small_config("host_pageable", heads=3, L=900, d=128, block=128, keep_ratio=0.3, seed=45)
    q, k, v = inputs(cfg)
    qh, kh, vh = (_host(x, cfg.dtype, False) for x in (q, k, v))
    a = lib.attn_fwd_host(qh, kh, vh, cfg.block, cfg.keep_ratio, chunk=2)
    torch.cuda.synchronize()
    b = lib.attn_fwd_host(qh, kh, vh, cfg.block, cfg.keep_ratio, chunk=2)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert lib.device_status() == 0
    kk = lib.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
    r = oracle_head(q[0, 1], k[0, 1], v[0, 1], cfg.block, kk)
    assert_output_close(a[0, 1].float().numpy(), r["out"], cfg.dtype, "pageable head 1")
