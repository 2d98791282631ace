"""The no-allocation entry point, pisa_attn_fwd_with_sel_noalloc.

It serves callers that are handed only their input and output buffers and
cannot create a workspace (no cudaMalloc: plugins living in another
framework's memory pool, pre-allocated serving runtimes).  The scratch that
pisa_attn_fwd_with_sel takes from the caller's workspace comes instead from a
fixed device array inside the library (PISA_NOALLOC_SCRATCH_BYTES = 32 MiB).

This file is collected last on purpose, so that a run which stops at the first
failure has already run every other test; each test also passes on its own in
a fresh process (the first call on a device sets the array's address up).
"""

import ctypes

import pytest
import torch

from workloads import small_config
from parity_util import inputs, to_device


def _raw_noalloc(lib, q, k, v, out, block, kbar, vsum, hbar, sel):
    """Call the entry point through the C ABI, on torch's current stream."""
    b, h, L, d = q.shape
    dtype = lib.PISA_BF16 if q.dtype == torch.bfloat16 else lib.PISA_FP32
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.raw_lib().pisa_attn_fwd_with_sel_noalloc(
        p(q), p(k), p(v), p(out), dtype, b, h, L, d, block, p(kbar), p(vsum), p(hbar), p(sel),
        int(sel.shape[-1]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


CASES = [
    small_config("noalloc_b128", L=3000, d=128, block=128, heads=3, keep_ratio=0.2, seed=31),
    small_config("noalloc_b64", L=1500, d=128, block=64, heads=2, keep_ratio=0.25, seed=32),
    small_config("noalloc_fp32", dtype="fp32", L=900, d=64, block=64, heads=2, keep_ratio=0.3, seed=35),
]


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice(lib):
    """Calls in a row (several shapes, so each reuses the array left by the one
    before) give exactly the output of pisa_attn_fwd_with_sel, which runs the
    same kernels on the same operands with a caller workspace: only where the
    scratch lives differs, so the outputs must be bit-identical."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    for cfg in CASES:
        q, k, v = inputs(cfg)
        qd, kd, vd = (to_device(x, cfg.dtype) for x in (q, k, v))
        B = cfg.block
        kk = lib.keep_count(cfg.L, B, cfg.keep_ratio)
        assert lib.fused_workspace_size(cfg.batch, cfg.heads, cfg.L, cfg.d, B) <= lib.NOALLOC_SCRATCH_BYTES
        qbar, kbar, vsum, hbar = lib.block_stats(qd, kd, vd, B)
        M = lib.cov_norm(kd, vd, B, kbar, vsum, hbar)
        sel = lib.select(qbar, kbar, M, cfg.L, B, kk)
        ref = lib.attn_fwd_with_sel(qd, kd, vd, B, kbar, vsum, hbar, sel)
        out = torch.full_like(ref, float("nan"))
        assert _raw_noalloc(lib, qd, kd, vd, out, B, kbar, vsum, hbar, sel) == lib.PISA_OK
        torch.cuda.synchronize()
        assert lib.device_status() == 0
        assert torch.equal(out, ref), f"{cfg.name}: differs from pisa_attn_fwd_with_sel"


def test_noalloc_rejects_shapes_beyond_its_array(lib):
    """Scratch needs above the fixed array are refused before any launch."""
    raw = lib.raw_lib()
    fake = ctypes.c_void_p(0x10000)
    heads, L = 64, 131072  # fused scratch far above 32 MiB
    assert lib.fused_workspace_size(1, heads, L, 128, 128) > lib.NOALLOC_SCRATCH_BYTES
    rc = raw.pisa_attn_fwd_with_sel_noalloc(fake, fake, fake, fake, lib.PISA_BF16, 1, heads, L, 128, 128,
                                            fake, fake, fake, fake, 8, None)
    assert rc == lib.PISA_ERR_WORKSPACE
