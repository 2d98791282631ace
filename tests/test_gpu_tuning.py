"""Launch tuning changes speed only: outputs with any tuning are bit-identical
to the built-in launch choices, and the tuning table survives a save/load."""

import os
import tempfile

import pytest
import torch

from workloads import small_config
from parity_util import inputs, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


CASES = [
    small_config("tune_b128", L=3000, d=128, block=128, heads=3, keep_ratio=0.2, seed=71),
    small_config("tune_b64", L=2000, d=128, block=64, heads=2, keep_ratio=0.25, seed=72),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_tuning_leaves_results_bit_identical(lib, cfg):
    q, k, v = inputs(cfg)
    qd, kd, vd = (to_device(x, cfg.dtype) for x in (q, k, v))
    shape = (cfg.batch, cfg.heads, cfg.L, cfg.d, cfg.block)
    lib.clear_tuning(*shape)
    ref = lib.attn_fwd(qd, kd, vd, cfg.block, cfg.keep_ratio)
    for t in [dict(cov_blocks_per_cta=1, select_rows_per_cta=8, fused_ctas=7),
              dict(cov_blocks_per_cta=5, select_rows_per_cta=3, fused_ctas=1),
              dict(cov_blocks_per_cta=1000, select_rows_per_cta=32, fused_ctas=10000)]:
        lib.set_tuning(*shape, **t)
        assert lib.get_tuning(*shape) == t
        out = lib.attn_fwd(qd, kd, vd, cfg.block, cfg.keep_ratio)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), t
    chosen = lib.autotune(qd, kd, vd, cfg.block, cfg.keep_ratio)
    assert lib.get_tuning(*shape) == chosen
    out = lib.attn_fwd(qd, kd, vd, cfg.block, cfg.keep_ratio)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert lib.device_status() == 0
    lib.clear_tuning(*shape)


def test_tuning_save_and_load_round_trip(lib):
    shape = (1, 5, 4096, 128, 128)
    lib.set_tuning(*shape, cov_blocks_per_cta=3, select_rows_per_cta=16, fused_ctas=120)
    with tempfile.TemporaryDirectory() as tmp:
        path = os.path.join(tmp, "tuning.txt")
        lib.tuning_save(path)
        lib.clear_tuning(*shape)
        assert lib.get_tuning(*shape) == dict(cov_blocks_per_cta=0, select_rows_per_cta=0, fused_ctas=0)
        lib.tuning_load(path)
        assert lib.get_tuning(*shape) == dict(cov_blocks_per_cta=3, select_rows_per_cta=16, fused_ctas=120)
        bad = os.path.join(tmp, "bad.txt")
        with open(bad, "w") as f:
            f.write("1 2 3\n")
        with pytest.raises(lib.PisaError):
            lib.tuning_load(bad)
    lib.clear_tuning(*shape)
