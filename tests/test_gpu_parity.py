"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small shapes are compared element by element at every stage (block stats,
H_j, Hbar, M_j, S_i, output); the named workloads run in the configuration the
bench times, with S_i compared bit for bit on sampled heads and the output on
sampled query blocks (the oracle computes those rows one block at a time).
"""

import concurrent.futures
import multiprocessing
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import config, load_redraws, small_config
from parity_util import (assert_output_close, assert_stat_close, inputs, oracle_head, oracle_routing,
                         to_device)

pytestmark = pytest.mark.gpu

SMALL = [
    small_config("ragged_bf16_b128", L=1000, d=128, block=128, heads=2, keep_ratio=0.25),
    small_config("ragged_bf16_b64", L=1000, d=128, block=64, heads=2, keep_ratio=0.2, seed=12),
    small_config("bf16_d64_b64", L=777, d=64, block=64, heads=2, keep_ratio=0.3, seed=13),
    small_config("bf16_d64_b128", L=700, d=64, block=128, heads=1, keep_ratio=0.4, seed=14),
    small_config("fp32_d128_b128", dtype="fp32", L=900, d=128, block=128, heads=2, keep_ratio=0.3, seed=15),
    small_config("fp32_d64_b64", dtype="fp32", L=640, d=64, block=64, heads=2, keep_ratio=0.25, seed=16),
    small_config("L_below_block", L=50, d=128, block=64, heads=2, keep_ratio=0.5, seed=17),
    small_config("single_token", L=1, d=64, block=64, heads=1, keep_ratio=1.0, seed=18),
    small_config("every_block", L=1100, d=128, block=128, heads=2, keep_ratio=1.0, seed=19),
    small_config("one_block_kept", L=1300, d=128, block=128, heads=2, keep_ratio=0.01, seed=20),
    small_config("batch2", batch=2, heads=3, L=600, d=128, block=64, keep_ratio=0.25, seed=21),
    small_config("outliers", L=2000, d=128, block=128, heads=1, keep_ratio=0.2, seed=22,
                 outlier_frac=0.01, A=2.0),
    small_config("many_blocks", L=8192, d=128, block=64, heads=1, keep_ratio=0.05, seed=23),
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def _run_stages(lib, cfg, q, k, v):
    B = cfg.block
    kk = lib.keep_count(cfg.L, B, cfg.keep_ratio)
    qd, kd, vd = (to_device(x, cfg.dtype) for x in (q, k, v))
    qbar, kbar, vsum, hbar = lib.block_stats(qd, kd, vd, B)
    H = lib.block_first_order(kd, vd, B, kbar, vsum)
    M = lib.cov_norm(kd, vd, B, kbar, vsum, hbar)
    sel = lib.select(qbar, kbar, M, cfg.L, B, kk)
    out_sel = lib.attn_fwd_with_sel(qd, kd, vd, B, kbar, vsum, hbar, sel)
    out = lib.attn_fwd(qd, kd, vd, B, cfg.keep_ratio)
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    f = lambda t: t.float().cpu().numpy()
    return kk, dict(qbar=f(qbar), kbar=f(kbar), vsum=f(vsum), hbar=f(hbar), H=f(H), M=f(M),
                    sel=sel.cpu().numpy(), out_sel=f(out_sel), out=f(out))


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_shapes_every_stage(lib, cfg):
    q, k, v = inputs(cfg)
    kk, g = _run_stages(lib, cfg, q, k, v)
    assert kk == oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
    # the staged call and the one-shot call run the same kernels
    np.testing.assert_array_equal(g["out"], g["out_sel"])
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            r = oracle_head(q[b, h], k[b, h], v[b, h], cfg.block, kk)
            tag = f"{cfg.name}[{b},{h}]"
            assert_stat_close(g["qbar"][b, h], r["qbar"], 1e-5, tag + " qbar")
            assert_stat_close(g["kbar"][b, h], r["kbar"], 1e-5, tag + " kbar")
            assert_stat_close(g["vsum"][b, h], r["vsum"], 1e-5, tag + " vsum")
            assert_stat_close(g["H"][b, h], r["H"], 1e-5, tag + " H")
            assert_stat_close(g["hbar"][b, h], r["Hbar"], 1e-4, tag + " Hbar")
            # M_j is a norm of H_j - Hbar: rounding in it scales with ||H_j||_F,
            # not with M_j (which is exactly 0 when nb = 1)
            h_scale = np.sqrt((r["H"] ** 2).sum(axis=(1, 2))).max()
            assert np.abs(g["M"][b, h] - r["M"]).max() <= 1e-5 * max(h_scale, 1e-30), tag + " M"
            np.testing.assert_array_equal(g["sel"][b, h], r["sel"], err_msg=tag + " S_i")
            assert_output_close(g["out"][b, h], r["out"], cfg.dtype, tag)


def test_tiny_workload_full(lib):
    cfg = config("tiny")
    q, k, v = inputs(cfg, redraws=load_redraws("tiny"))
    kk, g = _run_stages(lib, cfg, q, k, v)
    assert kk == 4
    r = oracle_head(q[0, 0], k[0, 0], v[0, 0], cfg.block, kk)
    np.testing.assert_array_equal(g["sel"][0, 0], r["sel"])
    assert_output_close(g["out"][0, 0], r["out"], "fp32", "tiny")


def test_repeat_calls_are_bit_identical(lib):
    cfg = SMALL[0]
    q, k, v = inputs(cfg)
    qd, kd, vd = (to_device(x, cfg.dtype) for x in (q, k, v))
    a = lib.attn_fwd(qd, kd, vd, cfg.block, cfg.keep_ratio)
    b = lib.attn_fwd(qd, kd, vd, cfg.block, cfg.keep_ratio)
    st_a = lib.block_stats(qd, kd, vd, cfg.block)
    st_b = lib.block_stats(qd, kd, vd, cfg.block)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    for x, y in zip(st_a, st_b):
        assert torch.equal(x, y)


# ---------------------------------------------------------------- named workloads

OUTPUT_HEADS = 8  # heads whose output rows are compared (spread over the batch x heads)


def _sample_blocks(nb, rng, n=6):
    pick = set(rng.choice(nb, size=min(n, nb), replace=False).tolist())
    pick.update({0, nb - 1})
    return sorted(pick)


@pytest.mark.parametrize("name", ["flux", "wan480", "wan720", "hunyuan"])
def test_named_workload(lib, name):
    """Every head: S_i bit for bit, Hbar and M_j against the oracle's
    statistics and routing.  Eight heads spread over the batch x heads: the
    output on sampled query blocks (always the first and the ragged last),
    computed by the oracle one block at a time."""
    cfg = config(name)
    q, k, v = inputs(cfg, redraws=load_redraws(name))
    kk = lib.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
    qd, kd, vd = (to_device(x, cfg.dtype) for x in (q, k, v))
    B = cfg.block
    out = lib.attn_fwd(qd, kd, vd, B, cfg.keep_ratio)
    qbar, kbar, vsum, hbar = lib.block_stats(qd, kd, vd, B)
    M = lib.cov_norm(kd, vd, B, kbar, vsum, hbar)
    sel = lib.select(qbar, kbar, M, cfg.L, B, kk)
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    out_np = out.float().cpu().numpy()
    assert np.isfinite(out_np).all()
    sel_np = sel.cpu().numpy()
    hbar_np, M_np = hbar.cpu().numpy(), M.cpu().numpy()
    del qd, kd, vd, out, qbar, kbar, vsum, hbar, M, sel
    torch.cuda.empty_cache()
    n_heads = cfg.batch * cfg.heads
    # the oracle's routing of every head, in a spawned worker pool (spawn: the
    # workers start clean, although this process already uses the GPU)
    ctx = multiprocessing.get_context("spawn")
    workers = max(1, min(8, (os.cpu_count() or 2) - 1, n_heads))
    with concurrent.futures.ProcessPoolExecutor(workers, mp_context=ctx) as pool:
        jobs = [pool.submit(oracle_routing, q[b, h], k[b, h], v[b, h], B, kk)
                for b, h in (divmod(bh, cfg.heads) for bh in range(n_heads))]
        routed = [j.result() for j in jobs]
    for bh in range(n_heads):
        b, h = divmod(bh, cfg.heads)
        r = routed[bh]
        np.testing.assert_array_equal(sel_np[b, h], r["sel"], err_msg=f"{name} [{b},{h}] S_i")
        assert_stat_close(hbar_np[b, h], r["Hbar"], 1e-4, f"{name} [{b},{h}] Hbar")
        assert np.abs(M_np[b, h] - r["M"]).max() <= 1e-5 * max(r["H_scale"], 1e-30), f"{name} [{b},{h}] M"
    rng = np.random.default_rng(cfg.seed)
    out_heads = np.unique(np.linspace(0, n_heads - 1, min(OUTPUT_HEADS, n_heads)).round().astype(int))
    for bh in out_heads:
        b, h = divmod(int(bh), cfg.heads)
        blocks = _sample_blocks(cfg.nb, rng)
        rows = np.concatenate([np.arange(i * B, min((i + 1) * B, cfg.L)) for i in blocks])
        r = oracle_head(q[b, h], k[b, h], v[b, h], B, kk, rows=rows)
        assert_output_close(out_np[b, h, rows], r["out"], cfg.dtype, f"{name} [{b},{h}]")


# ---------------------------------------------------------------- routing configurations for many blocks

MANY_BLOCKS = [
    # 1250 blocks: the tensor-core routing kernel runs 16 query blocks per CTA
    small_config("route_r16", L=80000, d=128, block=64, heads=1, keep_ratio=0.02, seed=61),
    # 2500 blocks: past its shared memory, the CUDA-core routing kernel takes over
    small_config("route_cuda_cores", L=160000, d=128, block=64, heads=1, keep_ratio=0.01, seed=62),
]


@pytest.mark.parametrize("cfg", MANY_BLOCKS, ids=lambda c: c.name)
def test_routing_for_many_blocks(lib, cfg):
    """S_i bit for bit against the oracle, M_j and sampled output rows, where
    nb is large enough to change the routing kernel's configuration."""
    q, k, v = inputs(cfg)
    kk = lib.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
    qd, kd, vd = (to_device(x, cfg.dtype) for x in (q, k, v))
    B = cfg.block
    qbar, kbar, vsum, hbar = lib.block_stats(qd, kd, vd, B)
    M = lib.cov_norm(kd, vd, B, kbar, vsum, hbar)
    sel = lib.select(qbar, kbar, M, cfg.L, B, kk)
    out = lib.attn_fwd(qd, kd, vd, B, cfg.keep_ratio)
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    r = oracle_routing(q[0, 0], k[0, 0], v[0, 0], B, kk)
    np.testing.assert_array_equal(sel[0, 0].cpu().numpy(), r["sel"], err_msg=f"{cfg.name} S_i")
    assert np.abs(M[0, 0].cpu().numpy() - r["M"]).max() <= 1e-5 * max(r["H_scale"], 1e-30)
    blocks = _sample_blocks(cfg.nb, np.random.default_rng(cfg.seed), n=4)
    rows = np.concatenate([np.arange(i * B, min((i + 1) * B, cfg.L)) for i in blocks])
    ro = oracle_head(q[0, 0], k[0, 0], v[0, 0], B, kk, rows=rows)
    assert_output_close(out[0, 0, rows].float().cpu().numpy(), ro["out"], cfg.dtype, cfg.name)
