"""Helpers for the GPU parity tests: run the CUDA path stage by stage through
the C ABI and compare each stage with the fp64 oracle on the same inputs."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from workloads import generate
from tie_guard import redraw_map

# Tolerances on the attention output (max-abs and relative L2 over the
# compared rows), per input dtype.
TOL = {"bf16": (2e-2, 5e-3), "fp32": (1e-4, 1e-4)}


def to_device(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def inputs(cfg, redraws=None, heads=None):
    """Tie-guarded inputs for ``cfg`` (redraws computed with the oracle when
    not stored), as float32 numpy arrays [b, h, L, d]."""
    if redraws is None:
        kk = oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
        redraws = redraw_map(cfg, kk)
    return generate(cfg, heads=heads, redraws=redraws)


def oracle_head(q, k, v, B, kk, rows=None):
    return oracle.pisa_head(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), B, kk,
                            rows=rows)


def oracle_routing(q, k, v, B, kk):
    """The oracle's statistics and routing for one (batch, head), without the
    output rows: returns dict(sel, Hbar, M)."""
    q, k, v = (x.astype(np.float64) for x in (q, k, v))
    s = 1.0 / math.sqrt(q.shape[1])
    qbar, kbar, vsum, n = oracle.block_stats(q, k, v, B)
    H = oracle.first_order_blocks(k, v, B, kbar)
    Hbar = oracle.hbar_mean(H)
    M = oracle.cov_norm(H, Hbar)
    sel = oracle.select_topk(oracle.route_scores(qbar, kbar, M, n, s), kk)
    return dict(sel=sel, Hbar=Hbar, M=M, H_scale=float(np.sqrt((H ** 2).sum(axis=(1, 2))).max()))


def output_errors(gpu: np.ndarray, ref: np.ndarray):
    diff = gpu.astype(np.float64) - ref
    return float(np.abs(diff).max()), float(np.linalg.norm(diff) / np.linalg.norm(ref))


def assert_output_close(gpu, ref, dtype, what=""):
    max_abs, rel = output_errors(gpu, ref)
    tol_abs, tol_rel = TOL[dtype]
    assert max_abs <= tol_abs and rel <= tol_rel, f"{what}: max-abs {max_abs:.3e}, rel-L2 {rel:.3e}"
    return max_abs, rel


def assert_stat_close(gpu, ref, rel_tol, what):
    gpu = np.asarray(gpu, dtype=np.float64)
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(gpu - ref).max() / scale
    assert err <= rel_tol, f"{what}: max error {err:.3e} of max |ref|"
