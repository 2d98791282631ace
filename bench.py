"""Benchmark of the PISA piecewise sparse attention forward on B200.

One step = one full forward (block stats -> covariance norm -> routing ->
fused attention) over one batch of the named synthetic workload, inputs
resident in HBM.  Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan720]
    python bench.py --impl reference ...   # the fp64 CPU oracle, bounded sample

Multi-GPU (torchrun, one rank per GPU): every rank runs the same workload on
its own GPU (weak scaling, no data-path collective); the step time is the max
over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import config as workload_config, generate, load_redraws  # noqa: E402

METRIC = "PISA attn fwd ms & effective TFLOPS at Wan-like shape; % of bf16 tensor peak"
DEFAULT_WORKLOAD = "wan720"
L2_BYTES = 126 * 1024 * 1024


def describe(cfg, kk):
    grid = "x".join(str(g) for g in cfg.grid) if cfg.grid else "-"
    return (f"{cfg.name}: batch {cfg.batch}, {cfg.heads} heads, L={cfg.L} ({grid}), head_dim {cfg.d}, "
            f"block {cfg.block}, keep {cfg.keep_ratio:g} (k={kk} of {cfg.nb}), {cfg.dtype}")


def block_sizes(cfg):
    n = np.full(cfg.nb, cfg.block, dtype=np.int64)
    n[-1] = cfg.L - (cfg.nb - 1) * cfg.block
    return n


def effective_flops(cfg, sel):
    """Algorithmic FLOPs of one forward: exact = 4 d sum_i n_i sum_{j in S_i} n_j;
    approx = 4 d sum_i n_i |U_i| + 2 L d^2 + L d (per batch*head, summed)."""
    n = block_sizes(cfg).astype(np.float64)
    d, L = cfg.d, cfg.L
    sel = sel.reshape(-1, cfg.nb, sel.shape[-1])
    kk = sel.shape[-1]
    exact = 4.0 * d * float((n[None, :] * n[sel].sum(axis=-1)).sum())
    approx_per = 4.0 * d * float(n.sum()) * (cfg.nb - kk) + 2.0 * L * d * d + L * d
    return exact, approx_per * sel.shape[0]


def executed_mma_flops(cfg, sel):
    """FLOPs of the MMAs the tensor-core fused kernel issues for selections
    ``sel`` (bf16 path).  Every 128-row query tile runs one step per 128 keys
    of its work list (one 128-token block, or two 64-token entries stacked),
    then one step per 128 block centroids (nb rounded up to 128, padding and
    selected columns masked but computed), each step an S = Q K^T and an
    O += P V MMA group (2 x 2 x 128 x 128 x d), then q Hbar as a hi + lo pair
    (2 x 2 x 128 x d x d).  The exact work list of a tile is the union of the
    selections of its 128 / block query blocks."""
    d, B, L, nb = cfg.d, cfg.block, cfg.L, cfg.nb
    G = 128 // B
    sel = sel.reshape(-1, nb, sel.shape[-1])
    bh = sel.shape[0]
    n_tiles = -(-L // 128)
    ncent = -(-nb // 128)
    if G == 1:
        steps = np.full((bh, n_tiles), sel.shape[-1], dtype=np.int64)
    else:
        mask = np.zeros((bh, nb, nb), dtype=bool)
        np.put_along_axis(mask, sel.astype(np.int64), True, axis=2)
        pad = n_tiles * G - nb
        if pad:
            mask = np.concatenate([mask, np.zeros((bh, pad, nb), dtype=bool)], axis=1)
        union = mask.reshape(bh, n_tiles, G, nb).any(axis=2)
        steps = -(-union.sum(axis=2) // G)
    per_step = 4.0 * 128 * 128 * d
    return float(((steps + ncent) * per_step).sum() + bh * n_tiles * 4.0 * 128 * d * d)


def stage_bytes(cfg, kk):
    """Algorithmic HBM bytes per launch of the streaming kernels."""
    bh, L, d, nb = cfg.batch * cfg.heads, cfg.L, cfg.d, cfg.nb
    e = 2 if cfg.dtype == "bf16" else 4
    stats = bh * (3 * L * d * e + 3 * nb * d * 4)
    cov = bh * (2 * L * d * e + 2 * nb * d * 4 + nb * 4)
    select = bh * (2 * nb * d * 4 + nb * 4 + nb * kk * 4)
    return dict(stats=stats, cov_norm=cov, select=select)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def host_info():
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return model, os.cpu_count() or 1


# ------------------------------------------------------------------ CPU oracle


def oracle_step(cfg, qh, kh, vh, kk, block_stride):
    """One bounded sample of the workload on the fp64 oracle: the whole (batch,
    head)'s statistics and routing, then the output rows of every
    ``block_stride``-th query block.  The statistics time is charged pro rata
    to the rows computed.  Returns (flops, charged seconds, rows)."""
    import oracle  # CPU baseline only: nothing else in the bench touches the oracle
    q, k, v = (x.astype(np.float64) for x in (qh, kh, vh))
    t0 = time.perf_counter()
    s = 1.0 / math.sqrt(cfg.d)
    qbar, kbar, vsum, n = oracle.block_stats(q, k, v, cfg.block)
    H = oracle.first_order_blocks(k, v, cfg.block, kbar)
    Hbar = oracle.hbar_mean(H)
    M = oracle.cov_norm(H, Hbar)
    sel = oracle.select_topk(oracle.route_scores(qbar, kbar, M, n, s), kk)
    t1 = time.perf_counter()
    blocks = np.arange(0, cfg.nb, block_stride)
    rows = np.concatenate([np.arange(i * cfg.block, min((i + 1) * cfg.block, cfg.L)) for i in blocks])
    oracle.pisa_rows(q, k, v, cfg.block, sel, kbar, vsum, n, Hbar, rows, s)
    t2 = time.perf_counter()
    nbk = block_sizes(cfg).astype(np.float64)
    ex = 4.0 * cfg.d * float((nbk[blocks] * nbk[sel[blocks]].sum(axis=-1)).sum())
    ap = 4.0 * cfg.d * float(nbk[blocks].sum()) * (cfg.nb - kk) + (2.0 * cfg.d * cfg.d + cfg.d) * len(rows)
    charged = (t1 - t0) * len(rows) / cfg.L + (t2 - t1)
    return ex + ap, charged, len(rows)


def cpu_oracle_sample(cfg, q, k, v, kk, budget_s, block_stride=4):
    """Time the oracle on successive (batch, head) samples until ``budget_s``
    charged seconds are spent.  Returns (TFLOP/s, description, threads, seconds)."""
    qf, kf, vf = (x.reshape(-1, cfg.L, cfg.d) for x in (q, k, v))
    flops = spent = 0.0
    rows = heads = 0
    for bh in range(qf.shape[0]):
        f, t, r = oracle_step(cfg, qf[bh], kf[bh], vf[bh], kk, block_stride)
        flops, spent, rows, heads = flops + f, spent + t, rows + r, heads + 1
        if spent >= budget_s:
            break
    desc = (f"{heads} (batch, head) slices: full statistics and routing, output rows of every "
            f"{block_stride}th query block ({rows} rows), statistics time charged per row")
    return flops / spent / 1e12, desc, os.cpu_count() or 1, spent


def run_reference(args, cfg, kk):
    """--impl reference: the fp64 oracle as it stands on the host cores; each
    step is one bounded sample (one (batch, head), every 4th query block)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    nsl = min(cfg.batch * cfg.heads, 4)
    table = load_redraws(cfg.name)
    q, k, v = generate(cfg, heads=list(range(nsl)), redraws={bh: table.get(bh, {}) for bh in range(nsl)})
    q, k, v = (x.reshape(-1, cfg.L, cfg.d) for x in (q, k, v))
    per_step = []
    for step in range(args.warmup + args.steps):
        bh = step % nsl
        t0 = time.perf_counter()
        f, charged, rows = oracle_step(cfg, q[bh], k[bh], v[bh], kk, 4)
        if step >= args.warmup:
            per_step.append((f, charged))
    flops = sum(f for f, _ in per_step)
    spent = sum(t for _, t in per_step)
    value = flops / spent / 1e12
    full_flops = None
    model, cores = host_info()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": spent / len(per_step) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": describe(cfg, kk), "parallelism": "host cores",
                   "sample": "per step: one (batch, head), full statistics and routing, output rows of "
                             "every 4th query block; statistics time charged per row"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count() or 1, "kind": "oracle",
                         "sample": "per step: one (batch, head), every 4th query block", "cpu": model},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU path


def dense_reference(pisa, cfg, qd, kd, vd, stats, fused_ms, forward_ms, reps=3):
    """Dense-attention context on the same inputs: this library's fused kernel
    with every block selected (U_i empty, so the result is exact softmax
    attention) and torch's scaled_dot_product_attention.  Each is timed with
    CUDA events over ``reps`` calls after one warm-up call."""
    import torch
    b, h, L, d, B, nb = cfg.batch, cfg.heads, cfg.L, cfg.d, cfg.block, cfg.nb
    dense_flops = 4.0 * L * L * d * b * h
    out = {"flops": dense_flops}

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        z.record()
        torch.cuda.synchronize()
        return a.elapsed_time(z) / reps

    sel_all = torch.arange(nb, dtype=torch.int32, device=qd.device).expand(b, h, nb, nb).contiguous()
    o = torch.empty_like(qd)
    ws = torch.empty(max(pisa.fused_workspace_size(b, h, L, d, B), 16), dtype=torch.uint8, device=qd.device)
    ms = timed(lambda: pisa.attn_fwd_with_sel(qd, kd, vd, B, stats[1], stats[2], stats[3], sel_all, out=o,
                                              workspace=ws))
    out["pisa_every_block"] = {"ms": ms, "TFLOP/s": dense_flops / (ms * 1e-3) / 1e12}
    del sel_all, ws
    try:
        from torch.nn.functional import scaled_dot_product_attention as sdpa
        ms = timed(lambda: sdpa(qd, kd, vd))
        out["torch_sdpa"] = {"ms": ms, "TFLOP/s": dense_flops / (ms * 1e-3) / 1e12}
        out["pisa_forward_speedup_vs_sdpa"] = ms / forward_ms
        out["pisa_fused_speedup_vs_sdpa"] = ms / fused_ms
    except Exception as e:  # noqa: BLE001  (context only: report and go on)
        out["torch_sdpa"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    del o
    torch.cuda.empty_cache()
    return out


SWEEP_GRIDS = {4096: (4, 32, 32), 8192: (8, 32, 32), 16384: (16, 32, 32), 32768: (32, 32, 32)}
SWEEP_KEEP = (0.05, 0.1, 0.25, 0.5)


def run_sweep(args):
    """Sequence-length x density sweep (4K-32K tokens, the axes of the pages'
    kernel comparison): 24 heads, d=128, block 128, the video-like generator
    on a frames x 32 x 32 grid.  For each length: torch SDPA and this
    library's fused kernel with every block selected (dense context), then the
    whole PISA forward and its fused kernel at each keep ratio.  Prints one
    JSON line holding every row."""
    import dataclasses
    import torch
    from workloads import Config
    import sparse_attention_diffusion_block_b200 as pisa
    from torch.nn.functional import scaled_dot_product_attention as sdpa

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    rows = []

    def timed(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        z.record()
        torch.cuda.synchronize()
        return a.elapsed_time(z) / reps

    for L, grid in SWEEP_GRIDS.items():
        cfg = Config(f"sweep{L}", "bf16", 1, 24, L, 128, 128, seed=5, keep_ratio=0.1, kind="grid",
                     grid=grid, R=16, A=1.5)
        q, k, v = generate(cfg, redraws={})
        qd, kd, vd = (torch.from_numpy(x).to(dev).to(torch.bfloat16) for x in (q, k, v))
        b, h, nb, d, B = cfg.batch, cfg.heads, cfg.nb, cfg.d, cfg.block
        dense_flops = 4.0 * L * L * d * b * h
        stats = pisa.block_stats(qd, kd, vd, B)
        M = pisa.cov_norm(kd, vd, B, stats[1], stats[2], stats[3])
        ws_f = torch.empty(max(pisa.fused_workspace_size(b, h, L, d, B), 16), dtype=torch.uint8, device=dev)
        o = torch.empty_like(qd)
        sdpa_ms = timed(lambda: sdpa(qd, kd, vd))
        sel_all = torch.arange(nb, dtype=torch.int32, device=dev).expand(b, h, nb, nb).contiguous()
        every_ms = timed(lambda: pisa.attn_fwd_with_sel(qd, kd, vd, B, stats[1], stats[2], stats[3], sel_all,
                                                        out=o, workspace=ws_f))
        rows.append({"L": L, "keep": 1.0, "torch_sdpa_ms": sdpa_ms, "pisa_every_block_ms": every_ms,
                     "dense_TFLOP/s_sdpa": dense_flops / sdpa_ms / 1e9,
                     "dense_TFLOP/s_pisa_every_block": dense_flops / every_ms / 1e9})
        del sel_all
        for keep in SWEEP_KEEP:
            kk = pisa.keep_count(L, B, keep)
            ws = torch.empty(pisa.workspace_size(b, h, L, d, B, kk), dtype=torch.uint8, device=dev)
            fwd_ms = timed(lambda: pisa.attn_fwd(qd, kd, vd, B, keep, out=o, workspace=ws))
            sel = pisa.select(stats[0], stats[1], M, L, B, kk)
            fused_ms = timed(lambda: pisa.attn_fwd_with_sel(qd, kd, vd, B, stats[1], stats[2], stats[3], sel,
                                                            out=o, workspace=ws_f))
            torch.cuda.synchronize()
            ex, ap_ = effective_flops(dataclasses.replace(cfg, keep_ratio=keep), sel.cpu().numpy())
            rows.append({"L": L, "keep": keep, "k": kk, "forward_ms": fwd_ms, "fused_ms": fused_ms,
                         "effective_TFLOP/s": (ex + ap_) / fwd_ms / 1e9,
                         "speedup_vs_sdpa": sdpa_ms / fwd_ms})
            del ws, sel
        if pisa.device_status() != 0:
            raise RuntimeError("device status set during the sweep")
        del qd, kd, vd, stats, M, ws_f, o
        torch.cuda.empty_cache()
    print(json.dumps({"sweep": "PISA forward vs dense attention, 24 heads, d=128, block 128, bf16",
                      "rows": rows}), flush=True)
    return 0


ABLATION_SHAPES = ((4096, (4, 32, 32)), (8192, (8, 32, 32)))
ABLATION_KEEP = (0.1, 0.25)


def run_ablation(args):
    """Accuracy / cost of the first-order term (the hybrid s beta_t (q_t Hbar)
    against each unselected block's own s alpha_{t,j} (q_t H_j)) on small
    video-like shapes: 8 heads, d=128, block 128, the 3-D generator on a
    frames x 32 x 32 grid.  Both run on the same selections; the error is
    measured against exact softmax attention (this library's fused kernel with
    every block selected, which the oracle pins to dense attention), as
    rel-L2 and max-abs over the whole output, and the time is that of the
    attention call alone.  One JSON line."""
    import torch
    from workloads import Config
    import sparse_attention_diffusion_block_b200 as pisa

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)

    def timed(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        z.record()
        torch.cuda.synchronize()
        return a.elapsed_time(z) / reps

    def errors(x, ref):
        diff = (x.float() - ref.float())
        return {"rel_l2": float(diff.norm() / ref.float().norm()), "max_abs": float(diff.abs().max())}

    rows = []
    for L, grid in ABLATION_SHAPES:
        cfg = Config(f"ablation{L}", "bf16", 1, 8, L, 128, 128, seed=6, keep_ratio=0.1, kind="grid",
                     grid=grid, R=16, A=1.5)
        q, k, v = generate(cfg, redraws={})
        qd, kd, vd = (torch.from_numpy(x).to(dev).to(torch.bfloat16) for x in (q, k, v))
        B, nb = cfg.block, cfg.nb
        qbar, kbar, vsum, hbar = pisa.block_stats(qd, kd, vd, B)
        H = pisa.block_first_order(kd, vd, B, kbar, vsum)
        M = pisa.cov_norm(kd, vd, B, kbar, vsum, hbar)
        sel_all = torch.arange(nb, dtype=torch.int32, device=dev).expand(1, cfg.heads, nb, nb).contiguous()
        dense = pisa.attn_fwd_with_sel(qd, kd, vd, B, kbar, vsum, hbar, sel_all)
        for keep in ABLATION_KEEP:
            kk = pisa.keep_count(L, B, keep)
            sel = pisa.select(qbar, kbar, M, L, B, kk)
            hyb = pisa.attn_fwd_with_sel(qd, kd, vd, B, kbar, vsum, hbar, sel)
            blk = pisa.attn_fwd_blockwise_with_sel(qd, kd, vd, B, kbar, vsum, H, sel)
            t_h = timed(lambda: pisa.attn_fwd_with_sel(qd, kd, vd, B, kbar, vsum, hbar, sel, out=hyb))
            t_b = timed(lambda: pisa.attn_fwd_blockwise_with_sel(qd, kd, vd, B, kbar, vsum, H, sel, out=blk),
                        reps=2)
            rows.append({"L": L, "keep": keep, "k": kk,
                         "hybrid": {"ms": t_h, **errors(hyb, dense)},
                         "blockwise": {"ms": t_b, **errors(blk, dense)}})
        if pisa.device_status() != 0:
            raise RuntimeError("device status set during the ablation")
        del qd, kd, vd, H, dense, sel_all
        torch.cuda.empty_cache()
    print(json.dumps({"ablation": "first-order term: hybrid (Hbar, tensor cores) vs per-block H_j (CUDA cores); "
                                  "error against exact softmax attention", "heads": 8, "d": 128, "block": 128,
                      "rows": rows}), flush=True)
    return 0


def max_over_ranks(x: float, dist, device) -> float:
    """The maximum of ``x`` over all ranks (the slowest rank's time); ``x``
    itself when not distributed."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(flops_per_rank: float, world: int, ms: float) -> float:
    """Weak scaling: every rank runs the same workload, so the job moves
    ``world`` times the per-rank FLOPs in the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def shard_range(n: int, world: int, rank: int):
    """The contiguous (batch, head) slices [lo, hi) that ``rank`` of ``world``
    computes when one batch is split by heads: every slice on exactly one
    rank, shard sizes differing by at most one.  Each slice is an independent
    problem (its statistics, routing and output rows use no other slice), so
    the ranks exchange no data."""
    if not 0 <= rank < world or n < world:
        raise ValueError(f"cannot split {n} slices over {world} ranks")
    return n * rank // world, n * (rank + 1) // world


def sum_over_ranks(x: float, dist, device) -> float:
    """Sum of ``x`` over all ranks (``x`` itself when not distributed)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def _source_sha(paths):
    import hashlib
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel, workload):
    """(DRAM bytes per launch, how they were obtained) from a committed ncu
    capture, or (None, reason) when the kernel's sources changed since the
    capture (or none was taken)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, "no capture"
    with open(path) as f:
        table = json.load(f)
    e = table.get(kernel, {}).get(workload)
    if not e:
        return None, "no capture for this workload"
    try:
        if _source_sha(e["sources"]) != e["source_sha"]:
            return None, "kernel sources changed since the capture"
    except OSError:
        return None, "kernel sources missing"
    return e["bytes_per_launch"], e.get("how", "")


def spread(xs):
    """Median, 10th and 90th percentile of a list of times."""
    a = np.asarray(xs, dtype=np.float64)
    return {"ms": float(np.median(a)), "p10_ms": float(np.percentile(a, 10)),
            "p90_ms": float(np.percentile(a, 90)), "mean_ms": float(a.mean())}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="pisa", choices=["pisa", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle time for the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--autotune", action="store_true",
                    help="tune the result-invariant launch parameters for the workload first")
    ap.add_argument("--route", default="covariance", choices=["covariance", "pooled", "spectral"],
                    help="routing variant: the default covariance score with the Frobenius norm, "
                         "the pooled score, or the covariance score with the spectral norm")
    ap.add_argument("--sweep", action="store_true",
                    help="sequence-length x density sweep (4K-32K tokens) instead of the bench line")
    ap.add_argument("--ablation", action="store_true",
                    help="first-order term ablation (hybrid vs per-block H_j) on small shapes instead of the "
                         "bench line")
    ap.add_argument("--no-dense-reference", action="store_true",
                    help="skip the dense-attention context (every block selected; torch SDPA)")
    ap.add_argument("--e2e-chunk", type=int, default=2,
                    help="(batch, head) slices per chunk of the host-buffer pipeline")
    ap.add_argument("--heads", type=int, default=None,
                    help="run only the first N heads of the workload (profiling captures)")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="with N ranks: every rank runs the whole workload (replicas, weak scaling), "
                         "or the batch x heads slices are split over the ranks (heads, strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.route != "covariance":
        args.no_e2e = True  # the host-buffer entry point runs the default routing
    cfg = workload_config(args.workload)
    if args.heads is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, heads=min(args.heads, cfg.heads))

    if args.sweep:
        return run_sweep(args)
    if args.ablation:
        return run_ablation(args)
    if args.impl == "reference":
        import oracle  # reference arm: the oracle as it stands
        return run_reference(args, cfg, oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio))

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)

    # inputs first (the generator's worker pool is spawned, before any CUDA use)
    full_cfg = cfg
    sharded = args.shard == "heads" and world > 1
    if sharded:
        import dataclasses
        lo, hi = shard_range(cfg.batch * cfg.heads, world, rank)
        q, k, v = generate(cfg, heads=range(lo, hi))  # stored redraws, keyed by flat slice index
        cfg = dataclasses.replace(cfg, batch=1, heads=hi - lo)
    else:
        q, k, v = generate(cfg)

    import torch
    import sparse_attention_diffusion_block_b200 as pisa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    kk = pisa.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    qd, kd, vd = (torch.from_numpy(x).to(dev).to(tdt) for x in (q, k, v))
    b, h, L, d, B, nb = cfg.batch, cfg.heads, cfg.L, cfg.d, cfg.block, cfg.nb
    f32 = dict(dtype=torch.float32, device=dev)
    stats = (torch.empty(b, h, nb, d, **f32), torch.empty(b, h, nb, d, **f32),
             torch.empty(b, h, nb, d, **f32), torch.empty(b, h, d, d, **f32))
    M = torch.empty(b, h, nb, **f32)
    sel = torch.empty(b, h, nb, kk, dtype=torch.int32, device=dev)
    out = torch.empty_like(qd)
    u8 = dict(dtype=torch.uint8, device=dev)
    ws_stats = torch.empty(max(pisa.stats_workspace_size(b, h, L, d, B), 16), **u8)
    ws_fused = torch.empty(max(pisa.fused_workspace_size(b, h, L, d, B), 16), **u8)
    ws_all = torch.empty(pisa.workspace_size(b, h, L, d, B, kk), **u8)

    def forward(ev=None):
        if ev: ev[0].record()
        pisa.block_stats(qd, kd, vd, B, workspace=ws_stats, out=stats)
        if ev: ev[1].record()
        if args.route == "covariance":
            pisa.cov_norm(kd, vd, B, stats[1], stats[2], stats[3], out=M)
        elif args.route == "spectral":
            # variant: M_j as the spectral norm, from the stored block matrices
            Hb = pisa.block_first_order(kd, vd, B, stats[1], stats[2])
            pisa.cov_norm_spectral(Hb, stats[3], L, B, out=M)
            del Hb
        if ev: ev[2].record()
        if args.route == "pooled":
            pisa.select_route(stats[0], stats[1], None, L, B, kk, route="pooled", out=sel)
        else:
            pisa.select(stats[0], stats[1], M, L, B, kk, out=sel)
        if ev: ev[3].record()
        pisa.attn_fwd_with_sel(qd, kd, vd, B, stats[1], stats[2], stats[3], sel, out=out, workspace=ws_fused)
        if ev: ev[4].record()

    tuning = None
    if args.autotune:
        # result-invariant launch parameters, tuned once for this shape
        tuning = pisa.autotune(qd, kd, vd, B, cfg.keep_ratio, out=out, workspace=ws_all)

    # correctness guard: the staged calls equal the one-shot entry point
    forward()
    if args.route == "covariance":
        ref_out = pisa.attn_fwd(qd, kd, vd, B, cfg.keep_ratio, workspace=ws_all)
        torch.cuda.synchronize()
        if not torch.equal(ref_out, out):
            raise RuntimeError("staged forward differs from pisa_attn_fwd")
        del ref_out
    torch.cuda.synchronize()
    status = pisa.device_status()
    if status != 0:
        raise RuntimeError(f"device status {pisa.status_string(status)}")
    sel_np = sel.cpu().numpy()
    exact, approx = effective_flops(cfg, sel_np)
    flops = exact + approx

    for _ in range(args.warmup):
        forward()
    torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record()
        for s in range(K):
            forward(evs[s])
        t1.record()
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    total_ms = t0.elapsed_time(t1)
    names = ["stats", "cov_norm", "select", "fused"]
    stage_times = {n: [e[i].elapsed_time(e[i + 1]) for e in evs] for i, n in enumerate(names)}
    stage_ms = {n: sum(t) / K for n, t in stage_times.items()}
    total_ms = max_over_ranks(total_ms, dist, dev)
    ms = total_ms / K
    # replicas: every rank moves the same FLOPs; heads: the ranks' shares add up
    job_flops = sum_over_ranks(flops, dist, dev) if sharded else world * flops
    value = job_flops / (ms * 1e-3) / 1e12

    # end to end through the public API with host buffers: pisa_attn_fwd_host
    # copies chunks of heads in, computes and copies out, overlapping the three
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (x.to("cpu").pin_memory() for x in (qd, kd, vd))
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        ws_host = torch.empty(pisa.host_workspace_size(tdt, b, h, L, d, B, kk, args.e2e_chunk),
                              dtype=torch.uint8, device=dev)
        def e2e_step():
            pisa.attn_fwd_host(qh, kh, vh, B, cfg.keep_ratio, out=oh, chunk=args.e2e_chunk,
                               workspace=ws_host)
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(K):
            e2e_step()
        z.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(z), dist, dev) / K
        in_bytes = sum(x.numel() * x.element_size() for x in (qd, kd, vd))
        e2e = {"value": job_flops / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out.numel() * out.element_size(),
               "api": f"pisa_attn_fwd_host, pinned host buffers, chunks of {args.e2e_chunk} heads"}
        del ws_host

    peaks = measured_peaks()
    fused_ms = stage_ms["fused"]
    achieved = flops / (fused_ms * 1e-3) / 1e12
    # the burst peak for a timed region under two seconds (the clocks have no
    # time to settle at the power cap), the sustained one beyond
    sustained = total_ms >= 2000.0
    peak = peaks["bf16_sustained"] if sustained else peaks["bf16"]
    traffic, traffic_how = stored_traffic("fused", f"{cfg.name}:{cfg.heads}")
    executed = executed_mma_flops(cfg, sel_np) if cfg.dtype == "bf16" else None
    roofline = {"kernel": "fused attention (attn_fwd_with_sel)", "bound": "tensor",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic, "traffic_source": traffic_how,
                "algorithmic_flops_per_launch": flops,
                "peak_source": (f"{peaks['source']} {'sustained' if sustained else 'burst'} cuBLAS bf16: "
                                f"timed region {total_ms / 1e3:.2f} s "
                                f"({'>=' if sustained else '<'} 2 s)")}
    if executed is not None:
        ex_tf = executed / (fused_ms * 1e-3) / 1e12
        roofline.update({"executed_mma_flops_per_launch": executed, "executed_TFLOP/s": ex_tf,
                         "executed_frac": ex_tf / peak})
    sbytes = stage_bytes(cfg, kk)
    stages = {}
    for n in names:
        ent = spread(stage_times[n])
        if n in sbytes:
            gbs = sbytes[n] / (ent["ms"] * 1e-3) / 1e9
            ent.update({"algorithmic_bytes": sbytes[n], "GB/s": gbs, "frac_hbm": gbs / peaks["hbm"]})
        stages[n] = ent
    stages["fused"]["TFLOP/s"] = flops / (stages["fused"]["ms"] * 1e-3) / 1e12
    step_ms = [sum(e[i].elapsed_time(e[i + 1]) for i in range(4)) for e in evs]
    stages["step"] = spread(step_ms)

    dense = None
    if rank == 0 and world == 1 and not args.no_dense_reference:
        dense = dense_reference(pisa, cfg, qd, kd, vd, stats, fused_ms, ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, desc, threads, spent = cpu_oracle_sample(cfg, q, k, v, kk, args.cpu_budget)
        model, _ = host_info()
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"fp64 oracle on {desc}; {spent:.1f} s", "cpu": model}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": describe(full_cfg, kk),
                       "global_batch": full_cfg.batch if sharded else world * cfg.batch,
                       "seq_len": cfg.L,
                       "parallelism": (f"batch x heads split over {world} GPUs ({cfg.heads} slices on "
                                       f"rank 0, no data-path collective)" if sharded else
                                       f"replicas x{world} (one full forward per GPU)"),
                       "l2": f"inputs {3 * qd.numel() * qd.element_size() / 1e9:.2f} GB > L2 126 MB",
                       "route": args.route,
                       "launch_tuning": tuning or "built-in heuristics",
                       "flops_exact": exact, "flops_approx": approx},
            "roofline": roofline,
            "stages": stages,
            "cpu_baseline": cpu,
            "dense_reference": dense,
            "e2e": e2e,
            "gpu_launches": K * pisa.launches("attn_fwd", tdt),
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
