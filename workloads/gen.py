"""Seeded synthetic Q/K/V generators for the PISA attention workloads.

The pages evaluate PISA inside Wan2.1, HunyuanVideo and FLUX.1 (gist.science
technical summary of PISA, section 4 "Experimental results").  No weights or
prompts are used here: these generators stand in for those workloads with the
same token counts and head shapes, queries and keys that share a smooth
low-rank positional term over the latent token grid (the spatial/temporal
locality that makes block routing meaningful), and unit-variance values.

Recipe (one independent stream per (batch, head) pair, index bh = b*heads+h):

* Generator(PCG64(SeedSequence([seed, bh]))); draw order Q noise, K noise,
  V noise (each [L, d], N(0, 1)), then the positional parameters, then the
  outlier rows.
* "tiny": Q, K, V ~ N(0, 1); every KV block j adds one offset c_j ~ N(0, 0.5^2)
  (standard deviation 0.5) to all its K rows.
* grid workloads: tokens in raster order over the grid (x fastest), normalised
  coordinates u_a = pos_a / N_a.  P_t = A R^{-1/2} sum_r phi_r(u_t) w_r with
  w_r ~ N(0, I_d), phi_r(u) = sqrt(2) cos(2 pi f_r.u + theta_r), f_r integer
  in {0,1,2} per axis (not all zero), theta_r ~ U[0, 2 pi).  Q = noise + P,
  K = noise + P (the same P), V = noise.
* outliers (Hunyuan-like): floor(frac * L) K rows, chosen uniformly without
  replacement, take Student-t(dof) noise instead of N(0, 1).
* near-tie redraws: the query noise of block i of stream bh is redrawn from
  SeedSequence([seed, bh, i, attempt]) for the (bh, i, attempt) triples listed
  in a redraw map (computed once by a committed script with the fp64 oracle,
  stored under tests/golden/).
* values are drawn in float64, rounded to float32 (RNE) and, for bf16
  workloads, then rounded RNE to bf16; the rounded values are what every
  consumer receives.  Arrays are returned as float32 holding those values.
"""

from __future__ import annotations

import concurrent.futures
import dataclasses
import json
import math
import multiprocessing
import os
from typing import Dict, Iterable, Optional, Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    dtype: str                 # "bf16" or "fp32"
    batch: int
    heads: int
    L: int
    d: int
    block: int
    seed: int
    keep_ratio: float          # k = clamp(ceil(rho*nb - 1e-9), 1, nb)
    kind: str = "grid"         # "grid" or "tiny"
    grid: Optional[Tuple[int, ...]] = None
    R: int = 8
    A: float = 1.0
    outlier_frac: float = 0.0
    outlier_dof: float = 3.0
    tiny_offset_std: float = 0.5

    @property
    def nb(self) -> int:
        return -(-self.L // self.block)


CONFIGS: Dict[str, Config] = {
    "tiny": Config("tiny", "fp32", 1, 1, 1024, 64, 64, 0, keep_ratio=4 / 16, kind="tiny"),
    "flux": Config("flux", "bf16", 1, 24, 4608, 128, 64, 1, keep_ratio=0.25,
                   grid=(64, 72), R=8, A=1.0),
    "wan480": Config("wan480", "bf16", 1, 40, 32760, 128, 128, 2, keep_ratio=0.15,
                     grid=(21, 30, 52), R=16, A=1.5),
    "wan720": Config("wan720", "bf16", 1, 40, 75600, 128, 128, 3, keep_ratio=0.10,
                     grid=(21, 45, 80), R=16, A=1.5),
    "hunyuan": Config("hunyuan", "bf16", 1, 24, 119040, 128, 128, 4, keep_ratio=0.08,
                      grid=(31, 48, 80), R=16, A=2.0, outlier_frac=0.01, outlier_dof=3.0),
}


def config(name: str) -> Config:
    return CONFIGS[name]


def small_config(name: str, dtype: str = "bf16", batch: int = 1, heads: int = 2, L: int = 1000,
                 d: int = 128, block: int = 128, keep_ratio: float = 0.25, seed: int = 11,
                 kind: str = "grid", R: int = 8, A: float = 1.5, outlier_frac: float = 0.0) -> Config:
    """An ad-hoc shape for edge-case tests; a 1-D token grid of length L."""
    return Config(name, dtype, batch, heads, L, d, block, seed, keep_ratio=keep_ratio,
                  kind=kind, grid=(L,) if kind == "grid" else None, R=R, A=A,
                  outlier_frac=outlier_frac)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round to float32 (RNE), then to the nearest bf16 (RNE on the float32 bits).

    Returns float32 holding bf16-representable values.  Finite inputs only.
    """
    x32 = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x32.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _round(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_round(x)
    if dtype == "fp32":
        return np.asarray(x, dtype=np.float32)
    raise ValueError(dtype)


def _grid_coords(grid: Tuple[int, ...], L: int) -> np.ndarray:
    if int(np.prod(grid)) != L:
        raise ValueError(f"grid {grid} does not hold {L} tokens")
    t = np.arange(L, dtype=np.int64)
    coords = np.zeros((L, len(grid)))
    rem = t
    for a in range(len(grid) - 1, -1, -1):      # x (last axis) fastest
        coords[:, a] = (rem % grid[a]) / grid[a]
        rem = rem // grid[a]
    return coords


def _smooth_term(rng: np.random.Generator, cfg: Config) -> np.ndarray:
    ndim = len(cfg.grid)
    F = rng.integers(0, 3, size=(cfg.R, ndim))
    while True:
        zero = np.nonzero(~F.any(axis=1))[0]
        if len(zero) == 0:
            break
        F[zero] = rng.integers(0, 3, size=(len(zero), ndim))
    theta = rng.uniform(0.0, 2.0 * math.pi, size=cfg.R)
    W = rng.standard_normal((cfg.R, cfg.d))
    u = _grid_coords(cfg.grid, cfg.L)
    phi = math.sqrt(2.0) * np.cos(2.0 * math.pi * (u @ F.T) + theta[None, :])
    return (cfg.A / math.sqrt(cfg.R)) * (phi @ W)


def generate_head(cfg: Config, bh: int, redraws: Optional[Dict[int, int]] = None,
                  return_pos: bool = False):
    """Q, K, V of one (batch, head) stream, float32 [L, d] each.

    ``redraws`` maps query block index i -> attempt number (> 0) for this
    stream; those blocks get their query noise from the redraw stream.
    """
    L, d, B = cfg.L, cfg.d, cfg.block
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg.seed, bh])))
    qn = rng.standard_normal((L, d))
    kn = rng.standard_normal((L, d))
    vn = rng.standard_normal((L, d))
    if cfg.kind == "tiny":
        nb = cfg.nb
        offsets = rng.normal(0.0, cfg.tiny_offset_std, size=(nb, d))
        pos = None
        kn += offsets[np.arange(L) // B]
    elif cfg.kind == "grid":
        pos = _smooth_term(rng, cfg)
        if cfg.outlier_frac > 0:
            n_out = int(math.floor(cfg.outlier_frac * L))
            rows = rng.choice(L, size=n_out, replace=False)
            kn[rows] = rng.standard_t(cfg.outlier_dof, size=(n_out, d))
        kn += pos
    else:
        raise ValueError(cfg.kind)
    if pos is not None:
        qn += pos
    q = _round(qn, cfg.dtype)
    if redraws:
        for i, attempt in sorted(redraws.items()):
            if attempt <= 0:
                continue
            a, b = i * B, min((i + 1) * B, L)
            q[a:b] = redraw_query_block(cfg, bh, i, attempt, None if pos is None else pos[a:b])
    if return_pos:
        return q, _round(kn, cfg.dtype), _round(vn, cfg.dtype), pos
    return q, _round(kn, cfg.dtype), _round(vn, cfg.dtype)


def redraw_query_block(cfg: Config, bh: int, i: int, attempt: int, pos_block):
    """Rounded queries of block i of stream bh drawn from redraw stream ``attempt``.

    ``pos_block`` is the positional term of the block's rows (None for "tiny").
    """
    a, b = i * cfg.block, min((i + 1) * cfg.block, cfg.L)
    r2 = np.random.Generator(np.random.PCG64(
        np.random.SeedSequence([cfg.seed, bh, int(i), int(attempt)])))
    qn = r2.standard_normal((b - a, cfg.d))
    if pos_block is not None:
        qn += pos_block
    return _round(qn, cfg.dtype)


def _golden_dir() -> str:
    return os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests", "golden")


def load_redraws(name: str) -> Dict[int, Dict[int, int]]:
    """Redraw map {bh: {i: attempt}} for a named workload ({} when none stored)."""
    path = os.path.join(_golden_dir(), "tie_redraws.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        table = json.load(f)
    entry = table.get("configs", {}).get(name)
    if not entry:
        return {}
    out: Dict[int, Dict[int, int]] = {}
    for bh, i, attempt in entry["redraws"]:
        out.setdefault(int(bh), {})[int(i)] = int(attempt)
    return out


def generate(cfg: Config, heads: Optional[Iterable[int]] = None,
             redraws: Optional[Dict[int, Dict[int, int]]] = None, workers: Optional[int] = None):
    """Q, K, V as float32 arrays [batch, heads, L, d].

    ``heads`` selects a subset of the flat (batch*heads) stream indices; the
    result then has shape [1, len(heads), L, d].  ``redraws`` defaults to the
    stored map for named workloads.
    """
    if redraws is None:
        redraws = load_redraws(cfg.name) if cfg.name in CONFIGS else {}
    bhs = list(range(cfg.batch * cfg.heads)) if heads is None else list(heads)
    shape = (len(bhs), cfg.L, cfg.d)
    q = np.empty(shape, dtype=np.float32)
    k = np.empty(shape, dtype=np.float32)
    v = np.empty(shape, dtype=np.float32)
    if workers is None:
        big = len(bhs) * cfg.L * cfg.d >= 4_000_000
        workers = min(len(bhs), os.cpu_count() or 1, 16) if big else 1
    if workers <= 1 or len(bhs) <= 1:
        for n, bh in enumerate(bhs):
            q[n], k[n], v[n] = generate_head(cfg, bh, redraws.get(bh))
    else:
        # spawn (never fork): callers may already hold a CUDA context
        ctx = multiprocessing.get_context("spawn")
        with concurrent.futures.ProcessPoolExecutor(max_workers=workers, mp_context=ctx) as ex:
            futs = {ex.submit(generate_head, cfg, bh, redraws.get(bh)): n for n, bh in enumerate(bhs)}
            for fut in concurrent.futures.as_completed(futs):
                n = futs[fut]
                q[n], k[n], v[n] = fut.result()
    if heads is None:
        return (q.reshape(cfg.batch, cfg.heads, cfg.L, cfg.d),
                k.reshape(cfg.batch, cfg.heads, cfg.L, cfg.d),
                v.reshape(cfg.batch, cfg.heads, cfg.L, cfg.d))
    return q[None], k[None], v[None]
