"""Near-tie guard for the routing scores, computed with the fp64 oracle.

S_i must match bit for bit between the CUDA path (fp32 scores) and the oracle
(fp64 scores).  The workloads are therefore drawn so that, for every query
block, the k-th and (k+1)-th largest oracle scores differ by at least
``MIN_GAP`` (1e-3 in the log domain): where a row falls short, its query noise
is redrawn from the next redraw stream (workloads.gen.redraw_query_block) until
it clears the gap, with a cap of 64 attempts.
"""

from __future__ import annotations

import math

import numpy as np

import oracle
from workloads import generate_head, redraw_query_block

MIN_GAP = 1e-3
MAX_ATTEMPTS = 64


def _gap(row: np.ndarray, kk: int) -> float:
    if kk >= row.shape[0]:
        return math.inf
    top = np.sort(row)[::-1]
    return float(top[kk - 1] - top[kk])


def find_redraws(cfg, bh: int, kk: int):
    """Return ([(i, attempt), ...], min_gap_after) for stream bh of ``cfg``."""
    q, k, v, pos = generate_head(cfg, bh, None, return_pos=True)
    q = q.astype(np.float64)
    k = k.astype(np.float64)
    v = v.astype(np.float64)
    B = cfg.block
    s = 1.0 / math.sqrt(cfg.d)
    qbar, kbar, vsum, n = oracle.block_stats(q, k, v, B)
    H = oracle.first_order_blocks(k, v, B, kbar)
    M = oracle.cov_norm(H, oracle.hbar_mean(H))
    scores = oracle.route_scores(qbar, kbar, M, n, s)
    out = []
    min_gap = math.inf
    for i in range(scores.shape[0]):
        g = _gap(scores[i], kk)
        attempt = 0
        while g < MIN_GAP:
            attempt += 1
            if attempt > MAX_ATTEMPTS:
                raise RuntimeError(f"{cfg.name}: no tie-free redraw for stream {bh} block {i}")
            a, b = i * B, min((i + 1) * B, cfg.L)
            qb = redraw_query_block(cfg, bh, i, attempt, None if pos is None else pos[a:b])
            qb = qb.astype(np.float64)
            qbar_i = oracle.block_stats(qb, qb, qb, B)[0]
            g = _gap(oracle.route_scores(qbar_i, kbar, M, n, s)[0], kk)
        if attempt:
            out.append((i, attempt))
        min_gap = min(min_gap, g)
    return out, min_gap


def redraw_map(cfg, kk: int):
    """{bh: {i: attempt}} for every stream of a (small) config, serially."""
    table = {}
    for bh in range(cfg.batch * cfg.heads):
        pairs, _ = find_redraws(cfg, bh, kk)
        if pairs:
            table[bh] = dict(pairs)
    return table
