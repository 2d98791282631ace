"""Writes tests/golden/tie_redraws.json: the query-noise redraws that keep every
named workload clear of routing-score near-ties (gap >= 1e-3 between the k-th
and (k+1)-th fp64 oracle score of every query block).

Calls only the oracle and the seeded generators.  Usage:
    python tests/golden/make_tie_redraws.py [config ...]
"""

from __future__ import annotations

import concurrent.futures
import json
import multiprocessing
import os
import sys
import time

# one BLAS thread per worker process: the pool already uses every core
for _var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_var, "1")

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(HERE))

import oracle  # noqa: E402
from workloads import CONFIGS  # noqa: E402
from tie_guard import MIN_GAP, find_redraws  # noqa: E402


def _one(name, bh):
    cfg = CONFIGS[name]
    kk = oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
    pairs, gap = find_redraws(cfg, bh, kk)
    return name, bh, pairs, gap


def main(names):
    path = os.path.join(HERE, "tie_redraws.json")
    table = {"min_gap": MIN_GAP, "configs": {}}
    if os.path.exists(path):
        with open(path) as f:
            table = json.load(f)
    ctx = multiprocessing.get_context("spawn")
    with concurrent.futures.ProcessPoolExecutor(max_workers=os.cpu_count(), mp_context=ctx) as ex:
        for name in names:
            t0 = time.time()
            cfg = CONFIGS[name]
            futs = [ex.submit(_one, name, bh) for bh in range(cfg.batch * cfg.heads)]
            redraws, gaps = [], []
            for fut in futs:
                _, bh, pairs, gap = fut.result()
                redraws += [[bh, i, a] for i, a in pairs]
                gaps.append(gap)
            redraws.sort()
            table["configs"][name] = {
                "k": oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio),
                "redraws": redraws,
                "min_gap_after": min(gaps),
            }
            print(f"{name}: {len(redraws)} redraws, min gap {min(gaps):.3e}, {time.time() - t0:.1f}s",
                  flush=True)
    with open(path, "w") as f:
        json.dump(table, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main(sys.argv[1:] or list(CONFIGS))
