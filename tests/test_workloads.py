"""The seeded generators: determinism, rounding, structure, and the stored
near-tie redraws (re-checked here against the fp64 oracle)."""

import math

import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, bf16_round, config, generate, generate_head, load_redraws, small_config
from tie_guard import MIN_GAP, find_redraws


def test_bf16_round_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 10 ** rng.uniform(-3, 3, 100000),
                        np.array([1.00390625, 1.01171875, -1.00390625, 0.0, -0.0])])
    x32 = x.astype(np.float32)
    ours = bf16_round(x32)
    theirs = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours.view(np.uint32), theirs.view(np.uint32))


def test_generation_is_deterministic_and_per_head_independent():
    cfg = config("flux")
    q1, k1, v1 = generate_head(cfg, 3)
    q2, k2, v2 = generate_head(cfg, 3)
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(v1, v2)
    q0, _, _ = generate_head(cfg, 2)
    assert not np.array_equal(q0, q1)
    qs, ks, vs = generate(cfg, heads=[3], redraws={})
    np.testing.assert_array_equal(qs[0, 0], q1)


def test_values_are_bf16_exact_and_shaped():
    cfg = config("flux")
    q, k, v = generate(cfg, heads=[0, 5])
    assert q.shape == (1, 2, 4608, 128) and q.dtype == np.float32
    for x in (q, k, v):
        assert np.all((x.view(np.uint32) & 0xFFFF) == 0)
    # unit-variance values, keys with the positional term on top
    assert abs(v.std() - 1) < 0.02
    assert k.std() > 1.2


def test_tiny_block_offsets_and_dtype():
    cfg = config("tiny")
    q, k, v = generate(cfg)
    assert q.shape == (1, 1, 1024, 64)
    means = k[0, 0].reshape(16, 64, 64).mean(axis=1)
    # per-block offsets N(0, 0.5): centroids differ between blocks far more than noise/8
    assert means.std(axis=0).mean() > 0.35


def test_outlier_rows_are_heavy_tailed():
    cfg = small_config("o", L=4000, heads=1, outlier_frac=0.01, A=0.0)
    _, k, _ = generate(cfg)
    row_max = np.abs(k[0, 0]).max(axis=1)
    assert (row_max > 8).sum() >= 5


def test_redraws_change_only_their_block():
    cfg = config("tiny")
    a = generate_head(cfg, 0, {})[0]
    b = generate_head(cfg, 0, {5: 2})[0]
    diff = np.nonzero(np.any(a != b, axis=1))[0]
    assert diff.min() >= 5 * 64 and diff.max() < 6 * 64 and len(diff) == 64


@pytest.mark.parametrize("name", ["tiny", "flux"])
def test_stored_redraws_clear_every_near_tie(name):
    """Regenerate with the stored redraw map and recheck every gap with the oracle."""
    cfg = config(name)
    kk = oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
    table = load_redraws(name)
    heads = range(cfg.batch * cfg.heads) if name == "tiny" else [0, 7, 23]
    for bh in heads:
        q, k, v = (x.astype(np.float64) for x in generate_head(cfg, bh, table.get(bh)))
        r = oracle.pisa_head(q, k, v, cfg.block, kk, rows=[])
        top = np.sort(r["scores"], axis=1)[:, ::-1]
        assert (top[:, kk - 1] - top[:, kk]).min() >= MIN_GAP


def test_stored_redraws_match_a_fresh_search():
    cfg = config("flux")
    kk = oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
    pairs, gap = find_redraws(cfg, 11, kk)
    assert gap >= MIN_GAP
    assert dict(pairs) == load_redraws("flux").get(11, {})


def test_every_named_workload_has_a_redraw_entry():
    import json, os
    path = os.path.join(os.path.dirname(__file__), "golden", "tie_redraws.json")
    table = json.load(open(path))
    for name, cfg in CONFIGS.items():
        entry = table["configs"][name]
        assert entry["k"] == oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
        assert entry["min_gap_after"] >= MIN_GAP
