"""Routing top-k on scores whose order is known exactly.

With M = 0, full blocks and small integers in two coordinates of the pooled
queries and key centroids (qbar_i = (a_i, b_i, 0, ...), kbar_j = (v_j, w_j,
0, ...)), every routing score is s (a_i v_j + b_i w_j) + ln B (AI Radio
summary of PISA, Score_{t,j}; gist.science summary, section 2, covariance-
aware routing).  The products are exact in the kernel's bf16 hi + lo split
and in fp32, so equal integer products give bitwise equal scores (exact
ties), and distinct ones differ by at least s, far above the fp32 rounding of
the score.  The selection is therefore known without the oracle: the k
largest a_i v_j + b_i w_j, exact ties to the smaller j, in ascending order (a
plain sort).

The key sets reach every top-k path of the library: 4, 8, 20 and 32 key
registers per lane (bitwise search below 16, interpolation search from 16
up), the shared-memory search past 1024 blocks and the CUDA-core routing
kernel past what the tensor-core kernel's shared memory holds.  They carry
many exact ties (values in -2..2), heavy tails (magnitudes spread over three
and a half decades, so the keys span many exponents), negative scores, k
from one block to all but one, and rows whose scores are all equal.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

D, B, HEADS = 128, 128, 2

# (nb, k, kind of key values, seed)
CASES = [
    (100, 7, "ties", 1),       # 4 key registers per lane
    (250, 25, "heavy", 2),     # 8
    (600, 60, "ties", 3),      # 20: interpolation search
    (600, 60, "heavy", 4),
    (600, 300, "mixed", 5),
    (640, 1, "heavy", 6),
    (900, 75, "heavy", 7),     # 32
    (900, 899, "ties", 8),
    (1300, 100, "heavy", 9),   # > 1024 blocks: keys searched in shared memory
    (2600, 50, "mixed", 10),   # CUDA-core routing kernel
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def _keys(nb, kind, rng):
    if kind == "ties":
        return rng.integers(-2, 3, nb), rng.integers(-2, 3, nb)
    if kind == "heavy":
        v = rng.choice([-1, 1], nb) * np.round(10.0 ** rng.uniform(0.0, 3.6, nb)).astype(np.int64)
        return v, rng.integers(-50, 51, nb)
    v1, w1 = _keys(nb // 2, "ties", rng)
    v2, w2 = _keys(nb - nb // 2, "heavy", rng)
    perm = rng.permutation(nb)
    return np.concatenate([v1, v2])[perm], np.concatenate([w1, w2])[perm]


def _expected(a, b, v, w, k):
    """Per row: the k largest a v_j + b w_j, ties to the smaller j, ascending."""
    nb = len(v)
    j = np.arange(nb)
    out = np.empty((len(a), k), dtype=np.int64)
    for i in range(len(a)):
        prod = a[i] * v + b[i] * w
        order = np.lexsort((j, -prod))  # by -prod, then by j
        out[i] = np.sort(order[:k])
    return out


@pytest.mark.parametrize("nb,k,kind,seed", CASES, ids=lambda c: str(c))
def test_topk_matches_exact_order(lib, nb, k, kind, seed):
    rng = np.random.default_rng(seed)
    qbar = np.zeros((1, HEADS, nb, D), np.float32)
    kbar = np.zeros((1, HEADS, nb, D), np.float32)
    expect = []
    for h in range(HEADS):
        a = rng.integers(-3, 4, nb)
        b = rng.integers(-3, 4, nb)
        a[0] = b[0] = 0  # a row whose scores are all equal: S_0 = 0 .. k-1
        v, w = _keys(nb, kind, rng)
        assert np.abs(v).max() < 2 ** 12 and np.abs(w).max() < 2 ** 12
        qbar[0, h, :, 0], qbar[0, h, :, 1] = a, b
        kbar[0, h, :, 0], kbar[0, h, :, 1] = v, w
        expect.append(_expected(a, b, v, w, k))
    dev = torch.device("cuda", 0)
    q_d, k_d = torch.from_numpy(qbar).to(dev), torch.from_numpy(kbar).to(dev)
    m_d = torch.zeros(1, HEADS, nb, dtype=torch.float32, device=dev)
    for route in ("covariance", "pooled"):
        if route == "covariance":
            sel = lib.select(q_d, k_d, m_d, nb * B, B, k)
        else:
            sel = lib.select_route(q_d, k_d, None, nb * B, B, k, route="pooled")
        torch.cuda.synchronize()
        assert lib.device_status() == lib.PISA_OK
        got = sel.cpu().numpy()
        for h in range(HEADS):
            bad = np.nonzero((got[0, h] != expect[h]).any(axis=1))[0]
            assert bad.size == 0, (
                f"{route}, head {h}: {bad.size} rows differ, first row {bad[0]}: "
                f"got {got[0, h, bad[0]].tolist()[:12]} expected {expect[h][bad[0]].tolist()[:12]}")
