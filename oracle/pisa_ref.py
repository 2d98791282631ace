"""fp64 CPU oracle of the PISA piecewise sparse attention forward pass.

Test infrastructure only (see the package docstring): plain NumPy in float64,
one (batch, head) at a time, one query block at a time, written to be checked
against the pages by eye.  A NumPy matmul is the only library primitive used
as a step; there is no blocking, fusion or reordering beyond what the
definitions below state.

Notation follows the gist.science technical summary of PISA (section 2,
"Method"): Q, K, V are cut into blocks of size B; for query block i the KV
blocks split into the selected set S_i and the unselected set U_i; the output
row is o_t = N_t / D_t.
"""

from __future__ import annotations

import math

import numpy as np


def block_bounds(L: int, B: int):
    """Token ranges T_j = [j*B, min((j+1)*B, L)) of the nb = ceil(L/B) blocks.

    Queries and keys use the same partition (AI Radio summary: "partition
    everything into blocks of size B").  The last block may be partial
    (reading R12: it keeps its true size n_j).
    """
    if L < 1 or B < 1:
        raise ValueError("L and B must be positive")
    nb = -(-L // B)
    starts = np.arange(nb, dtype=np.int64) * B
    ends = np.minimum(starts + B, L)
    return starts, ends


def keep_count(L: int, B: int, keep_ratio: float) -> int:
    """Number k of exactly computed KV blocks per query block (reading R9).

    k = clamp(ceil(rho * nb - 1e-9), 1, nb).  rho travels through the C ABI as
    a 32-bit float, so it is rounded to float32 first and the product is taken
    in float64.
    """
    nb = -(-L // B)
    rho = float(np.float32(keep_ratio))
    k = math.ceil(rho * nb - 1e-9)
    return int(min(max(k, 1), nb))


def block_stats(q: np.ndarray, k: np.ndarray, v: np.ndarray, B: int):
    """Per-block zeroth-order statistics (gist.science summary, section 2,
    hardware implementation: "precompute" of block centroids and value sums).

    Returns qbar [nb,d] (mean query of each block, reading R8), kbar [nb,d]
    (key centroid kbar_j), vsum [nb,d] (value sum sigma_j = sum_n v_{j,n}) and
    n [nb] (block sizes n_j), all float64.
    """
    L = q.shape[0]
    starts, ends = block_bounds(L, B)
    nb = len(starts)
    d = q.shape[1]
    dv = v.shape[1]
    qbar = np.zeros((nb, d))
    kbar = np.zeros((nb, d))
    vsum = np.zeros((nb, dv))
    n = (ends - starts).astype(np.float64)
    for j in range(nb):
        a, b = starts[j], ends[j]
        qbar[j] = q[a:b].sum(axis=0) / (b - a)
        kbar[j] = k[a:b].sum(axis=0) / (b - a)
        vsum[j] = v[a:b].sum(axis=0)
    return qbar, kbar, vsum, n


def first_order_blocks(k: np.ndarray, v: np.ndarray, B: int, kbar: np.ndarray) -> np.ndarray:
    """Block-wise first-order matrices H_j (reading R3), shape [nb, d_k, d_v].

    First-order Taylor expansion of exp(s q k_n) around the centroid kbar_j
    gives exp(s q kbar_j) (1 + s q (k_n - kbar_j)); summed against v_n its
    first-order coefficient is H_j = sum_{n in T_j} (k_n - kbar_j)^T v_n.  The
    keys are centred explicitly here (the CUDA path uses a different, algebraically
    equal form).
    """
    starts, ends = block_bounds(k.shape[0], B)
    nb = len(starts)
    H = np.zeros((nb, k.shape[1], v.shape[1]))
    for j in range(nb):
        a, b = starts[j], ends[j]
        centred = k[a:b] - kbar[j][None, :]
        H[j] = centred.T @ v[a:b]
    return H


def hbar_mean(H: np.ndarray) -> np.ndarray:
    """Global first-order statistic Hbar: the mean of the block-wise first-order
    matrices over all blocks of the head (gist.science summary, section 2,
    core algorithm, "hybrid-order approximation"; reading R4)."""
    return H.sum(axis=0) / H.shape[0]


def cov_norm(H: np.ndarray, Hbar: np.ndarray) -> np.ndarray:
    """M_j = ||H_j - Hbar|| (gist.science summary, section 2, covariance-aware
    routing), with the Frobenius norm (reading R6)."""
    diff = H - Hbar[None, :, :]
    return np.sqrt((diff * diff).sum(axis=(1, 2)))


def cov_norm_spectral(H: np.ndarray, Hbar: np.ndarray) -> np.ndarray:
    """M_j = ||H_j - Hbar||_2 read as the spectral norm (largest singular
    value): the other reading of the matrix 2-norm in the covariance-aware
    routing paragraph (gist.science summary, section 2).  A variant of reading
    R6, not the default."""
    diff = H - Hbar[None, :, :]
    return np.linalg.norm(diff, ord=2, axis=(1, 2))


def route_scores_pooled(qbar: np.ndarray, kbar: np.ndarray, n: np.ndarray, s: float) -> np.ndarray:
    """Routing score without the covariance term: s qbar_i . kbar_j + ln n_j,
    the log of the block's zeroth-order softmax mass (the attention part of
    Score_{t,j} alone; a variant of reading R7, plain pooled block-sparse
    routing)."""
    att = s * (qbar @ kbar.T)
    return att + np.log(n)[None, :]


def route_scores(qbar: np.ndarray, kbar: np.ndarray, M: np.ndarray, n: np.ndarray, s: float) -> np.ndarray:
    """Routing score of KV block j for query block i (reading R7).

    score_{i,j} = s qbar_i . kbar_j + ln(n_j + s ||qbar_i||_2 M_j): the log of
    the block's zeroth-order softmax mass times (its size plus the
    Cauchy-Schwarz bound on the first-order error that Hbar leaves).  Combines
    the attention score with the covariance norm, as the AI Radio summary and
    the gist.science routing paragraph say Score_{t,j} does.
    """
    qnorm = np.sqrt((qbar * qbar).sum(axis=1))
    att = s * (qbar @ kbar.T)
    return att + np.log(n[None, :] + s * qnorm[:, None] * M[None, :])


def select_topk(scores: np.ndarray, kk: int) -> np.ndarray:
    """S_i = indices of the kk largest scores of row i, ties to the smaller
    index (reading R10), returned in ascending index order.  Shape [nb, kk]."""
    nb_q, nb = scores.shape
    if not 1 <= kk <= nb:
        raise ValueError("need 1 <= k <= nb")
    sel = np.zeros((nb_q, kk), dtype=np.int64)
    idx = np.arange(nb)
    for i in range(nb_q):
        order = np.lexsort((idx, -scores[i]))
        sel[i] = np.sort(order[:kk])
    return sel


def pisa_rows(q, k, v, B, sel, kbar, vsum, n, Hbar, rows, s, return_parts=False, H_blocks=None):
    """Output rows o_t = N_t / D_t for the query tokens ``rows`` (gist.science
    summary, section 2, core algorithm).

    With ``H_blocks`` (the [nb, d, d] block-wise matrices H_j) the first-order
    term is the un-hybridised one the summary's hybrid-order paragraph starts
    from: every unselected block keeps its own H_j,
      N_t = ... + s sum_{j in U} e^{y_{t,j}} (q_t H_j)
    instead of s beta_t (q_t Hbar) (a variant for the accuracy / cost
    comparison; it costs |U| d^2 per query row).

    For t in query block i (S = S_i, U = U_i the complement):
      x_{t,n} = s q_t . k_n      for every token n of every block in S
      y_{t,j} = s q_t . kbar_j   for j in U        (alpha_{t,j} = e^{y_{t,j}})
      N_t = sum_n e^{x} v_n + sum_{j in U} e^{y} sigma_j + s beta_t (q_t Hbar)
      D_t = sum_n e^{x}     + sum_{j in U} e^{y} n_j
      beta_t = sum_{j in U} e^{y}                   (reading R5)
    Every exponential is taken relative to m_t = max(x, y); the shift cancels
    in N_t / D_t.
    """
    L = q.shape[0]
    starts, ends = block_bounds(L, B)
    nb = len(starts)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(rows), v.shape[1]))
    D_all = np.zeros(len(rows))
    exact_all = np.zeros(len(rows))
    blocks_of_rows = rows // B
    for i in np.unique(blocks_of_rows):
        pick = np.nonzero(blocks_of_rows == i)[0]
        S = np.asarray(sel[i], dtype=np.int64)
        U = np.setdiff1d(np.arange(nb), S)
        cols = np.concatenate([np.arange(starts[j], ends[j]) for j in S])
        qi = q[rows[pick]]
        x = s * (qi @ k[cols].T)
        y = s * (qi @ kbar[U].T)
        m = x.max(axis=1)
        if len(U):
            m = np.maximum(m, y.max(axis=1))
        ex = np.exp(x - m[:, None])
        ey = np.exp(y - m[:, None])
        exact_den = ex.sum(axis=1)
        D = exact_den + ey @ n[U]
        beta = ey.sum(axis=1)
        if H_blocks is None:
            first = s * beta[:, None] * (qi @ Hbar)
        else:
            first = np.zeros((len(pick), v.shape[1]))
            for c, j in enumerate(U):
                first += ey[:, c:c + 1] * (qi @ H_blocks[j])
            first *= s
        N = ex @ v[cols] + ey @ vsum[U] + first
        if not np.all(D > 0):
            raise AssertionError("D_t must be positive")
        out[pick] = N / D[:, None]
        D_all[pick] = D
        exact_all[pick] = exact_den
    if return_parts:
        return out, D_all, exact_all
    return out


def pisa_head(q, k, v, B, kk, s=None, rows=None, norm="frobenius", route="covariance",
              first_order="hybrid"):
    """The whole method on one (batch, head): stats, Hbar, M, scores, S, output.

    q, k, v: [L, d] arrays (promoted to float64).  ``rows`` limits the output
    to the given query tokens (all rows when None).  Returns a dict of every
    intermediate so that each stage can be compared on its own.

    Variants (defaults are readings R6, R7 and the pages' hybrid term):
    ``norm`` "frobenius" or "spectral" for M_j; ``route`` "covariance" or
    "pooled" (no M term); ``first_order`` "hybrid" (Hbar) or "blockwise"
    (each unselected block's own H_j).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, d = q.shape
    if s is None:
        s = 1.0 / math.sqrt(d)
    qbar, kbar, vsum, n = block_stats(q, k, v, B)
    H = first_order_blocks(k, v, B, kbar)
    Hbar = hbar_mean(H)
    if norm == "frobenius":
        M = cov_norm(H, Hbar)
    elif norm == "spectral":
        M = cov_norm_spectral(H, Hbar)
    else:
        raise ValueError(norm)
    if route == "covariance":
        scores = route_scores(qbar, kbar, M, n, s)
    elif route == "pooled":
        scores = route_scores_pooled(qbar, kbar, n, s)
    else:
        raise ValueError(route)
    sel = select_topk(scores, kk)
    if rows is None:
        rows = np.arange(L)
    if first_order not in ("hybrid", "blockwise"):
        raise ValueError(first_order)
    out = pisa_rows(q, k, v, B, sel, kbar, vsum, n, Hbar, rows, s,
                    H_blocks=H if first_order == "blockwise" else None)
    return dict(out=out, sel=sel, qbar=qbar, kbar=kbar, vsum=vsum, n=n,
                H=H, Hbar=Hbar, M=M, scores=scores, s=s)


def pisa_attention(q, k, v, B, kk):
    """PISA forward over [batch, heads, L, d] inputs; returns (out, sel)."""
    q = np.asarray(q)
    b, h, L, d = q.shape
    nb = -(-L // B)
    out = np.zeros((b, h, L, v.shape[-1]))
    sel = np.zeros((b, h, nb, kk), dtype=np.int64)
    for bi in range(b):
        for hi in range(h):
            r = pisa_head(q[bi, hi], k[bi, hi], v[bi, hi], B, kk)
            out[bi, hi] = r["out"]
            sel[bi, hi] = r["sel"]
    return out, sel
