"""Brute-force dense softmax attention in float64 (test infrastructure only).

The operation PISA approximates (gist.science technical summary of PISA,
section 1 "Problem statement": full self-attention over L tokens, O(L^2)).
Used only as an independent pin: with every KV block selected, or with keys
constant inside every block, PISA must reproduce it.
"""

from __future__ import annotations

import math

import numpy as np


def dense_attention(q, k, v, s=None, row_chunk=1024):
    """softmax(s Q K^T) V for one head, q,k: [L,d], v: [L,dv], float64.

    Written as an explicit max-shifted exponential and row sums, one chunk of
    query rows at a time; no online accumulation.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if s is None:
        s = 1.0 / math.sqrt(q.shape[1])
    out = np.zeros((q.shape[0], v.shape[1]))
    for a in range(0, q.shape[0], row_chunk):
        logits = s * (q[a:a + row_chunk] @ k.T)
        logits -= logits.max(axis=1, keepdims=True)
        w = np.exp(logits)
        out[a:a + row_chunk] = (w @ v) / w.sum(axis=1, keepdims=True)
    return out
