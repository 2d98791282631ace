"""Test infrastructure: the fp64 CPU oracle of PISA's piecewise sparse attention.

This package is NOT part of the product path.  Only the test-suite, the smoke
check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import
it.  It shares no code with the CUDA library (no kernels, headers, helpers,
tables or pre/post-processing) and imports nothing from it.

Sources (all restated from the pages, never copied):

* "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
  Transformers" - gist.science technical summary (Japanese), section 2
  "Method": core algorithm (the N_t equation and the definition of alpha_{t,j}),
  covariance-aware routing (M_j = ||H_j - Hbar||), hardware implementation
  (precompute of centroids, value sums and Hbar).
* The same paper, AI Radio episode summary: S_i / U_i split per query block;
  Hbar shared by all unselected blocks through one scale factor beta_t; a
  routing score Score_{t,j}.

Readings where the pages are silent (each listed in the design notes):
R1 softmax scale s = 1/sqrt(d) inside every exponent and in the first-order
term; R2 D_t = exact part + sum_U n_j alpha (the first-order part of D vanishes
around the centroid); R3 H_j = sum_n (k_n - kbar_j)^T v_n (a sum, d_k x d_v);
R4 Hbar = plain mean of H_j over all blocks of a (batch, head); R5 beta_t =
sum_{j in U_i} alpha_{t,j}; R6 ||.|| is the Frobenius norm; R7 score_{i,j} =
s qbar_i.kbar_j + ln(n_j + s ||qbar_i|| M_j); R8 queries pooled by block mean;
R9 k = clamp(ceil(rho nb - 1e-9), 1, nb); R10 ties to the smaller index, no
forced block; R11 non-causal; R12 true counts n_j for a partial tail block.

Variants of three readings, kept beside the defaults for comparison: the
spectral norm for M_j (R6), the pooled score without the covariance term
(R7), and the un-hybridised first-order term with each unselected block's own
H_j (the summary's starting point before Hbar).

The pages print neither the routing score nor the matrix norm, so R6 and R7
are readings, not formulas taken from the pages.  Each function that
implements them is pinned to the reading's own derivation: the score equals
the log of alpha n_j plus the first-order error bound alpha ||s qbar_i (H_j -
Hbar)|| wherever Cauchy-Schwarz is tight (rank-one deviations with qbar_i
parallel to them), the ranking is monotone in M_j at equal centroids, V = 0
reduces it to pooled block-sparse routing, and M_j meets closed forms.
"""

from .pisa_ref import (  # noqa: F401
    block_bounds,
    keep_count,
    block_stats,
    first_order_blocks,
    hbar_mean,
    cov_norm,
    cov_norm_spectral,
    route_scores,
    route_scores_pooled,
    select_topk,
    pisa_rows,
    pisa_head,
    pisa_attention,
)
from .dense_ref import dense_attention  # noqa: F401
