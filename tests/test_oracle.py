"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these retypes the oracle's formula: each checks it against an
independent definition (brute-force dense attention, pure-Python sorting),
a closed form, an invariance, or a convergence rate.  Every pin is built so a
plausible slip (a dropped term, a wrong sign, index or scale, a transposed
operand) fails at least one test.
"""

import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(12345)


def _rand(L, d, scale=1.0, rng=RNG):
    return scale * rng.standard_normal((L, d))


# ---------------------------------------------------------------- special cases


@pytest.mark.parametrize("L,B,d", [(1000, 128, 64), (300, 64, 32), (257, 16, 8), (64, 64, 16)])
def test_every_block_selected_equals_dense(L, B, d):
    """k = nb (no unselected block): PISA is plain softmax attention."""
    rng = np.random.default_rng(L + B + d)
    q, k, v = _rand(L, d, 1.0, rng), _rand(L, d, 1.0, rng), _rand(L, d, 1.0, rng)
    nb = -(-L // B)
    r = oracle.pisa_head(q, k, v, B, nb)
    ref = oracle.dense_attention(q, k, v)
    err = np.abs(r["out"] - ref).max() / np.abs(ref).max()
    assert err < 1e-12


def test_single_block_equals_dense():
    """L <= B: one block, k = 1."""
    q, k, v = _rand(50, 16), _rand(50, 16), _rand(50, 16)
    r = oracle.pisa_head(q, k, v, 64, 1)
    assert r["sel"].shape == (1, 1)
    np.testing.assert_allclose(r["out"], oracle.dense_attention(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("kk", [1, 2, 5])
@pytest.mark.parametrize("L,B", [(256, 32), (250, 32)])
def test_constant_keys_per_block_exact_for_any_k(L, B, kk):
    """Keys constant inside every block: H_j = 0, and the zeroth-order term is
    exact, so PISA equals dense attention whatever the selection."""
    rng = np.random.default_rng(7 * L + kk)
    d = 16
    nb = -(-L // B)
    centres = rng.standard_normal((nb, d)) * 2.0
    k = centres[np.arange(L) // B]
    q, v = rng.standard_normal((L, d)) * 2.0, rng.standard_normal((L, d))
    r = oracle.pisa_head(q, k, v, B, kk)
    assert np.abs(r["H"]).max() < 1e-12
    np.testing.assert_allclose(r["out"], oracle.dense_attention(q, k, v), rtol=0, atol=1e-12)


def test_zeroth_order_exact_on_a_constant_key_block():
    """For one block whose keys all equal kbar_j: sum_n e^{s q k_n} v_n =
    alpha * sigma_j and sum_n e^{s q k_n} = n_j * alpha."""
    rng = np.random.default_rng(3)
    d, n = 16, 37
    s = 1 / math.sqrt(d)
    key = rng.standard_normal(d)
    kblock = np.tile(key, (n, 1))
    vblock = rng.standard_normal((n, d))
    q = rng.standard_normal(d)
    _, kbar, vsum, nn = oracle.block_stats(kblock, kblock, vblock, 64)
    alpha = math.exp(s * q @ kbar[0])
    exact_num = sum(math.exp(s * q @ kblock[t]) * vblock[t] for t in range(n))
    exact_den = sum(math.exp(s * q @ kblock[t]) for t in range(n))
    np.testing.assert_allclose(alpha * vsum[0], exact_num, rtol=1e-13)
    assert abs(nn[0] * alpha - exact_den) < 1e-12 * exact_den


# ---------------------------------------------------------------- invariants


def _case(L=600, B=64, d=32, seed=0):
    rng = np.random.default_rng(seed)
    pos = np.cumsum(rng.standard_normal((L, d)) * 0.15, axis=0)
    q = rng.standard_normal((L, d)) + pos
    k = rng.standard_normal((L, d)) + pos
    v = rng.standard_normal((L, d))
    return q, k, v


def test_denominator_positive_and_above_exact_part():
    q, k, v = _case()
    r = oracle.pisa_head(q, k, v, 64, 3)
    out, D, exact = oracle.pisa_rows(q, k, v, 64, r["sel"], r["kbar"], r["vsum"], r["n"],
                                     r["Hbar"], np.arange(q.shape[0]), r["s"], return_parts=True)
    assert np.all(D > 0)
    assert np.all(D >= exact)
    assert np.all(D > exact)  # every row has unselected blocks here


def test_value_shift_moves_output_by_the_shift():
    """o(V + 1c^T) = o(V) + c; H_j (hence M, S) is unchanged since the centred
    keys sum to zero."""
    q, k, v = _case(seed=1)
    c = np.linspace(-2, 3, v.shape[1])
    a = oracle.pisa_head(q, k, v, 64, 3)
    b = oracle.pisa_head(q, k, v + c[None, :], 64, 3)
    np.testing.assert_array_equal(a["sel"], b["sel"])
    np.testing.assert_allclose(b["H"], a["H"], rtol=0, atol=1e-9)
    np.testing.assert_allclose(b["out"], a["out"] + c[None, :], rtol=0, atol=1e-11)


def test_key_shift_leaves_output_unchanged():
    """o(K + 1c^T) = o(K): every exponent of a row moves by s q_t.c; routing
    scores move by a per-row constant."""
    q, k, v = _case(seed=2)
    c = np.linspace(1, -1, k.shape[1])
    a = oracle.pisa_head(q, k, v, 64, 3)
    b = oracle.pisa_head(q, k + c[None, :], v, 64, 3)
    np.testing.assert_array_equal(a["sel"], b["sel"])
    np.testing.assert_allclose(b["M"], a["M"], rtol=1e-12)
    diff = b["scores"] - a["scores"]
    np.testing.assert_allclose(diff, diff[:, :1] * np.ones_like(diff), rtol=0, atol=1e-10)
    np.testing.assert_allclose(b["out"], a["out"], rtol=0, atol=1e-11)


def test_permutation_inside_blocks_is_invisible():
    """Permuting tokens inside each block (same permutation for K and V) keeps
    kbar, sigma, H, M, S and the output."""
    q, k, v = _case(L=640, seed=3)
    B = 64
    rng = np.random.default_rng(9)
    perm = np.concatenate([j * B + rng.permutation(B) for j in range(640 // B)])
    a = oracle.pisa_head(q, k, v, B, 4)
    b = oracle.pisa_head(q, k[perm], v[perm], B, 4)
    np.testing.assert_array_equal(a["sel"], b["sel"])
    np.testing.assert_allclose(b["H"], a["H"], rtol=0, atol=1e-10)
    np.testing.assert_allclose(b["out"], a["out"], rtol=0, atol=1e-11)


# ---------------------------------------------------------------- first-order term


def _taylor_case(eps, shared, seed=4, L=96, B=12, d=8):
    """Keys k_n = c_j + eps*delta_{n mod B}.  With ``shared`` the values repeat
    the same pattern in every block, which makes every H_j equal to Hbar."""
    rng = np.random.default_rng(seed)
    nb = L // B
    centres = rng.standard_normal((nb, d)) * 1.5
    delta = rng.standard_normal((B, d))
    k = centres[np.arange(L) // B] + eps * delta[np.arange(L) % B]
    if shared:
        v = rng.standard_normal((B, d))[np.arange(L) % B]
    else:
        v = rng.standard_normal((L, d))
    q = rng.standard_normal((L, d)) * 1.5
    return q, k, v


def _pisa_fixed_sel(q, k, v, B, sel, zero_hbar=False):
    s = 1 / math.sqrt(q.shape[1])
    qbar, kbar, vsum, n = oracle.block_stats(q, k, v, B)
    H = oracle.first_order_blocks(k, v, B, kbar)
    Hbar = oracle.hbar_mean(H)
    if zero_hbar:
        Hbar = np.zeros_like(Hbar)
    return oracle.pisa_rows(q, k, v, B, sel, kbar, vsum, n, Hbar, np.arange(q.shape[0]), s)


def _slope(shared, zero_hbar):
    B = 12
    sel = np.array([[i, (i + 3) % 8] for i in range(8)])
    sel.sort(axis=1)
    eps = np.array([1e-1, 3e-2, 1e-2, 3e-3, 1e-3])
    errs = []
    for e in eps:
        q, k, v = _taylor_case(e, shared)
        errs.append(np.abs(_pisa_fixed_sel(q, k, v, B, sel, zero_hbar) - oracle.dense_attention(q, k, v)).max())
    return np.polyfit(np.log(eps), np.log(errs), 1)[0]


def test_first_order_term_is_second_order_exact_when_blocks_share_structure():
    """All H_j equal Hbar: the hybrid first-order term is the block's own
    first-order Taylor term, so the error is O(eps^2)."""
    assert _slope(shared=True, zero_hbar=False) == pytest.approx(2.0, abs=0.15)


def test_dropping_the_first_order_term_leaves_first_order_error():
    """Same inputs with Hbar removed (a planted slip): the error is O(eps)."""
    assert _slope(shared=True, zero_hbar=True) == pytest.approx(1.0, abs=0.15)


def test_hybrid_error_is_first_order_for_generic_blocks():
    """Different H_j per block: Hbar only captures their mean, error O(eps)."""
    assert _slope(shared=False, zero_hbar=False) == pytest.approx(1.0, abs=0.15)


def test_first_order_matrix_identity():
    """H_j = K_j^T V_j - n_j kbar_j^T vbar_j, and sum_j H_j = K^T V - sum_j n_j kbar_j^T vbar_j."""
    q, k, v = _case(L=650, seed=5)
    B = 64
    qbar, kbar, vsum, n = oracle.block_stats(q, k, v, B)
    H = oracle.first_order_blocks(k, v, B, kbar)
    total = np.zeros_like(H[0])
    for j in range(len(n)):
        a, b = j * B, min((j + 1) * B, 650)
        alt = k[a:b].T @ v[a:b] - np.outer(kbar[j], vsum[j])
        np.testing.assert_allclose(H[j], alt, rtol=0, atol=1e-10)
        total += np.outer(kbar[j], vsum[j])
    np.testing.assert_allclose(H.sum(axis=0), k.T @ v - total, rtol=0, atol=1e-9)
    np.testing.assert_allclose(oracle.hbar_mean(H), H.sum(axis=0) / len(n), rtol=1e-14)


# ---------------------------------------------------------------- routing


def test_covariance_norm_closed_form():
    """H_j = lambda_j * c * e_1 w^T (only coordinate 0 of the keys varies inside
    a block, values lambda_j delta_n w): M_j = |lambda_j - mean(lambda)| c ||w||."""
    rng = np.random.default_rng(6)
    B, nb, d = 16, 6, 8
    delta = rng.standard_normal(B)
    delta -= delta.mean()
    lam = rng.standard_normal(nb)
    w = rng.standard_normal(d)
    centres = rng.standard_normal((nb, d))
    k = np.zeros((nb * B, d))
    v = np.zeros((nb * B, d))
    for j in range(nb):
        k[j * B:(j + 1) * B] = centres[j]
        k[j * B:(j + 1) * B, 0] += delta
        v[j * B:(j + 1) * B] = lam[j] * delta[:, None] * w[None, :]
    _, kbar, _, _ = oracle.block_stats(k, k, v, B)
    H = oracle.first_order_blocks(k, v, B, kbar)
    M = oracle.cov_norm(H, oracle.hbar_mean(H))
    c = (delta ** 2).sum()
    np.testing.assert_allclose(M, np.abs(lam - lam.mean()) * c * np.linalg.norm(w), rtol=1e-12)


def _brute_topk_pooled(q, k, B, kk):
    """Pure-Python pooled block-sparse routing: block means, scaled dot plus
    ln(block size), full sort with ties to the smaller index."""
    L, d = len(q), len(q[0])
    nb = -(-L // B)
    s = 1 / math.sqrt(d)
    means = []
    for X in (q, k):
        mm = []
        for j in range(nb):
            rows = X[j * B:min((j + 1) * B, L)]
            mm.append([sum(r[a] for r in rows) / len(rows) for a in range(d)])
        means.append(mm)
    sizes = [min((j + 1) * B, L) - j * B for j in range(nb)]
    sel, gaps = [], []
    for i in range(nb):
        sc = [(s * sum(means[0][i][a] * means[1][j][a] for a in range(d)) + math.log(sizes[j]), j)
              for j in range(nb)]
        ranked = sorted(sc, key=lambda t: (-t[0], t[1]))
        sel.append(sorted(j for _, j in ranked[:kk]))
        if kk < nb:
            gaps.append(ranked[kk - 1][0] - ranked[kk][0])
    return sel, min(gaps)


@pytest.mark.parametrize("L,B,kk", [(500, 50, 3), (470, 50, 4), (256, 32, 1)])
def test_zero_values_reduce_routing_to_pooled_topk(L, B, kk):
    """V = 0: every H_j = 0, M = 0, and the score is textbook pooled block
    routing s qbar.kbar + ln n_j (brute force, pure Python)."""
    q, k, _ = _case(L=L, B=B, d=12, seed=L + kk)
    v = np.zeros_like(q)
    r = oracle.pisa_head(q, k, v, B, kk)
    assert np.abs(r["M"]).max() == 0.0
    sel, gap = _brute_topk_pooled(q.tolist(), k.tolist(), B, kk)
    assert gap > 1e-9
    np.testing.assert_array_equal(r["sel"], np.array(sel))


def test_topk_ties_go_to_the_smaller_index():
    scores = np.array([[1.0, 3.0, 3.0, 2.0, 3.0],
                       [0.0, 0.0, 0.0, 0.0, 0.0]])
    np.testing.assert_array_equal(oracle.select_topk(scores, 2), [[1, 2], [0, 1]])
    np.testing.assert_array_equal(oracle.select_topk(scores, 3), [[1, 2, 4], [0, 1, 2]])


def test_scores_reduce_to_pooled_when_covariance_norm_constant():
    """With M_j constant over j and full blocks, the ranking is the pooled one."""
    rng = np.random.default_rng(8)
    qbar, kbar = rng.standard_normal((10, 6)), rng.standard_normal((10, 6))
    n = np.full(10, 32.0)
    a = oracle.route_scores(qbar, kbar, np.full(10, 5.0), n, 0.4)
    b = 0.4 * qbar @ kbar.T
    np.testing.assert_array_equal(oracle.select_topk(a, 3), oracle.select_topk(b, 3))


def _aligned_rank_one_case(L=230, B=20, d=8, seed=41):
    """Raw Q, K, V whose block statistics are known in closed form.

    Keys k_n = c_j + a_n e (unit direction e, per-block centred scalars a_n),
    so kbar_j = c_j and H_j - Hbar = e (w_j - wbar)^T with w_j = sum_n a_n v_n
    (rank one).  Queries q_t = b_i e + r_t with per-block centred noise r_t,
    so qbar_i = b_i e is parallel to e.  The last block is partial (L is not
    a multiple of B), so n_j is not constant.  Returns q, k, v and the closed
    forms (b, c, w, n)."""
    rng = np.random.default_rng(seed)
    nb = -(-L // B)
    blk = np.arange(L) // B
    e = rng.standard_normal(d)
    e /= np.linalg.norm(e)

    def centred(x):
        x = x.copy()
        for j in range(nb):
            x[blk == j] -= x[blk == j].mean(axis=0)
        return x

    a = centred(rng.standard_normal(L))
    c = rng.standard_normal((nb, d))
    k = c[blk] + a[:, None] * e[None, :]
    v = rng.standard_normal((L, d))
    # |b_i| spread well away from 1, so a squared norm cannot pass for the norm
    b = rng.choice([-1.0, 1.0], nb) * rng.uniform(0.3, 3.0, nb)
    q = b[blk][:, None] * e[None, :] + centred(rng.standard_normal((L, d)))
    w = np.stack([(a[blk == j, None] * v[blk == j]).sum(axis=0) for j in range(nb)])
    n = np.bincount(blk).astype(np.float64)
    return q, k, v, (b, c, e, w, n)


def test_routing_score_is_the_tight_cauchy_schwarz_bound_on_rank_one_blocks():
    """Score_{i,j} (reading R7) from raw inputs, without the oracle's norm.

    The score is the log of block j's zeroth-order softmax mass alpha n_j plus
    the bound alpha ||s qbar_i (H_j - Hbar)|| on the first-order error that
    Hbar leaves in that block (gist.science summary, section 2,
    covariance-aware routing; AI Radio summary, Score_{t,j}).  When H_j - Hbar
    = e u_j^T and qbar_i is parallel to e, Cauchy-Schwarz is an equality:
    ||s qbar_i (H_j - Hbar)|| = s ||qbar_i|| ||H_j - Hbar||, so the score must
    equal ln(alpha_ij n_j + ||alpha_ij s qbar_i (H_j - Hbar)||) with
    alpha_ij = exp(s qbar_i . kbar_j), every factor taken from the
    construction.  A dropped s, a squared query norm, or the log split as
    ln n_j + s||qbar||M_j each fail this."""
    L, B, d = 230, 20, 8
    q, k, v, (b, c, e, w, n) = _aligned_rank_one_case(L, B, d)
    s = 1.0 / math.sqrt(d)
    r = oracle.pisa_head(q, k, v, B, 3)
    np.testing.assert_allclose(r["kbar"], c, atol=1e-12)
    np.testing.assert_allclose(r["qbar"], b[:, None] * e[None, :], atol=1e-12)
    u = w - w.mean(axis=0)  # H_j - Hbar = e u_j^T
    qbar = b[:, None] * e[None, :]
    for i in range(len(b)):
        for j in range(len(n)):
            alpha = math.exp(s * float(qbar[i] @ c[j]))
            err_vec = s * (qbar[i] @ np.outer(e, u[j]))  # s qbar_i (H_j - Hbar), a d-vector
            want = math.log(alpha * n[j] + alpha * float(np.linalg.norm(err_vec)))
            assert abs(r["scores"][i, j] - want) <= 1e-12 * max(1.0, abs(want)), (i, j)
    # the construction really exercises the covariance term: it moves the
    # scores by far more than the tolerance, and n_j differs on the tail
    assert np.abs(r["scores"] - (s * qbar @ c.T + np.log(n)[None, :])).max() > 0.1
    assert n[-1] != n[0]


def test_routing_ranks_blocks_by_covariance_norm_at_equal_centroids():
    """Monotone in M_j: blocks with the same centroid and size differ only in
    their covariance norm, and for any query block with qbar_i != 0 the block
    with the larger M_j scores higher (the error bound grows with it).

    Block j's keys are the centroid plus a shared centred pattern scaled by
    t_j = 2^j, with the same values in every block, so H_j = t_j H_0, Hbar =
    mean(t) H_0 and M_j = |t_j - mean(t)| ||H_0||_F (closed form).  With
    mean(t) = 127/7 the order of M is 6, 0, 1, 2, 5, 3, 4: every score row
    must follow it, and the top 3 are blocks {0, 1, 6}."""
    rng = np.random.default_rng(44)
    nb, B, d = 7, 16, 6
    L = nb * B
    blk = np.arange(L) // B
    base = rng.standard_normal((B, d))
    base -= base.mean(axis=0)
    centroid = rng.standard_normal(d)
    vb = rng.standard_normal((B, d))
    v = np.tile(vb, (nb, 1))
    t = 2.0 ** np.arange(nb)
    k = centroid[None, :] + base[np.arange(L) % B] * t[blk][:, None]
    q = rng.standard_normal((L, d)) + 0.5
    r = oracle.pisa_head(q, k, v, B, 3)
    np.testing.assert_allclose(r["kbar"], np.tile(centroid, (nb, 1)), atol=1e-12)
    want_M = np.abs(t - t.mean()) * np.linalg.norm(base.T @ vb)
    np.testing.assert_allclose(r["M"], want_M, rtol=1e-10)
    order = np.argsort(-want_M)
    assert order.tolist() == [6, 0, 1, 2, 5, 3, 4]
    for i in range(nb):
        assert np.all(np.diff(r["scores"][i, order]) < 0), i
    np.testing.assert_array_equal(r["sel"], np.tile([0, 1, 6], (nb, 1)))


def test_keep_count_on_the_workloads():
    assert oracle.keep_count(1024, 64, 4 / 16) == 4
    assert oracle.keep_count(4608, 64, 0.25) == 18
    assert oracle.keep_count(32760, 128, 0.15) == 39
    assert oracle.keep_count(75600, 128, 0.10) == 60
    assert oracle.keep_count(119040, 128, 0.08) == 75
    assert oracle.keep_count(100, 128, 0.01) == 1
    assert oracle.keep_count(1000, 100, 1.0) == 10


def test_block_bounds_partial_tail():
    s, e = oracle.block_bounds(300, 128)
    assert s.tolist() == [0, 128, 256] and e.tolist() == [128, 256, 300]


# ---------------------------------------------------------------- variants of the readings


def _rank_one_case(L=200, B=20, d=8, seed=9):
    """Keys k_n = c_j + a_n e with one unit direction e and per-block centred
    scalars a_n: every H_j - Hbar is then e (w_j - wbar)^T, of rank one, with
    w_j = sum_n a_n v_n."""
    rng = np.random.default_rng(seed)
    nb = L // B
    e = rng.standard_normal(d)
    e /= np.linalg.norm(e)
    a = rng.standard_normal(L)
    for j in range(nb):
        a[j * B:(j + 1) * B] -= a[j * B:(j + 1) * B].mean()
    k = rng.standard_normal((nb, d))[np.arange(L) // B] + a[:, None] * e[None, :]
    v = rng.standard_normal((L, d))
    w = np.stack([(a[j * B:(j + 1) * B, None] * v[j * B:(j + 1) * B]).sum(axis=0) for j in range(nb)])
    return k, v, w


def test_spectral_norm_of_rank_one_deviations_is_their_vector_norm():
    """Rank-one H_j - Hbar: spectral norm = Frobenius norm = ||w_j - wbar||."""
    k, v, w = _rank_one_case()
    B = 20
    kbar = oracle.block_stats(k, k, v, B)[1]
    H = oracle.first_order_blocks(k, v, B, kbar)
    Hbar = oracle.hbar_mean(H)
    want = np.linalg.norm(w - w.mean(axis=0), axis=1)
    np.testing.assert_allclose(oracle.cov_norm_spectral(H, Hbar), want, rtol=1e-10)
    np.testing.assert_allclose(oracle.cov_norm(H, Hbar), want, rtol=1e-10)


def test_spectral_norm_bounds_for_generic_blocks():
    """||A||_2 <= ||A||_F <= sqrt(rank) ||A||_2, and ||A||_2 >= the largest
    column norm of A (A e_c for a unit vector e_c)."""
    rng = np.random.default_rng(21)
    q, k, v = rng.standard_normal((3, 240, 12))
    B = 24
    kbar = oracle.block_stats(q, k, v, B)[1]
    H = oracle.first_order_blocks(k, v, B, kbar)
    Hbar = oracle.hbar_mean(H)
    spec, frob = oracle.cov_norm_spectral(H, Hbar), oracle.cov_norm(H, Hbar)
    assert (spec <= frob * (1 + 1e-12)).all()
    assert (frob <= math.sqrt(12) * spec * (1 + 1e-12)).all()
    col = np.sqrt(((H - Hbar) ** 2).sum(axis=1)).max(axis=1)
    assert (spec >= col * (1 - 1e-12)).all()
    assert (spec < frob).any()  # not the Frobenius norm again


@pytest.mark.parametrize("L,B,kk", [(500, 50, 3), (256, 32, 1)])
def test_pooled_routing_is_brute_force_top_k(L, B, kk):
    """Pooled score s qbar.kbar + ln n_j, selection checked against a pure
    Python sort; with V = 0 (M = 0) the covariance score equals it."""
    rng = np.random.default_rng(L + kk)
    q, k = rng.standard_normal((2, L, 16))
    s = 0.25
    qbar, kbar, _, n = oracle.block_stats(q, k, k, B)
    sc = oracle.route_scores_pooled(qbar, kbar, n, s)
    sel = oracle.select_topk(sc, kk)
    for i in range(len(qbar)):
        pairs = [(-(s * sum(qbar[i][a] * kbar[j][a] for a in range(16)) + math.log(n[j])), j)
                 for j in range(len(kbar))]
        assert sorted(j for _, j in sorted(pairs)[:kk]) == list(sel[i])
    zeros = np.zeros((len(kbar),))
    np.testing.assert_allclose(oracle.route_scores(qbar, kbar, zeros, n, s), sc, rtol=0, atol=1e-12)


def _blockwise_slope(shared):
    B = 12
    sel = np.array([[i, (i + 3) % 8] for i in range(8)])
    sel.sort(axis=1)
    eps = np.array([1e-1, 3e-2, 1e-2, 3e-3, 1e-3])
    errs = []
    for e in eps:
        q, k, v = _taylor_case(e, shared)
        s = 1 / math.sqrt(q.shape[1])
        qbar, kbar, vsum, n = oracle.block_stats(q, k, v, B)
        H = oracle.first_order_blocks(k, v, B, kbar)
        o = oracle.pisa_rows(q, k, v, B, sel, kbar, vsum, n, oracle.hbar_mean(H), np.arange(q.shape[0]), s,
                             H_blocks=H)
        errs.append(np.abs(o - oracle.dense_attention(q, k, v)).max())
    return np.polyfit(np.log(eps), np.log(errs), 1)[0]


def test_blockwise_first_order_is_second_order_for_generic_blocks():
    """Each unselected block keeps its own H_j: a true first-order Taylor
    expansion per block, so the error is O(eps^2) even when the H_j differ
    (where the hybrid Hbar term is only O(eps))."""
    assert _blockwise_slope(shared=False) == pytest.approx(2.0, abs=0.15)


def test_blockwise_equals_hybrid_when_every_block_shares_hbar():
    q, k, v = _taylor_case(1e-2, shared=True)
    B = 12
    s = 1 / math.sqrt(q.shape[1])
    sel = np.sort(np.array([[i, (i + 5) % 8] for i in range(8)]), axis=1)
    qbar, kbar, vsum, n = oracle.block_stats(q, k, v, B)
    H = oracle.first_order_blocks(k, v, B, kbar)
    Hbar = oracle.hbar_mean(H)
    rows = np.arange(q.shape[0])
    a = oracle.pisa_rows(q, k, v, B, sel, kbar, vsum, n, Hbar, rows, s)
    b = oracle.pisa_rows(q, k, v, B, sel, kbar, vsum, n, Hbar, rows, s, H_blocks=H)
    np.testing.assert_allclose(b, a, rtol=0, atol=1e-12)


def test_head_variants_run_and_differ_only_where_expected():
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((3, 300, 16))
    base = oracle.pisa_head(q, k, v, 30, 3)
    spec = oracle.pisa_head(q, k, v, 30, 3, norm="spectral")
    pooled = oracle.pisa_head(q, k, v, 30, 3, route="pooled")
    block = oracle.pisa_head(q, k, v, 30, 3, first_order="blockwise")
    np.testing.assert_array_equal(block["sel"], base["sel"])          # routing untouched
    assert not np.allclose(block["out"], base["out"])                # first-order term changed
    assert (spec["M"] <= base["M"] * (1 + 1e-12)).all()
    np.testing.assert_allclose(pooled["M"], base["M"])                # M computed, not used
    with pytest.raises(ValueError):
        oracle.pisa_head(q, k, v, 30, 3, norm="nuclear")
