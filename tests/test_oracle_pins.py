"""Pins of the fp64 oracle against facts the paper or mathematics fix.

Each test checks an oracle step against something other than itself: values
printed in the paper (tests/golden), closed forms, invariants, brute force on
tiny inputs, or an independent library route.  No GPU is needed.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng0 = np.random.default_rng(12345)


def _rand(shape, seed=0, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ----------------------------------------------------------------- generator
def test_splitmix64_published_sequence():
    # Reference outputs of SplitMix64 seeded with 1234567 (Vigna's splitmix64.c
    # test sequence).
    got = O.splitmix64_outputs(1234567, 5)
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def test_kmeans_init_indices_range_and_streams():
    a = O.kmeans_init_indices(4, 0, 0, 1000, 75600)
    b = O.kmeans_init_indices(4, 0, 1, 1000, 75600)
    c = O.kmeans_init_indices(4, 1, 0, 1000, 75600)
    assert a.min() >= 0 and a.max() < 75600
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    # draw -> row: top 32 bits u give floor(u N / 2^32)
    x = O.splitmix64_mix(4 ^ O.splitmix64_mix(1 * 0x9E3779B97F4A7C15))
    first = O.splitmix64_outputs(x, 1)[0]
    assert a[0] == math.floor((first >> 32) * 75600 / 2**32)
    # uniform with replacement: roughly uniform over the rows
    big = O.kmeans_init_indices(7, 3, 0, 20000, 1000)
    counts = np.bincount(big, minlength=1000)
    assert counts.min() > 0 and counts.max() < 60


# ------------------------------------------------------- dense/sparse (§3)
def test_dense_attention_matches_library_sdpa():
    q, k, v = _rand((37, 16), 1), _rand((53, 16), 2), _rand((53, 16), 3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None])[0].numpy()
    np.testing.assert_allclose(O.dense_attention(q, k, v), ref, rtol=1e-12, atol=1e-12)


def test_sparse_attention_all_cells_is_dense():
    N, d = 64, 8
    q, k, v = _rand((N, d), 4, 1.5), _rand((N, d), 5, 1.5), _rand((N, d), 6)
    ql = np.arange(N) % 3
    kl = (np.arange(N) * 7) % 5
    mask = np.ones((3, 5), dtype=bool)
    np.testing.assert_allclose(O.sparse_attention(q, k, v, ql, kl, mask),
                               O.dense_attention(q, k, v), rtol=1e-12, atol=1e-12)


def test_sparse_attention_brute_force_and_residual_identity():
    """§3.1 hard-drop identity: O^dense - O^sp = p_U (O_U - O^sp), p_U the dense
    attention mass on the dropped keys and O_U the attention output over them."""
    N, d = 48, 8
    q, k, v = _rand((N, d), 7, 1.3), _rand((N, d), 8, 1.3), _rand((N, d), 9)
    ql = np.arange(N) % 4
    kl = np.arange(N) % 6
    mask = np.random.default_rng(3).random((4, 6)) < 0.5
    mask[:, 0] = True
    mask[:, 5] = False
    osp = O.sparse_attention(q, k, v, ql, kl, mask)
    od = O.dense_attention(q, k, v)
    for i in range(N):
        sel = mask[ql[i]][kl]
        logits = np.array([sum(q[i, t] * k[j, t] for t in range(d)) / math.sqrt(d) for j in range(N)])
        e = np.exp(logits - logits.max())
        p = e / e.sum()
        o_sel = (p[sel, None] * v[sel]).sum(0) / p[sel].sum()     # brute-force Eq. (2)
        np.testing.assert_allclose(osp[i], o_sel, rtol=1e-11, atol=1e-12)
        pU = p[~sel].sum()
        oU = (p[~sel, None] * v[~sel]).sum(0) / pU
        np.testing.assert_allclose(od[i] - osp[i], pU * (oU - osp[i]), rtol=1e-9, atol=1e-12)


def test_key_shift_leaves_attention_unchanged():
    """B.2: adding one vector to every key shifts each query's logits by a
    constant, which softmax ignores (dense and sparse)."""
    N, d = 40, 8
    q, k, v = _rand((N, d), 10), _rand((N, d), 11), _rand((N, d), 12)
    ql, kl = np.arange(N) % 2, np.arange(N) % 4
    mask = np.array([[1, 0, 1, 0], [0, 1, 1, 1]], dtype=bool)
    shift = _rand(d, 13, 3.0)
    np.testing.assert_allclose(O.dense_attention(q, k + shift, v), O.dense_attention(q, k, v),
                               rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(O.sparse_attention(q, k + shift, v, ql, kl, mask),
                               O.sparse_attention(q, k, v, ql, kl, mask), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------- partitioning (§4.1)
def test_sample_indices_evenly_spaced():
    assert list(O.sample_indices(10, 4)) == [0, 2, 5, 7]
    assert list(O.sample_indices(5, 9)) == [0, 1, 2, 3, 4]
    idx = O.sample_indices(75600, 1024)
    assert len(np.unique(idx)) == 1024 and idx[0] == 0 and idx[-1] == (1023 * 75600) // 1024


def test_key_coordinates_reproduce_response_metric():
    """§4.1: squared distances of phi_K are the mean squared logit differences
    over the sampled queries (full rank, scale 1/sqrt(d) per reading R2)."""
    N, d, Ms = 30, 6, 11
    q, k = _rand((N, d), 20), _rand((N, d), 21)
    idx = O.sample_indices(N, Ms)
    F = O.key_factor(O.key_metric(q, idx), d, len(idx))
    phi = k @ F
    for (j1, j2) in [(0, 1), (3, 17), (29, 5)]:
        resp = [sum(q[s, t] * (k[j1, t] - k[j2, t]) for t in range(d)) / math.sqrt(d) for s in idx]
        want = sum(x * x for x in resp) / len(idx)
        assert abs(((phi[j1] - phi[j2]) ** 2).sum() - want) < 1e-10 * max(1.0, want)


def test_key_factor_truncation_and_eigen_order():
    d = 8
    A = _rand((20, d), 22)
    M = A.T @ A / 20
    w, U = O.eigh_desc(M)
    assert np.all(np.diff(w) <= 0)
    np.testing.assert_allclose(U @ np.diag(w) @ U.T, M, atol=1e-12)
    F = O.key_factor(M, 3, 100)
    np.testing.assert_allclose(F @ F.T * d, U[:, :3] @ np.diag(w[:3]) @ U[:, :3].T, atol=1e-12)
    assert O.key_factor(M, 48, 5).shape[1] == 5        # r_K' = min(r_K, d, M_s)


def test_kmeans_assign_is_nearest_centre_brute_force():
    X, C = _rand((50, 5), 30), _rand((7, 5), 31)
    labels, _ = O.kmeans_assign(X, C)
    for i in range(50):
        dist = [sum((X[i, t] - C[c, t]) ** 2 for t in range(5)) for c in range(7)]
        assert labels[i] == int(np.argmin(dist))


def test_kmeans_assign_ties_go_to_lowest_index():
    X = _rand((20, 3), 32)
    C = np.stack([_rand(3, 33), _rand(3, 34), _rand(3, 33)])   # centre 2 duplicates centre 0
    labels, _ = O.kmeans_assign(X, C)
    assert not np.any(labels == 2)
    assert O.argmax_rows(np.array([[1.0, 3.0, 3.0], [2.0, 2.0, 0.0]])).tolist() == [1, 0]


def test_kmeans_objective_non_increasing_and_update_means():
    X = _rand((300, 4), 35)
    init = O.kmeans_init_indices(9, 0, 0, 12, 300)
    labels, centres, n_it, hist = O.kmeans(X, init, 25, 0)
    cen = X[init].copy()
    prev_obj = np.inf
    for t, lab in enumerate(hist):
        if t > 0:
            cen = O.kmeans_update(X, hist[t - 1], cen)
        obj = ((X - cen[lab]) ** 2).sum()
        assert obj <= prev_obj + 1e-9
        prev_obj = obj
    # update = member means (explicit loop)
    upd = O.kmeans_update(X, labels, centres)
    for c in range(12):
        mem = [i for i in range(300) if labels[i] == c]
        if mem:
            np.testing.assert_allclose(upd[c], np.mean(X[mem], axis=0), atol=1e-12)
        else:
            np.testing.assert_allclose(upd[c], centres[c])


def test_kmeans_recovers_separated_clusters_and_stop_rule():
    rng = np.random.default_rng(36)
    true = rng.integers(0, 4, 400)
    X = np.eye(4)[true] * 50.0 + rng.standard_normal((400, 4)) * 0.1
    init = np.array([int(np.nonzero(true == c)[0][0]) for c in range(4)])
    labels, _, n_it, _ = O.kmeans(X, init, 25, 0)
    assert np.array_equal(labels, true)
    assert n_it == 2                # second assignment changes nothing -> stop
    assert O.kmeans_stop_count(1e-4, 75600) == 7 and O.kmeans_stop_count(1e-4, 8192) == 0


def test_kmeans_labels_invariant_to_factor_sign_flips():
    N, d = 200, 8
    q, k = _rand((N, d), 37), _rand((N, d), 38)
    F = O.key_factor(O.key_metric(q, O.sample_indices(N, 64)), 4, 64)
    init = O.kmeans_init_indices(1, 0, 0, 9, N)
    l1 = O.kmeans(k @ F, init, 25, 0)[0]
    l2 = O.kmeans(k @ (F * np.array([1, -1, -1, 1])), init, 25, 0)[0]
    assert np.array_equal(l1, l2)


def test_compact_labels():
    lab = np.array([5, 2, 5, 7, 2, 2])
    new, C, sizes = O.compact_labels(lab, 9)
    assert new.tolist() == [1, 0, 1, 2, 0, 0] and C == 3 and sizes.tolist() == [3, 2, 1]


def test_query_metric_centring_and_rank():
    Kb = _rand((6, 5), 40)
    M1 = O.query_metric(Kb)
    np.testing.assert_allclose(O.query_metric(Kb + _rand(5, 41, 4.0)), M1, atol=1e-12)
    Kt = Kb - Kb.mean(0)
    np.testing.assert_allclose(M1, sum(np.outer(r, r) for r in Kt) / (6 * 5), atol=1e-12)
    assert np.linalg.matrix_rank(M1, tol=1e-10) <= 5
    assert O.query_rank(64, 128, 1000) == 64 and O.query_rank(64, 64, 32) == 31


def test_query_coords_rmsnorm():
    q = _rand((10, 6), 42)
    F = _rand((6, 4), 43)
    phi = O.query_coords(q, F, 1e-6)
    np.testing.assert_allclose((phi ** 2).sum(1), 4.0, rtol=1e-12)
    z = O.query_coords(np.zeros((1, 6)), F, 1e-6)
    assert np.all(z == 0)
    # direction preserved
    zf = q @ F
    cos = (phi * zf).sum(1) / np.linalg.norm(phi, axis=1) / np.linalg.norm(zf, axis=1)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-12)


def test_query_distances():
    phi = _rand((12, 3), 44)
    lab = np.arange(12) % 3
    c, dist = O.query_distances(phi, lab, 3)
    for i in range(12):
        mem = phi[lab == lab[i]]
        assert abs(dist[i] - np.linalg.norm(phi[i] - mem.mean(0))) < 1e-12


# --------------------------------------------------------- routing (B.3)
def test_routing_score_brute_force_and_expanded_form():
    N, d, Cq, Ck = 24, 4, 3, 4
    k, v = _rand((N, d), 50, 1.2), _rand((N, d), 51)
    kl = np.arange(N) % Ck
    qbar = _rand((Cq, d), 52, 1.2)
    kbar = np.stack([k[kl == b].mean(0) for b in range(Ck)])
    vbar = np.stack([v[kl == b].mean(0) for b in range(Ck)])
    s = O.routing_score(qbar, k, v, kbar, vbar, kl)
    sq = math.sqrt(d)
    for a in range(Cq):
        m = max(max(qbar[a] @ k[j] / sq for j in range(N)), max(qbar[a] @ kbar[b] / sq for b in range(Ck)))
        for b in range(Ck):
            mem = [j for j in range(N) if kl[j] == b]
            tot = 0.0
            for j in mem:
                diff = math.exp(qbar[a] @ kbar[b] / sq - m) * vbar[b] - math.exp(qbar[a] @ k[j] / sq - m) * v[j]
                tot += float(diff @ diff)
            assert abs(s[a, b] - tot / len(mem)) <= 1e-12 * max(1.0, tot)
            # expanded form used by the GPU: |A|^2 - 2 A.mean(B_j) + mean |B_j|^2
            A = math.exp(qbar[a] @ kbar[b] / sq - m) * vbar[b]
            Bj = np.stack([math.exp(qbar[a] @ k[j] / sq - m) * v[j] for j in mem])
            exp_form = A @ A - 2 * A @ Bj.mean(0) + (Bj * Bj).sum(1).mean()
            assert abs(exp_form - s[a, b]) <= 1e-10 * max(1.0, A @ A + (Bj * Bj).sum(1).mean())


def test_probe_fractions_table_c2():
    g = json.load(open(os.path.join(GOLDEN, "table_c2_probe_fractions.json")))
    for row in g["rows"]:
        Nq = row["N_q"]
        p_route = 0
        p_exec = O.executed_pairs(p_route, g["M"], Nq)
        assert round(100.0 * p_exec / (Nq * Nq), 3) == row["percent"]
    lo, hi = g["range_text_percent"]
    fr = [100.0 * g["M"] / r["N_q"] for r in g["rows"]]
    assert round(min(fr), 3) == lo and round(max(fr), 3) == hi


def test_key_budget_reading():
    assert O.key_budget(0.22, 512, 75600, 75600) == 16120
    assert O.key_budget(0.22, 64, 118800, 118800) == math.ceil(0.22 * 118800 - 64 - 1e-6)
    assert O.key_budget(1.0 + 32 / 1024, 32, 1024, 1024) == 1024
    assert O.key_budget(0.001, 512, 1024, 1024) == 0


def test_route_prefix_rule():
    rng = np.random.default_rng(53)
    Cq, Ck = 5, 9
    s = rng.random((Cq, Ck))
    s[0, 3] = s[0, 6]                        # a tie: lower index ranks first
    kv = rng.integers(1, 20, Ck)
    qs = rng.integers(1, 30, Cq)
    beta = 37
    mask, p_route = O.route(s, kv, qs, beta)
    total = 0
    for a in range(Cq):
        order = sorted(range(Ck), key=lambda b: (-s[a, b], b))
        sel = [b for b in range(Ck) if mask[a, b]]
        n = len(sel)
        assert set(sel) == set(order[:n])            # a prefix of the ranking
        assert kv[order[:n]].sum() >= beta            # reaches the budget
        assert kv[order[:n - 1]].sum() < beta         # shortest such prefix
        total += qs[a] * kv[sel].sum()
    assert total == p_route
    assert O.route(s, kv, qs, int(kv.sum()))[0].all()        # full budget -> dense
    assert (O.route(s, kv, qs, 0)[0].sum(1) == 1).all()       # at least one group
    m2, _ = O.route(np.zeros((1, 3)), np.array([5, 5, 5]), np.array([1]), 6)
    assert m2.tolist() == [[True, True, False]]


def test_executed_pair_accounting():
    assert O.executed_pairs(1000, 64, 500) - 1000 == 64 * 500


def test_group_permutation_bijection_and_restore():
    lab = np.random.default_rng(54).integers(0, 6, 100)
    perm, off = O.group_permutation(lab, 6)
    assert sorted(perm.tolist()) == list(range(100))
    x = np.random.default_rng(55).random(100)
    xp = x[perm]
    restored = np.empty_like(xp)
    restored[perm] = xp
    assert np.array_equal(restored, x)
    for g in range(6):
        seg = perm[off[g]:off[g + 1]]
        assert np.all(lab[seg] == g) and np.all(np.diff(seg) > 0)


# ------------------------------------------------- probes and fit (A.2, A.3)
def test_probe_allocation_largest_remainder():
    assert O.probe_allocation(np.array([5, 3, 2]), 4, 10).tolist() == [2, 1, 1]
    assert O.probe_allocation(np.array([3, 3, 4]), 5, 10).tolist() == [2, 1, 2]
    assert O.probe_allocation(np.array([3, 7]), 5, 10).tolist() == [1, 4]
    sizes = np.random.default_rng(56).integers(1, 400, 300)
    N = int(sizes.sum())
    m = O.probe_allocation(sizes, 512, N)
    assert m.sum() == 512 and np.all(m <= sizes)
    assert np.all(np.abs(m - 512 * sizes / N) < 1.0)
    assert np.array_equal(O.probe_allocation(sizes, N + 5, N), sizes)


def test_probe_select_smallest_distance_then_index():
    lab = np.array([0, 1, 0, 0, 1, 0])
    d = np.array([0.5, 0.1, 0.2, 0.2, 0.3, 0.9])
    assert O.probe_select(lab, d, np.array([2, 1])).tolist() == [2, 3, 1]


def test_coverage_weights():
    sizes = np.array([10, 30, 5])
    m = np.array([2, 3, 1])
    groups = np.array([0, 0, 1, 1, 1, 2])
    w, alpha, wt = O.coverage_weights(groups, sizes, m, 6)
    assert abs(wt.sum() - 6) < 1e-12 and abs(alpha.sum() - 1) < 1e-12
    for a in range(3):
        assert abs(w[groups == a].sum() - sizes[a]) < 1e-12


def _fit_case(M=40, d=6, seed=60):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, d)) * 0.7 + 0.3
    R = rng.standard_normal((M, d)) * 0.05
    w = rng.integers(1, 5, M).astype(float)
    alpha = w / w.sum()
    return X, R, alpha, M * alpha


def test_ridge_fit_normal_equations_and_independent_solve():
    X, R, alpha, wt = _fit_case()
    lam = 0.7
    f = O.ridge_fit(X, R, alpha, wt, lam, 1e-6)
    Xb, Rb, B = f["Xbar"], f["Rbar"], f["B"]
    # weighted standardisation and centring (D.3)
    np.testing.assert_allclose(alpha @ Xb, 0, atol=1e-12)
    var = alpha @ (X - alpha @ X) ** 2
    np.testing.assert_allclose(alpha @ Xb ** 2, var / (var + 1e-6), rtol=1e-12)
    np.testing.assert_allclose(alpha @ Rb, 0, atol=1e-14)
    # normal equations of the penalised objective
    grad = Xb.T @ (wt[:, None] * (Rb - Xb @ B)) - lam * B
    assert np.abs(grad).max() < 1e-11
    # independent route: augmented least squares
    Aug = np.vstack([np.sqrt(wt)[:, None] * Xb, math.sqrt(lam) * np.eye(X.shape[1])])
    rhs = np.vstack([np.sqrt(wt)[:, None] * Rb, np.zeros((X.shape[1], X.shape[1]))])
    B2 = np.linalg.lstsq(Aug, rhs, rcond=None)[0]
    np.testing.assert_allclose(B, B2, atol=1e-11)
    # finite-difference check of the objective at B
    def obj(Bm):
        E = Rb - Xb @ Bm
        return float((wt[:, None] * E * E).sum() + lam * (Bm * Bm).sum())
    for (i, j) in [(0, 0), (2, 5), (4, 1)]:
        Eij = np.zeros_like(B)
        Eij[i, j] = 1e-5
        assert abs(obj(B + Eij) - obj(B - Eij)) < 1e-9


def test_ridge_fit_rejects_singular_gram_without_penalty():
    X = np.ones((5, 3))
    with pytest.raises(O.NumericError):
        O.ridge_fit(X, np.zeros((5, 3)), np.full(5, 0.2), np.ones(5), 0.0, 1e-6)


def test_planted_affine_map_is_recovered():
    """Residuals that are exactly affine in the sparse output are recovered as
    lambda -> 0, and the residual row space has the planted rank."""
    rng = np.random.default_rng(61)
    N, d, r = 300, 12, 8
    Osp = rng.standard_normal((N, d))
    bstar = rng.standard_normal(d) * 0.1
    U, Vt = rng.standard_normal((d, r)), rng.standard_normal((r, d)) * 0.1
    Odense = Osp + bstar + Osp @ U @ Vt
    P = np.arange(0, N, 5)
    alpha = np.full(len(P), 1.0 / len(P))
    f = O.ridge_fit(Osp[P], Odense[P] - Osp[P], alpha, len(P) * alpha, 1e-9, 1e-6)
    S = np.linalg.svd(np.sqrt(len(P) * alpha)[:, None] * f["Rbar"], compute_uv=False)
    assert int((S > 1e-10 * S.max()).sum()) == r
    out = O.apply_correction(Osp, P, Odense[P], f)
    np.testing.assert_allclose(out, Odense, atol=1e-7)
    # closed form B = (Xb^T W Xb + lam I)^-1 Xb^T W Xb diag(sigma) U V^T
    Xb, wt = f["Xbar"], len(P) * alpha
    G = Xb.T @ (wt[:, None] * Xb) + 1e-9 * np.eye(d)
    Bc = np.linalg.solve(G, Xb.T @ (wt[:, None] * Xb) @ np.diag(f["sigma"]) @ U @ Vt)
    np.testing.assert_allclose(f["B"], Bc, atol=1e-8)


def test_residual_span_projection():
    X, R, alpha, wt = _fit_case(M=10, d=8, seed=62)
    f = O.ridge_fit(X, R, alpha, wt, 1.0, 1e-6)
    B = f["B"]
    np.testing.assert_allclose(O.residual_span_projection(B, f["Rbar"], wt), B, atol=1e-12)
    # fewer probes than channels: rank(Rbar) < d and the projection is still the identity
    X2, R2, a2, w2 = _fit_case(M=5, d=8, seed=63)
    f2 = O.ridge_fit(X2, R2, a2, w2, 1.0, 1e-6)
    np.testing.assert_allclose(O.residual_span_projection(f2["B"], f2["Rbar"], w2), f2["B"], atol=1e-12)
    Bt = O.residual_span_projection(B, f["Rbar"], wt, rank=2)
    assert np.linalg.matrix_rank(Bt, tol=1e-10) == 2


def test_apply_correction_formula():
    X, R, alpha, wt = _fit_case(M=12, d=5, seed=64)
    f = O.ridge_fit(X, R, alpha, wt, 1.0, 1e-6)
    Osp = _rand((20, 5), 65)
    P = np.array([3, 7])
    Od = _rand((2, 5), 66)
    out = O.apply_correction(Osp, P, Od, f)
    for i in range(20):
        if i in P:
            np.testing.assert_array_equal(out[i], Od[list(P).index(i)])
        else:
            xb = (Osp[i] - f["mu_X"]) / f["sigma"]
            np.testing.assert_allclose(out[i], Osp[i] + f["mu_R"] + xb @ f["B"], atol=1e-13)


# ------------------------------------------------------------ evaluation
def test_table2_error_reductions():
    g = json.load(open(os.path.join(GOLDEN, "table2_errors.json")))
    sem = g["semantic_no_repair"]["mean"]
    semr = g["semantic_with_repair"]
    ours = g["sparsepr"]
    red = [round(100 * O.error_reduction(o, s), 1) for o, s in zip(ours["mean"], sem)]
    assert red == [66.3, 61.6, 90.5, 78.8]
    assert [min(red), max(red)] == g["claims"]["mean_reduction_vs_semantic_no_repair_percent"]
    r2 = [round(100 * O.error_reduction(o, s), 1) for o, s in zip(ours["mean"], semr["mean"])]
    assert [min(r2), max(r2)] == g["claims"]["mean_reduction_vs_semantic_with_repair_percent"]
    r3 = [round(100 * O.error_reduction(o, s), 1) for o, s in zip(ours["p99"], semr["p99"])]
    assert [min(r3), max(r3)] == g["claims"]["p99_reduction_vs_semantic_with_repair_percent"]


def test_relative_error_definition():
    Od = np.array([[3.0, 4.0], [0.0, 0.0]])
    Oh = np.array([[3.0, 5.0], [0.0, 1e-9]])
    e = O.relative_error(Oh, Od)
    assert abs(e[0] - 1.0 / (5.0 + 1e-8)) < 1e-15 and abs(e[1] - 1e-9 / 1e-8) < 1e-12


# ------------------------------------------------------------ whole call
def _tiny_head(**kw):
    from synthetic import get_workload, generate_head
    w = get_workload("tiny", grid=(2, 8, 8), **kw)
    q, k, v = generate_head(w, 0, 1)
    return w, q, k, v


def test_whole_call_invariants_on_tiny():
    w, q, k, v = _tiny_head()
    r = O.sparsepr_head(q, k, v, bh=1, want_dense=True, **O.workload_kwargs(w))
    N = w.N
    assert r["pairs_exec"] - r["pairs_route"] == w.M * N
    assert r["pairs_exec"] / N / N >= w.density - 1e-12          # plain >= beta rule
    assert r["m"].sum() == w.M and len(np.unique(r["probes"])) == w.M
    np.testing.assert_allclose(r["O"][r["probes"]], r["O_dense"][r["probes"]], atol=1e-13)
    assert abs(r["wt"].sum() - w.M) < 1e-9


def test_whole_call_full_density_is_dense():
    w, q, k, v = _tiny_head()
    kw = O.workload_kwargs(w)
    kw["density"] = 1.0 + w.M / w.N
    r = O.sparsepr_head(q, k, v, bh=0, want_dense=True, **kw)
    assert r["mask"].all()
    np.testing.assert_allclose(r["O_sp"], r["O_dense"], atol=1e-12)


def test_whole_call_all_rows_probes_is_exact():
    w, q, k, v = _tiny_head()
    kw = O.workload_kwargs(w)
    kw["M"] = w.N
    r = O.sparsepr_head(q, k, v, bh=0, want_dense=True, **kw)
    np.testing.assert_array_equal(r["O"], r["O_dense"])


# ------------------------------------------------------------- warm start (C.1)
def _spd(d, seed, gap=None):
    """Symmetric positive definite d x d matrix; with ``gap`` its spectrum is
    geometric with that ratio between neighbours."""
    U, _ = np.linalg.qr(_rand((d, d), seed))
    w = (gap ** -np.arange(d)) if gap else np.exp(_rand(d, seed + 1))
    return U @ np.diag(w) @ U.T


@pytest.mark.parametrize("scale", [1.0, 1.0 / math.sqrt(8)])
def test_warm_factor_from_exact_eigenbasis_is_cold_factor(scale):
    """Started from the cold factor of the same metric, the subspace iteration
    stays on the leading eigenspace, so F F^T is the truncated metric."""
    d, r = 8, 3
    M = _spd(d, 60)
    w, U = O.eigh_desc(M)
    F0 = U[:, :r] * np.sqrt(w[:r])           # spans the leading eigenspace, not orthonormal
    F = O.warm_factor(M, F0, r, scale)
    want = U[:, :r] @ np.diag(w[:r]) @ U[:, :r].T * scale * scale
    np.testing.assert_allclose(F @ F.T, want, atol=1e-12 * np.abs(want).max())


def test_warm_factor_is_projected_metric_of_iterated_subspace():
    """Independent route: F F^T = P M P with P the orthogonal projector on
    span(M^2 F_prev), built by Householder QR."""
    d, r = 10, 4
    M = _spd(d, 61)
    F0 = _rand((d, r), 62)
    F = O.warm_factor(M, F0, r, 0.5, iters=2)
    Qh, _ = np.linalg.qr(M @ M @ F0)
    P = Qh @ Qh.T
    np.testing.assert_allclose(F @ F.T, 0.25 * P @ M @ P, atol=1e-11 * np.abs(M).max())
    # one iteration: projector on span(M F_prev)
    F1 = O.warm_factor(M, F0, r, 1.0, iters=1)
    Q1, _ = np.linalg.qr(M @ F0)
    np.testing.assert_allclose(F1 @ F1.T, Q1 @ Q1.T @ M @ Q1 @ Q1.T, atol=1e-11 * np.abs(M).max())


def test_warm_factor_exact_on_metric_of_rank_r():
    d, r = 9, 3
    A = _rand((r, d), 63)
    M = A.T @ A
    F = O.warm_factor(M, _rand((d, r), 64), r, 1.0, iters=1)
    np.testing.assert_allclose(F @ F.T, M, atol=1e-10 * np.abs(M).max())


def test_warm_factor_converges_to_cold_factor():
    d, r = 12, 4
    M = _spd(d, 65, gap=1.6)
    w, U = O.eigh_desc(M)
    want = U[:, :r] @ np.diag(w[:r]) @ U[:, :r].T
    errs = []
    for it in (1, 2, 8, 80):
        F = O.warm_factor(M, _rand((d, r), 66), r, 1.0, iters=it)
        errs.append(np.abs(F @ F.T - want).max())
    assert errs[0] > errs[1] > errs[2] > errs[3]
    assert errs[3] < 1e-10 * w[0]


def test_warm_factor_falls_back_to_cold():
    d = 6
    M = _spd(d, 67)
    assert O.warm_factor(M, _rand((d, 2), 68), 3, 1.0) is None          # fewer columns than the rank
    F0 = _rand((d, 3), 69)
    F0[:, 1] = 0.0                                                        # a vanishing pivot
    assert O.warm_factor(M, F0, 3, 1.0) is None
    assert O.cholesky_checked(np.diag([4.0, 1e-13])) is None
    np.testing.assert_allclose(O.cholesky_checked(np.diag([4.0, 1.0])), np.diag([2.0, 1.0]))


def test_warm_centres_projection_and_rmsnorm():
    N, d, r, C = 40, 5, 3, 6
    Y = _rand((N, r), 70)
    cbar = _rand((4, d), 71)
    F = _rand((d, r), 72)
    init = O.kmeans_init_indices(3, 0, 0, C, N)
    cen = O.warm_centres(Y, cbar, F, C, init)
    for b in range(4):
        for j in range(r):
            assert abs(cen[b, j] - sum(cbar[b, t] * F[t, j] for t in range(d))) < 1e-12
    np.testing.assert_array_equal(cen[4:], Y[init[4:]])
    # query side: a group of identical rows has its coordinate as the centre
    q = np.repeat(_rand((3, d), 73), [5, 7, 4], axis=0)
    labels = np.repeat(np.arange(3), [5, 7, 4])
    phi = O.query_coords(q, F, 1e-6)
    qbar = O.group_means(q, labels, 3)
    cq = O.warm_centres(phi, qbar, F, 3, np.zeros(3, np.int64), rms_eps=1e-6)
    np.testing.assert_allclose(cq, O.group_means(phi, labels, 3), atol=1e-12)
    # RMS floor: a zero centroid stays zero
    cz = O.warm_centres(phi, np.zeros((1, d)), F, 3, np.zeros(3, np.int64), rms_eps=1e-6)
    assert np.all(cz[0] == 0.0)


def test_warm_start_from_converged_keys_is_a_fixed_point():
    """Converged K/V groups are reproduced by one warm assignment: the
    projected previous centroids are the converged centres (phi_K is linear)."""
    rng = np.random.default_rng(74)
    N, d, C = 240, 6, 5
    k = np.repeat(rng.standard_normal((C, d)) * 4, N // C, axis=0) + rng.standard_normal((N, d)) * 0.3
    q = rng.standard_normal((N, d))
    F = O.key_factor(O.key_metric(q, O.sample_indices(N, 64)), 4, 64)
    init = O.kmeans_init_indices(5, 0, 0, C, N)
    lab, _, _, _ = O.kmeans(k @ F, init, 200, 0)
    lab_c, C2, _ = O.compact_labels(lab, C)
    assert C2 == C
    kbar = O.group_means(k, lab_c, C2)
    cen = O.warm_centres(k @ F, kbar, F, C, init)
    lab_w, _, n_it, _ = O.kmeans(k @ F, init, 2, 0, cen)
    assert np.array_equal(O.compact_labels(lab_w, C)[0], lab_c)
    assert n_it == 2                       # the second assignment changes nothing


def test_warm_call_on_same_input_keeps_converged_kv_groups():
    w, q, k, v = _tiny_head()
    kw = O.workload_kwargs(w)
    kw.update(kmeans_iters=200, kmeans_tol=0.0)
    cold = O.sparsepr_head(q, k, v, bh=0, **kw)
    kw["kmeans_iters"] = 2
    warm = O.sparsepr_head(q, k, v, bh=0, warm=O.warm_state(cold), **kw)
    assert warm["warm_factor_used"] == (True, True)
    np.testing.assert_allclose(warm["F_K"] @ warm["F_K"].T, cold["F_K"] @ cold["F_K"].T,
                               atol=1e-9 * np.abs(cold["F_K"]).max() ** 2)
    assert np.array_equal(warm["kv_labels"], cold["kv_labels"])
    assert warm["kmeans_iters_k"] <= 2 and warm["kmeans_iters_q"] <= 2
    assert warm["pairs_exec"] / w.N / w.N >= w.density - 1e-12


# ------------------------------------------------------ semantic partition (R16)
def _blob_keys(seed=80, N=160, d=6):
    """Keys in two far blobs along e_0, a direction no query has: raw-key
    clustering splits the blobs, the response metric cannot see them."""
    rng = np.random.default_rng(seed)
    blob = np.arange(N) % 2
    k = rng.standard_normal((N, d)) * 0.2
    k[:, 0] += np.where(blob == 1, 50.0, -50.0)
    k[:, 1:] += rng.standard_normal((N, d - 1)) * 2.0
    q = rng.standard_normal((N, d))
    q[:, 0] = 0.0
    v = rng.standard_normal((N, d))
    return q, k, v, blob


def _kw(**over):
    kw = dict(seed=3, density=0.5, M=8, Ms=64, lam=1.0, Cq=4, Ck=2, rK=4, rQ=4, kmeans_iters=25,
              kmeans_tol=0.0)
    kw.update(over)
    return kw


def test_semantic_keys_split_raw_blobs_response_keys_do_not():
    q, k, v, blob = _blob_keys()
    sem = O.sparsepr_head(q, k, v, bh=0, partition="semantic", **_kw())
    res = O.sparsepr_head(q, k, v, bh=0, partition="response", **_kw())
    lab = sem["kv_labels"]
    assert sem["Ck"] == 2 and (np.array_equal(lab, blob) or np.array_equal(lab, 1 - blob))
    # phi_K = k F_K has no e_0 component, so the blobs coincide in response coordinates
    assert np.abs(res["F_K"][0]).max() < 1e-12
    agree = max((res["kv_labels"] == blob).mean(), (res["kv_labels"] != blob).mean())
    assert agree < 0.75


def test_semantic_query_distances_are_raw_space():
    q, k, v, _ = _blob_keys(81)
    r = O.sparsepr_head(q, k, v, bh=0, partition="semantic", **_kw())
    for a in range(r["Cq"]):
        mem = np.nonzero(r["q_labels"] == a)[0]
        mean = q[mem].mean(axis=0)
        for i in mem[:5]:
            assert abs(r["d_i"][i] - math.sqrt(sum((q[i, t] - mean[t]) ** 2 for t in range(q.shape[1])))) < 1e-12


def test_key_response_variant_mixes_the_two():
    q, k, v, _ = _blob_keys(82)
    sem = O.sparsepr_head(q, k, v, bh=0, partition="semantic", **_kw())
    res = O.sparsepr_head(q, k, v, bh=0, partition="response", **_kw())
    kr = O.sparsepr_head(q, k, v, bh=0, partition="key_response", **_kw())
    assert np.array_equal(kr["kv_labels"], res["kv_labels"])
    assert np.array_equal(kr["q_labels"], sem["q_labels"])


def test_semantic_call_is_rotation_invariant():
    """Rotating queries and keys by one orthogonal map changes no distance
    between raw rows and no logit, so the semantic call's output is unchanged."""
    q, k, v, _ = _blob_keys(83)
    R, _ = np.linalg.qr(_rand((6, 6), 84))
    a = O.sparsepr_head(q, k, v, bh=0, partition="semantic", **_kw(Cq=5, Ck=3))
    b = O.sparsepr_head(q @ R, k @ R, v, bh=0, partition="semantic", **_kw(Cq=5, Ck=3))
    assert np.array_equal(a["kv_labels"], b["kv_labels"]) and np.array_equal(a["q_labels"], b["q_labels"])
    np.testing.assert_allclose(a["O"], b["O"], atol=1e-10)


# ------------------------------------------------ probe variants and families
def test_random_probes_are_a_uniform_sample():
    """Floyd's algorithm draws every M-subset with equal probability: all 20
    subsets of 3 rows out of 6 appear equally often over 20000 seeds."""
    counts = {}
    for seed in range(20000):
        P = O.random_probes(seed, 0, 6, 3)
        assert len(P) == 3 and len(set(P.tolist())) == 3 and P.min() >= 0 and P.max() < 6
        counts[tuple(P)] = counts.get(tuple(P), 0) + 1
    assert len(counts) == 20
    exp, sd = 1000.0, math.sqrt(20000 * (1 / 20) * (19 / 20))
    assert all(abs(c - exp) < 5 * sd for c in counts.values())
    assert np.array_equal(O.random_probes(1, 3, 9, 9), np.arange(9))
    assert not np.array_equal(O.random_probes(1, 0, 1000, 10), O.random_probes(1, 1, 1000, 10))


def test_uniform_probes_closed_form():
    assert O.uniform_probes(10, 4).tolist() == [1, 3, 6, 8]
    assert np.array_equal(O.uniform_probes(7, 7), np.arange(7))
    P = O.uniform_probes(75600, 512)
    assert len(np.unique(P)) == 512 and np.all(np.diff(P) >= 147)


def test_probes_listed_by_group_then_index():
    labels = np.array([2, 0, 1, 0, 2, 1, 0])
    P, m = O.listed_by_group(np.array([6, 0, 3, 4, 5]), labels, 3)
    assert P.tolist() == [3, 6, 5, 0, 4] and m.tolist() == [2, 1, 2]


def _fit_problem(seed=90, M=60, d=5):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, d)) * rng.uniform(0.5, 2.0, d) + rng.standard_normal(d)
    R = rng.standard_normal((M, d))
    w = rng.uniform(0.5, 2.0, M)
    alpha = w / w.sum()
    return X, R, alpha, M * alpha


@pytest.mark.parametrize("family", ["diagonal", "scalar"])
def test_restricted_fits_minimise_the_penalised_objective(family):
    """D.4: each family minimises sum_p w~_p |Rbar_p - Xbar_p B|^2 + lambda |B|_F^2
    over its own parameters (zero derivative by central differences)."""
    X, R, alpha, wt = _fit_problem()
    lam = 0.7
    f = O.restricted_fit(X, R, alpha, wt, lam, 1e-6, family)
    Xb, Rb, B = f["Xbar"], f["Rbar"], f["B"]
    d = X.shape[1]

    def obj(Bm):
        E = Rb - Xb @ Bm
        return float((wt[:, None] * E * E).sum() + lam * (Bm * Bm).sum())

    params = [np.diag(np.eye(d)[j]) for j in range(d)] if family == "diagonal" else [np.eye(d)]
    for D in params:
        h = 1e-5
        g = (obj(B + h * D) - obj(B - h * D)) / (2 * h)
        assert abs(g) < 1e-6 * max(1.0, obj(B))
    assert np.count_nonzero(B - np.diag(np.diag(B))) == 0
    if family == "scalar":
        assert np.allclose(B, B[0, 0] * np.eye(d))


def test_restricted_fits_recover_planted_maps_and_mean_only():
    X, _, alpha, wt = _fit_problem(91)
    f0 = O.ridge_fit(X, np.zeros_like(X), alpha, wt, 1.0, 1e-6)
    Xb = f0["Xbar"]
    c = np.array([0.5, -1.0, 2.0, 0.0, 3.0])
    fd = O.restricted_fit(X, Xb * c, alpha, wt, 0.0, 1e-6, "diagonal")      # residual = Xbar diag(c)
    np.testing.assert_allclose(np.diag(fd["B"]), c, atol=1e-10)
    fs = O.restricted_fit(X, 1.7 * Xb, alpha, wt, 0.0, 1e-6, "scalar")
    np.testing.assert_allclose(fs["B"], 1.7 * np.eye(5), atol=1e-10)
    fm = O.restricted_fit(X, Xb * c + 3.0, alpha, wt, 1.0, 1e-6, "mean")
    assert not fm["B"].any()
    np.testing.assert_allclose(fm["mu_R"], alpha @ (Xb * c) + 3.0, atol=1e-12)


def test_whole_call_variants_on_tiny():
    w, q, k, v = _tiny_head()
    kw = O.workload_kwargs(w)
    base = O.sparsepr_head(q, k, v, bh=0, want_dense=True, **kw)
    for probes in ("random", "uniform"):
        r = O.sparsepr_head(q, k, v, bh=0, probes=probes, **kw)
        assert len(np.unique(r["probes"])) == w.M and r["m"].sum() == w.M
        assert abs(r["wt"].sum() - w.M) < 1e-9
        np.testing.assert_array_equal(r["O_sp"], base["O_sp"])     # the sparse base does not depend on probes
    full_rank = O.sparsepr_head(q, k, v, bh=0, residual_rank=w.d, **kw)
    np.testing.assert_allclose(full_rank["O"], base["O"], atol=1e-9)   # R8: full rank is the identity
    mean = O.sparsepr_head(q, k, v, bh=0, correction="mean", **kw)
    unp = np.setdiff1d(np.arange(w.N), mean["probes"])
    np.testing.assert_allclose(mean["O"][unp], base["O_sp"][unp] + mean["fit"]["mu_R"][None, :], atol=1e-12)


# ------------------------------------------------------------------ GQA (R19)
def test_gqa_metric_is_the_mean_of_the_heads_metrics():
    """G M_s evenly spaced rows of the stacked heads are each head's own M_s
    sampled rows, so the shared metric is the mean of the per-head metrics."""
    G, N, d, Ms = 3, 50, 4, 7
    qs = [_rand((N, d), 100 + g) for g in range(G)]
    stacked = np.concatenate(qs)
    idx = O.sample_indices(G * N, G * Ms)
    shared = O.key_metric(stacked, idx)
    per_head = [O.key_metric(x, O.sample_indices(N, Ms)) for x in qs]
    np.testing.assert_allclose(shared, np.mean(per_head, axis=0), atol=1e-13)


def test_gqa_heads_share_the_kv_partition():
    w, q, k, v = _tiny_head()
    kw = O.workload_kwargs(w)
    kw.pop("Ms")
    qs = [q, q[::-1].copy(), 0.5 * q]
    res = O.sparsepr_gqa(qs, k, v, kvh=1, Ms=w.Ms, **kw)
    for r in res[1:]:
        assert np.array_equal(r["kv_labels"], res[0]["kv_labels"])
        np.testing.assert_array_equal(r["F_K"], res[0]["F_K"])
    assert not np.array_equal(res[0]["q_labels"], res[1]["q_labels"])
    # G = 1 is the single-head call with the K/V stream of head kvh
    one = O.sparsepr_gqa([q], k, v, kvh=0, Ms=w.Ms, **kw)[0]
    ref = O.sparsepr_head(q, k, v, bh=0, Ms=w.Ms, **kw)
    np.testing.assert_array_equal(one["O"], ref["O"])


def test_gqa_warm_start_keeps_converged_shared_groups():
    """Warm-starting a GQA call from its own converged state reproduces the
    shared K/V groups (one assignment from the converged centres)."""
    w, q, k, v = _tiny_head()
    kw = O.workload_kwargs(w)
    Ms = kw.pop("Ms")
    kw.update(kmeans_iters=200, kmeans_tol=0.0)
    qs = [q, q[::-1].copy()]
    cold = O.sparsepr_gqa(qs, k, v, kvh=0, Ms=Ms, **kw)
    kw["kmeans_iters"] = 2
    warm = O.sparsepr_gqa(qs, k, v, kvh=0, Ms=Ms, warms=[O.warm_state(r) for r in cold], **kw)
    for c, r in zip(cold, warm):
        assert r["warm_factor_used"][0]
        assert np.array_equal(r["kv_labels"], c["kv_labels"])
    assert np.array_equal(warm[0]["kv_labels"], warm[1]["kv_labels"])


def test_drift_inputs_are_seeded_and_small():
    from synthetic import drift_inputs, generate_inputs
    from synthetic import get_workload
    w = get_workload("tiny", grid=(2, 8, 8))
    x0 = generate_inputs(w)
    a, b = drift_inputs(w, x0, step=1), drift_inputs(w, x0, step=1)
    c = drift_inputs(w, x0, step=2)
    for u, u2, u3, x in zip(a, b, c, x0):
        assert np.array_equal(u, u2) and not np.array_equal(u, u3)
        assert 0.02 < np.std(u - x) / np.std(x) < 0.08
