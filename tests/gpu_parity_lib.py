"""Helpers shared by the GPU parity tests: run the staged C-ABI path on
seeded synthetic inputs and compare every stage with the fp64 oracle."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
from synthetic import generate_inputs
from synthetic.video_grid import bf16_bits

TOL_ATTN = 2e-3       # per-row relative L2, bf16 attention with fp32 accumulation
TOL_ATTN_F32 = 2e-5   # fp32 inputs on the CUDA-core kernel
TOL_FIT = 1e-4        # fp32 ridge fit and corrected output
TOL_TF32 = 1e-3       # k-means coordinates and centres are stored TF32-rounded (2^-11 relative)


def to_device(w, arrays, device="cuda"):
    out = []
    for a in arrays:
        if w.dtype == "bf16":
            t = torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
        out.append(t.to(device))
    return out


def run_staged(cfg, q, k, v, debug=False):
    import free_block_sparse_sampled_b200 as S
    ws = S.alloc_workspace(cfg)
    part = S.partition(cfg, q, k, v, ws, debug=debug, extras=True)
    rt = S.route(cfg, part, ws)
    O_sp, pd, ps = S.attention(cfg, part, rt, ws)
    fit = S.probe_fit(cfg, part, rt, ps, pd, ws)
    out = S.apply(cfg, part, rt, O_sp, pd, fit, ws)
    torch.cuda.synchronize()
    status = S.device_status(ws)
    res = {"part": part, "route": rt, "O_sp": O_sp, "probe_dense": pd, "probe_sparse": ps, "fit": fit,
           "out": out, "status": status, "ws": ws}
    return res


def np64(t):
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy().astype(np.float64)


def npi(t):
    return t.detach().cpu().numpy().astype(np.int64)


def head_view(res, cfg, bh):
    """Per-head numpy views of the GPU outputs."""
    p, r = res["part"], res["route"]
    Cq2, Ck2 = (int(x) for x in npi(p["n_groups"][bh]))
    N, Mp = cfg.N, cfg.Mp
    h = {"Cq": Cq2, "Ck": Ck2, "bh": bh}
    for k in ["q_label", "kv_label", "perm_q", "perm_kv", "pos_q"]:
        h[k] = npi(p[k][bh])
    h["q_offsets"] = npi(p["q_offsets"][bh])[: Cq2 + 1]
    h["kv_offsets"] = npi(p["kv_offsets"][bh])[: Ck2 + 1]
    b, hh = divmod(bh, cfg.H)
    hk = hh // (cfg.H // cfg.Hk)   # permuted K/V live per K/V head
    h["Qp"] = np64(p["Qp"][b, hh])
    h["Kp"], h["Vp"] = (np64(p[n][b, hk]) for n in ("Kp", "Vp"))
    h["q_centroid"] = np64(p["q_centroid"][bh])[:Cq2]
    h["k_centroid"] = np64(p["k_centroid"][bh])[:Ck2]
    h["v_centroid"] = np64(p["v_centroid"][bh])[:Ck2]
    h["q_dist"] = np64(p["q_dist"][bh])
    h["score"] = np64(r["score"][bh])[:Cq2, :Ck2]
    h["mask"] = npi(r["mask"][bh])[:Cq2, :Ck2].astype(bool)
    h["sel_count"] = npi(r["sel_count"][bh])[:Cq2]
    h["sel_groups"] = npi(r["sel_groups"][bh])[:Cq2]
    h["pairs"] = npi(r["pairs"][bh])
    h["probe_idx"] = npi(r["probe_idx"][bh])[:Mp]
    h["probe_group"] = npi(r["probe_group"][bh])[:Mp]
    h["probe_weight"] = np64(r["probe_weight"][bh])[:Mp]
    h["probe_alloc"] = npi(r["probe_alloc"][bh])[:Cq2]
    h["O_sp"] = np64(res["O_sp"][bh])
    h["probe_dense"] = np64(res["probe_dense"][bh])[:Mp]
    h["probe_sparse"] = np64(res["probe_sparse"][bh])[:Mp]
    for k in ["B", "mu_x", "sigma", "mu_r"]:
        h["fit_" + k] = np64(res["fit"][k][bh])
    h["out"] = np64(res["out"][b, hh])
    for k in ["F_K", "F_Q", "phi_K", "phi_Q", "kv_centres", "q_centres"]:
        if k in p:
            h[k] = np64(p[k][bh])
    if "debug_kv_scores" in p:
        h["debug_kv_scores"] = p["debug_kv_scores"][bh].cpu().numpy()
        h["debug_q_scores"] = p["debug_q_scores"][bh].cpu().numpy()
        h["debug_kv_hist"] = npi(p["debug_kv_hist"][bh])
        h["debug_q_hist"] = npi(p["debug_q_hist"][bh])
    h["iters"] = npi(p["kmeans_iters_run"][bh])
    return h


def row_rel_l2(a, b):
    return np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-30)


def check_integer_chain(h, cfg):
    """Integer steps, each fed the GPU's own upstream values (bit-exact);
    probes follow the config's probe selection."""
    N = cfg.N
    # group-major permutation and offsets from the GPU labels
    for lab_key, perm_key, off_key, C in [("q_label", "perm_q", "q_offsets", h["Cq"]),
                                          ("kv_label", "perm_kv", "kv_offsets", h["Ck"])]:
        perm, off = O.group_permutation(h[lab_key], C)
        assert np.array_equal(perm, h[perm_key]), perm_key
        assert np.array_equal(off, h[off_key]), off_key
        assert np.all(np.bincount(h[lab_key], minlength=C) > 0)      # compacted: all nonempty
    inv = np.empty(N, np.int64)
    inv[h["perm_q"]] = np.arange(N)
    assert np.array_equal(inv, h["pos_q"])
    # routing from the GPU's fp32 scores
    kv_sizes = np.diff(h["kv_offsets"])
    q_sizes = np.diff(h["q_offsets"])
    beta = O.key_budget(cfg.density, cfg.Mp, N, N)
    mask, p_route = O.route(h["score"], kv_sizes, q_sizes, beta)
    assert np.array_equal(mask, h["mask"])
    assert p_route == h["pairs"][0]
    assert O.executed_pairs(p_route, cfg.Mp, N) == h["pairs"][1]
    for a in range(h["Cq"]):
        n = h["sel_count"][a]
        assert list(h["sel_groups"][a][:n]) == list(np.nonzero(mask[a])[0])
    # probes from the GPU's labels and fp32 d_i
    if cfg.Mp > 0:
        if cfg.probe_select == "stratified" or cfg.Mp >= N:
            m = O.probe_allocation(q_sizes, cfg.Mp, N)
            P = O.probe_select(h["q_label"], h["q_dist"], m)
        else:
            bh = h["bh"]
            rows = O.random_probes(cfg.seed, bh, N, cfg.Mp) if cfg.probe_select == "random" else \
                O.uniform_probes(N, cfg.Mp)
            P, m = O.listed_by_group(rows, h["q_label"], h["Cq"])
        assert np.array_equal(m, h["probe_alloc"])
        assert np.array_equal(P, h["probe_idx"])
        assert np.array_equal(h["q_label"][P], h["probe_group"])
        _, _, wt = O.coverage_weights(h["q_label"][P], q_sizes, m, cfg.Mp)
        np.testing.assert_allclose(h["probe_weight"], wt, rtol=1e-6)


def check_kmeans_chain(h, cfg, which):
    """k-means (debug export): argmax of the GPU's own fp32 scores gives its
    labels; the stop rule on its label history gives its iteration count;
    scores and centres agree with fp64 recomputation from its features."""
    if which == "kv":
        scores, hist, phi, cen, n_it, C = (h["debug_kv_scores"], h["debug_kv_hist"], h["phi_K"],
                                          h["kv_centres"], h["iters"][0], cfg.Ck)
    else:
        scores, hist, phi, cen, n_it, C = (h["debug_q_scores"], h["debug_q_hist"], h["phi_Q"],
                                          h["q_centres"], h["iters"][1], cfg.Cq)
    assert 1 <= n_it <= cfg.kmeans_iters
    final = hist[n_it - 1]
    assert np.array_equal(O.argmax_rows(scores.astype(np.float64)), final)
    stop = O.kmeans_stop_count(cfg.kmeans_tol, cfg.N)
    changed = [int((hist[t] != hist[t - 1]).sum()) for t in range(1, n_it)]
    if n_it < cfg.kmeans_iters:
        assert changed[-1] <= stop
    assert all(c > stop for c in changed[:-1])
    # fp32 scores vs fp64 recomputation from the GPU's features and centres
    ref = phi @ cen.T - 0.5 * (cen * cen).sum(1)[None, :]
    scale = np.linalg.norm(phi, axis=1)[:, None] * np.linalg.norm(cen, axis=1)[None, :] + (cen * cen).sum(1)[None, :]
    assert np.all(np.abs(scores - ref) <= 1e-5 * scale + 1e-6)
    # final centres = member means of the previous assignment (empty keep value)
    if n_it >= 2:
        prev = hist[n_it - 2]
        counts = np.bincount(prev, minlength=C)
        sums = np.zeros_like(cen)
        np.add.at(sums, prev, phi)
        nz = counts > 0
        np.testing.assert_allclose(cen[nz], sums[nz] / counts[nz][:, None], rtol=TOL_TF32, atol=1e-5)
    # compaction of the final raw labels gives the exported group labels
    lab, C2, _ = O.compact_labels(final, C)
    key = "kv_label" if which == "kv" else "q_label"
    assert np.array_equal(lab, h[key]) and C2 == (h["Ck"] if which == "kv" else h["Cq"])


def check_attention(h, cfg, tol):
    """Eq. (2) on the GPU's permuted Q/K/V and selected cells, per row."""
    qlab_p = h["q_label"][h["perm_q"]]
    klab_p = h["kv_label"][h["perm_kv"]]
    ref = O.sparse_attention(h["Qp"], h["Kp"], h["Vp"], qlab_p, klab_p, h["mask"])
    err = row_rel_l2(h["O_sp"], ref)
    assert err.max() <= tol, f"sparse attention max rel-L2 {err.max():.3e}"
    if cfg.Mp > 0:
        q = h["Qp"][h["pos_q"][h["probe_idx"]]]
        dref = O.dense_attention(q, h["Kp"], h["Vp"])
        derr = row_rel_l2(h["probe_dense"], dref)
        assert derr.max() <= tol, f"probe rows max rel-L2 {derr.max():.3e}"
        assert np.array_equal(h["probe_sparse"], h["O_sp"][h["pos_q"][h["probe_idx"]]])
    return float(err.max())


def fit_reference(h, cfg):
    """The oracle's fit (family and rank of the config) on the GPU's probe rows."""
    q_sizes = np.diff(h["q_offsets"])
    _, alpha, wt = O.coverage_weights(h["probe_group"], q_sizes, h["probe_alloc"], cfg.Mp)
    X, D = h["probe_sparse"], h["probe_dense"]
    f = O.restricted_fit(X, D - X, alpha, wt, cfg.lam, cfg.eps_std, cfg.correction)
    if 0 < cfg.residual_rank < cfg.d:
        f = {**f, "B": O.residual_span_projection(f["B"], f["Rbar"], wt, cfg.residual_rank)}
    return f


def check_fit_and_apply(h, cfg):
    """Ridge fit and corrected output from the GPU's own sparse / dense probe rows."""
    if cfg.Mp == 0:
        np.testing.assert_array_equal(h["out"], h["O_sp"][h["pos_q"]])
        return
    X, D = h["probe_sparse"], h["probe_dense"]
    f = fit_reference(h, cfg)
    for k in ["mu_X", "sigma", "mu_R"]:
        g = h["fit_" + {"mu_X": "mu_x", "sigma": "sigma", "mu_R": "mu_r"}[k]]
        np.testing.assert_allclose(g, f[k], rtol=TOL_FIT, atol=TOL_FIT * np.abs(f[k]).max() + 1e-12)
    Bn = max(np.abs(f["B"]).max(), 1e-30)
    assert np.abs(h["fit_B"] - f["B"]).max() <= TOL_FIT * Bn, "ridge B"
    O_sp = h["O_sp"][h["pos_q"]]                           # original order
    ref = O.apply_correction(O_sp, h["probe_idx"], D, f)
    err = row_rel_l2(h["out"], ref)
    assert err.max() <= TOL_FIT, f"corrected output max rel-L2 {err.max():.3e}"
    assert np.array_equal(h["out"][h["probe_idx"]], D)


def _tf32(x):
    """Round fp64 values (fp32-representable) to TF32, nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0xFFF) + ((u >> np.uint64(13)) & np.uint64(1))) & np.uint64(0xFFFFE000)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def check_factor_spectral(F, M, r, scale):
    """A metric factor F = U_r sqrt(Lambda_r) * scale checked without needing a
    spectral gap at r: its columns are orthogonal, each column f is an
    eigenvector of M with eigenvalue |f|^2 / scale^2, and those eigenvalues are
    the r largest of M.  Where eigenvalues cluster around the truncation rank,
    F F^T is not unique but these properties still hold (Weyl's bound)."""
    Fr = F[:, :r]
    lam = (Fr * Fr).sum(0) / scale ** 2
    w, _ = O.eigh_desc(M)
    top = w[0]
    assert np.all(np.abs(np.sort(lam)[::-1] - w[:r]) <= 2e-4 * top), "factor eigenvalues"
    G = Fr.T @ Fr
    off = G - np.diag(np.diag(G))
    assert np.abs(off).max() <= 2e-4 * top * scale ** 2, "factor columns not orthogonal"
    res = M @ Fr - Fr * lam[None, :]
    assert np.all(np.linalg.norm(res, axis=0) <= 1e-3 * top * np.linalg.norm(Fr, axis=0) + 1e-12), "eigen residual"
    assert np.all(F[:, r:] == 0.0)


def check_partition_floats(h, cfg, q, k, v, warm=None, semantic_keys=False, semantic_queries=False, M_K=None,
                           score_rows=None):
    """Float outputs of the partition against fp64 recomputation from the
    GPU's own integer decisions.  ``warm`` (F_K, F_Q of the state a warm call
    started from, fp64) switches the factor references to the warm factor;
    a semantic side has the raw rows (TF32-rounded) as coordinates and the
    identity as its factor.  ``M_K`` overrides the key metric (GQA: the
    metric the query heads of one K/V head share).  ``score_rows`` limits the
    routing-score comparison to those query groups (default: all).
    Returns which cold factors were compared.  Every cold factor gets the
    gap-free spectral check; F F^T is also compared with the truncated metric
    where the metric has a spectral gap at the truncation rank (without one,
    F F^T is not unique)."""
    kl, ql = h["kv_label"], h["q_label"]
    np.testing.assert_allclose(h["k_centroid"], O.group_means(k, kl, h["Ck"]), rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(h["v_centroid"], O.group_means(v, kl, h["Ck"]), rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(h["q_centroid"], O.group_means(q, ql, h["Cq"]), rtol=1e-4, atol=1e-5)
    # phi_K = K F_K with the GPU factor; phi_Q = RMSNorm(q F_Q) with its factor
    rq = O.query_rank(cfg.rQ, cfg.d, h["Ck"])
    if semantic_keys:
        assert np.array_equal(h["phi_K"], _tf32(k)) and np.array_equal(h["F_K"], np.eye(cfg.d))
    else:
        np.testing.assert_allclose(h["phi_K"], k @ h["F_K"], rtol=TOL_TF32, atol=1e-4 * np.abs(h["phi_K"]).max())
    if semantic_queries:
        assert np.array_equal(h["phi_Q"], _tf32(q)) and np.array_equal(h["F_Q"], np.eye(cfg.d))
    else:
        z = q @ h["F_Q"]
        rms = np.sqrt((z * z).sum(1) / rq)
        np.testing.assert_allclose(h["phi_Q"], z / np.maximum(rms, cfg.eps_rms)[:, None], rtol=TOL_TF32, atol=1e-4)
    _, dist = O.query_distances(h["phi_Q"], ql, h["Cq"])
    np.testing.assert_allclose(h["q_dist"], dist, rtol=1e-4, atol=1e-5)
    # metric factors: F F^T reproduces the (truncated) metric
    idx = O.sample_indices(cfg.N, cfg.Ms)
    MK = O.key_metric(q, idx) if M_K is None else M_K
    w, U = O.eigh_desc(MK)
    r = min(cfg.rK, cfg.d, len(idx))
    ref = U[:, :r] @ np.diag(w[:r]) @ U[:, :r].T / cfg.d
    FK = h["F_K"]
    gap_ok = (r == cfg.d or (w[r - 1] - w[r]) > 1e-2 * w[0]) and not semantic_keys
    Fw = None if warm is None else O.warm_factor(MK, warm["F_K"], r, 1.0 / math.sqrt(cfg.d))
    compared = {"F_K": False, "F_Q": False}
    if Fw is None and not semantic_keys:
        check_factor_spectral(FK, MK, r, 1.0 / math.sqrt(cfg.d))
        compared["F_K"] = True
    if Fw is not None:
        ref = Fw @ Fw.T
        assert np.abs(FK @ FK.T - ref).max() <= 2e-4 * np.abs(ref).max(), "warm F_K"
    elif gap_ok:
        assert np.abs(FK @ FK.T - ref).max() <= 2e-4 * np.abs(ref).max()
        compared["F_K"] = True
    MQ = O.query_metric(h["k_centroid"])
    wq, Uq = O.eigh_desc(MQ)
    refq = Uq[:, :rq] @ np.diag(wq[:rq]) @ Uq[:, :rq].T
    FQ = h["F_Q"]
    Fwq = None if warm is None else O.warm_factor(MQ, warm["F_Q"], rq, 1.0)
    if Fwq is None and not semantic_queries:
        check_factor_spectral(FQ, MQ, rq, 1.0)
        compared["F_Q"] = True
    if Fwq is not None:
        refq = Fwq @ Fwq.T
        assert np.abs(FQ @ FQ.T - refq).max() <= 2e-4 * np.abs(refq).max(), "warm F_Q"
    elif not semantic_queries and (rq >= int((wq > 1e-9 * wq[0]).sum()) or (wq[rq - 1] - wq[rq]) > 1e-2 * wq[0]):
        assert np.abs(FQ @ FQ.T - refq).max() <= 2e-4 * np.abs(refq).max()
        compared["F_Q"] = True
    # routing scores vs the direct sum on the GPU's groups and centroids
    rows = np.arange(h["Cq"]) if score_rows is None else np.asarray(score_rows)
    s_ref = O.routing_score(h["q_centroid"][rows], k, v, h["k_centroid"], h["v_centroid"], kl)
    scale = np.abs(s_ref).max(axis=1, keepdims=True)
    assert np.all(np.abs(h["score"][rows] - s_ref) <= 2e-4 * scale + 1e-30)
    return compared


def sample_rows(h, n, seed=0):
    """Permuted rows to check at full size: the first and last rows of the
    first and last query groups (ragged tails) and random rows."""
    N = len(h["perm_q"])
    off = h["q_offsets"]
    fixed = [0, 1, off[1] - 1, off[-2], N - 2, N - 1]
    rnd = np.random.default_rng(seed).choice(N, size=max(0, n - len(fixed)), replace=False)
    return np.unique(np.concatenate([fixed, rnd]).astype(np.int64))


def check_attention_rows(h, cfg, rows, tol):
    """Eq. (2) for the sampled permuted rows, each computed on its own."""
    klab_p = h["kv_label"][h["perm_kv"]]
    qgrp = np.searchsorted(h["q_offsets"], rows, side="right") - 1
    worst = 0.0
    for p, a in zip(rows, qgrp):
        keys = np.nonzero(h["mask"][a][klab_p])[0]
        ref = O.dense_attention(h["Qp"][p:p + 1], h["Kp"][keys], h["Vp"][keys])
        err = float(row_rel_l2(h["O_sp"][p:p + 1], ref)[0])
        worst = max(worst, err)
    assert worst <= tol, f"sampled sparse rows max rel-L2 {worst:.3e}"
    if cfg.Mp > 0:
        sel = np.unique(np.linspace(0, cfg.Mp - 1, 24).astype(np.int64))
        q = h["Qp"][h["pos_q"][h["probe_idx"][sel]]]
        dref = O.dense_attention(q, h["Kp"], h["Vp"])
        derr = row_rel_l2(h["probe_dense"][sel], dref)
        assert derr.max() <= tol, f"sampled probe rows max rel-L2 {derr.max():.3e}"
    return worst


def check_fit_and_apply_rows(h, cfg, rows):
    q_sizes = np.diff(h["q_offsets"])
    _, alpha, wt = O.coverage_weights(h["probe_group"], q_sizes, h["probe_alloc"], cfg.Mp)
    X, D = h["probe_sparse"], h["probe_dense"]
    f = O.ridge_fit(X, D - X, alpha, wt, cfg.lam, cfg.eps_std)
    assert np.abs(h["fit_B"] - f["B"]).max() <= TOL_FIT * np.abs(f["B"]).max()
    orig = h["perm_q"][rows]
    O_sp = h["O_sp"][rows]
    xb = (O_sp - f["mu_X"]) / f["sigma"]
    ref = O_sp + f["mu_R"] + xb @ f["B"]
    is_probe = np.isin(orig, h["probe_idx"])
    err = row_rel_l2(h["out"][orig][~is_probe], ref[~is_probe])
    assert err.max() <= TOL_FIT, f"sampled corrected rows max rel-L2 {err.max():.3e}"
