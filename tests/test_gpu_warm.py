"""Warm-started partition (paper C.1 warm start, Table C.1 limit of 2
assignments after the first call) on the GPU, through the C ABI.

The state a warm call starts from comes from the oracle's cold call on the
previous step's inputs (rounded to fp32 as the C ABI stores it), so no
expected value or input comes from the CUDA path.  The warm call runs on the
next step's inputs (the previous ones plus a small seeded drift).  Checks:
the warm factors against the oracle's subspace iteration on the same metric,
the initial centres against the oracle's projection of the previous
centroids, and every downstream stage as in the cold parity tests."""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import drift_inputs, generate_inputs
from synthetic.workloads import Workload

from gpu_parity_lib import (TOL_ATTN, TOL_TF32, check_attention, check_fit_and_apply, check_integer_chain,
                            check_kmeans_chain, check_partition_floats, head_view, np64, npi, to_device)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

W = Workload("warm_bf16_d128", 1, 2, 128, (3, 20, 36), "bf16", 24, 128, 0.22, 256, 100, 1.0,
             Cq=12, Ck=48, seed=21)
W64 = Workload("warm_bf16_d64", 1, 2, 64, (2, 16, 40), "bf16", 16, 128, 0.25, 128, 64, 1.0,
               Cq=10, Ck=40, seed=22)


def _cfg(w, **kw):
    from free_block_sparse_sampled_b200 import SparsePRConfig
    return SparsePRConfig.from_workload(w, **kw)


def _oracle_state(w, cfg, qkv):
    """Oracle cold call per head -> warm-state tensors in the C ABI layout."""
    q, k, v = qkv
    kw = O.workload_kwargs(w)
    BH, d = cfg.BH, cfg.d
    FK = np.zeros((BH, d, cfg.RKp), np.float32)
    FQ = np.zeros((BH, d, cfg.RQp), np.float32)
    kc = np.zeros((BH, cfg.Ck, d), np.float32)
    qc = np.zeros((BH, cfg.Cq, d), np.float32)
    ng = np.zeros((BH, 2), np.int32)
    for bh in range(BH):
        b, h = divmod(bh, cfg.H)
        r = O.sparsepr_head(q[b, h].astype(np.float64), k[b, h].astype(np.float64), v[b, h].astype(np.float64),
                            bh=bh, **kw)
        FK[bh, :, :r["F_K"].shape[1]] = r["F_K"]
        FQ[bh, :, :r["F_Q"].shape[1]] = r["F_Q"]
        kc[bh, :r["Ck"]] = r["kbar"]
        qc[bh, :r["Cq"]] = r["qbar"]
        ng[bh] = (r["Cq"], r["Ck"])
    t = {"F_K": FK, "F_Q": FQ, "k_centroid": kc, "q_centroid": qc, "n_groups": ng}
    return {n: torch.from_numpy(a).cuda() for n, a in t.items()}


def _run(cfg, qd, kd, vd, warm, debug=True):
    import free_block_sparse_sampled_b200 as S
    ws = S.alloc_workspace(cfg)
    part = S.partition(cfg, qd, kd, vd, ws, debug=debug, extras=True, warm=warm)
    rt = S.route(cfg, part, ws)
    O_sp, pd, ps = S.attention(cfg, part, rt, ws)
    fit = S.probe_fit(cfg, part, rt, ps, pd, ws)
    out = S.apply(cfg, part, rt, O_sp, pd, fit, ws)
    torch.cuda.synchronize()
    return {"part": part, "route": rt, "O_sp": O_sp, "probe_dense": pd, "probe_sparse": ps, "fit": fit,
            "out": out, "status": S.device_status(ws), "ws": ws}


def _state64(warm, bh, cfg):
    return {"F_K": np64(warm["F_K"][bh]), "F_Q": np64(warm["F_Q"][bh]),
            "kbar": np64(warm["k_centroid"][bh]), "qbar": np64(warm["q_centroid"][bh]),
            "ng": npi(warm["n_groups"][bh])}


@pytest.mark.parametrize("w", [W, W64], ids=lambda w: w.name)
def test_warm_call_every_stage(w):
    x0 = generate_inputs(w)
    x1 = drift_inputs(w, x0, step=1)
    cfg0 = _cfg(w)
    warm = _oracle_state(w, cfg0, x0)
    cfg = _cfg(w, kmeans_iters=2)
    qd, kd, vd = to_device(w, x1)
    res = _run(cfg, qd, kd, vd, warm)
    assert res["status"] == 0
    q, k, v = (a.astype(np.float64) for a in x1)
    for bh in range(cfg.BH):
        b, h = divmod(bh, cfg.H)
        hv = head_view(res, cfg, bh)
        st = _state64(warm, bh, cfg)
        assert (hv["iters"] <= 2).all() and (hv["iters"] >= 1).all()
        check_kmeans_chain(hv, cfg, "kv")
        check_kmeans_chain(hv, cfg, "q")
        check_integer_chain(hv, cfg)
        rq_prev = O.query_rank(cfg.rQ, cfg.d, int(st["ng"][1]))
        check_partition_floats(hv, cfg, q[b, h], k[b, h], v[b, h],
                               warm={"F_K": st["F_K"][:, :cfg.RKp], "F_Q": st["F_Q"][:, :rq_prev]})
        check_attention(hv, cfg, TOL_ATTN)
        check_fit_and_apply(hv, cfg)


def test_warm_initial_centres():
    """One assignment: the exported centres are the initial ones."""
    w = W
    x0 = generate_inputs(w)
    x1 = drift_inputs(w, x0, step=1)
    warm = _oracle_state(w, _cfg(w), x0)
    cfg = _cfg(w, kmeans_iters=1)
    res = _run(cfg, *to_device(w, x1), warm)
    assert res["status"] == 0
    for bh in range(cfg.BH):
        hv = head_view(res, cfg, bh)
        st = _state64(warm, bh, cfg)
        Cq_prev, Ck_prev = (int(x) for x in st["ng"])
        # K/V side: kbar_b F_K for b < C_k'(prev), sampled rows after
        init_k = O.kmeans_init_indices(cfg.seed, bh, 0, cfg.Ck, cfg.N)
        ref = O.warm_centres(hv["phi_K"], st["kbar"][:Ck_prev], hv["F_K"], cfg.Ck, init_k)
        np.testing.assert_allclose(hv["kv_centres"], ref, rtol=TOL_TF32, atol=1e-4 * np.abs(ref).max())
        np.testing.assert_array_equal(hv["kv_centres"][Ck_prev:], hv["phi_K"][init_k[Ck_prev:]])
        # query side: RMSNorm(qbar_a F_Q) over this call's r_Q'
        rq = O.query_rank(cfg.rQ, cfg.d, hv["Ck"])
        init_q = O.kmeans_init_indices(cfg.seed, bh, 1, cfg.Cq, cfg.N)
        refq = O.warm_centres(hv["phi_Q"][:, :rq], st["qbar"][:Cq_prev], hv["F_Q"][:, :rq], cfg.Cq, init_q,
                              rms_eps=cfg.eps_rms)
        np.testing.assert_allclose(hv["q_centres"][:, :rq], refq, rtol=TOL_TF32, atol=1e-4)
        assert not hv["q_centres"][:, rq:].any()


def test_warm_factor_falls_back_to_cold_on_vanishing_pivot():
    """A previous state with zero factors cannot be iterated: every head takes
    the cold eigen-factor (the centres still start from the previous centroids)."""
    w = W
    x0 = generate_inputs(w)
    warm = _oracle_state(w, _cfg(w), x0)
    warm["F_K"].zero_()
    warm["F_Q"].zero_()
    cfg = _cfg(w, kmeans_iters=2)
    res = _run(cfg, *to_device(w, x0), warm)
    assert res["status"] == 0
    q, k, v = (a.astype(np.float64) for a in x0)
    for bh in range(cfg.BH):
        b, h = divmod(bh, cfg.H)
        hv = head_view(res, cfg, bh)
        check_integer_chain(hv, cfg)
        check_partition_floats(hv, cfg, q[b, h], k[b, h], v[b, h])   # cold factor references


def test_fused_warm_call_matches_staged_warm_partition():
    """sparsepr_call with the warm flag reads the previous fused call's state
    from its workspace: same output as the staged path given that state
    explicitly; on a workspace without a complete state it is the cold call."""
    import free_block_sparse_sampled_b200 as S
    from free_block_sparse_sampled_b200 import _abi
    w = W
    x0 = generate_inputs(w)
    x1 = drift_inputs(w, x0, step=1)
    d0, d1 = to_device(w, x0), to_device(w, x1)
    cold_cfg = _cfg(w)
    warm_cfg = _cfg(w, kmeans_iters=2, flags=_abi.FLAG_WARM_START)
    plain_cfg = _cfg(w, kmeans_iters=2)
    # fused: cold call on x0, then warm call on x1 in the same workspace
    ws = S.alloc_workspace(cold_cfg)
    S.call(cold_cfg, *d0, ws)
    o_warm, _ = S.call(warm_cfg, *d1, ws)
    # staged: cold partition of x0 gives the state explicitly
    ws2 = S.alloc_workspace(cold_cfg)
    p0 = S.partition(cold_cfg, *d0, ws2, extras=True)
    state = {n: p0[n].clone() for n in ("F_K", "F_Q", "k_centroid", "q_centroid", "n_groups")}
    part = S.partition(plain_cfg, *d1, ws2, warm=state)
    rt = S.route(plain_cfg, part, ws2)
    O_sp, pd, ps = S.attention(plain_cfg, part, rt, ws2)
    fit = S.probe_fit(plain_cfg, part, rt, ps, pd, ws2)
    o_staged = S.apply(plain_cfg, part, rt, O_sp, pd, fit, ws2)
    torch.cuda.synchronize()
    assert S.device_status(ws) == 0 and S.device_status(ws2) == 0
    assert torch.equal(o_warm, o_staged)
    # a staged partition leaves no fused state: the warm flag then runs cold
    o_cold, _ = S.call(plain_cfg, *d1, ws2)
    S.partition(cold_cfg, *d0, ws2)
    o_flag, _ = S.call(warm_cfg, *d1, ws2)
    torch.cuda.synchronize()
    assert torch.equal(o_flag, o_cold)


WG = Workload("warm_gqa_bf16_d128", 1, 4, 128, (3, 20, 36), "bf16", 24, 128, 0.22, 256, 100, 1.0,
              Cq=12, Ck=48, seed=23)
G = 2


def _gqa_inputs(step):
    q, k, v = generate_inputs(WG)
    x0 = (q, np.ascontiguousarray(k[:, ::G]), np.ascontiguousarray(v[:, ::G]))
    return x0 if step == 0 else drift_inputs(WG, x0, step=step)


def test_warm_call_under_gqa():
    """GQA (G = 2) warm-started from the oracle's cold GQA call: K/V head h
    starts from query head h*G's state; every stage checked as above, with
    the shared key metric."""
    from free_block_sparse_sampled_b200 import SparsePRConfig
    x0, x1 = _gqa_inputs(0), _gqa_inputs(1)
    cfg0 = SparsePRConfig.from_workload(WG, Hkv=WG.H // G)
    kw = O.workload_kwargs(WG)
    Ms = kw.pop("Ms")
    BH, d = cfg0.BH, cfg0.d
    st = {"F_K": np.zeros((BH, d, cfg0.RKp), np.float32), "F_Q": np.zeros((BH, d, cfg0.RQp), np.float32),
          "k_centroid": np.zeros((BH, cfg0.Ck, d), np.float32), "q_centroid": np.zeros((BH, cfg0.Cq, d), np.float32),
          "n_groups": np.zeros((BH, 2), np.int32)}
    q0, k0, v0 = (a.astype(np.float64) for a in x0)
    for b in range(WG.B):
        for h in range(WG.H // G):
            kvh = b * (WG.H // G) + h
            res = O.sparsepr_gqa([q0[b, h * G + g] for g in range(G)], k0[b, h], v0[b, h], kvh=kvh, Ms=Ms, **kw)
            for g, r in enumerate(res):
                bh = kvh * G + g
                st["F_K"][bh, :, :r["F_K"].shape[1]] = r["F_K"]
                st["F_Q"][bh, :, :r["F_Q"].shape[1]] = r["F_Q"]
                st["k_centroid"][bh, :r["Ck"]] = r["kbar"]
                st["q_centroid"][bh, :r["Cq"]] = r["qbar"]
                st["n_groups"][bh] = (r["Cq"], r["Ck"])
    warm = {n: torch.from_numpy(a).cuda() for n, a in st.items()}
    cfg = SparsePRConfig.from_workload(WG, Hkv=WG.H // G, kmeans_iters=2)
    res = _run(cfg, *to_device(WG, x1), warm)
    assert res["status"] == 0
    q, k, v = (a.astype(np.float64) for a in x1)
    p = res["part"]
    for bh in range(cfg.BH):
        b, h = divmod(bh, cfg.H)
        kvh = bh // G
        hv = head_view(res, cfg, bh)
        hv["debug_kv_scores"] = p["debug_kv_scores"][kvh].cpu().numpy()
        hv["debug_kv_hist"] = p["debug_kv_hist"][kvh].cpu().numpy().astype(np.int64)
        assert (hv["iters"] <= 2).all()
        check_kmeans_chain(hv, cfg, "kv")
        check_kmeans_chain(hv, cfg, "q")
        check_integer_chain(hv, cfg)
        qs = [q[b, (h // G) * G + g] for g in range(G)]
        MK = O.key_metric(np.concatenate(qs), O.sample_indices(G * cfg.N, G * cfg.Ms))
        rq_prev = O.query_rank(cfg.rQ, cfg.d, int(st["n_groups"][bh][1]))
        check_partition_floats(hv, cfg, q[b, h], k[b, h // G], v[b, h // G], M_K=MK,
                               warm={"F_K": st["F_K"][kvh * G].astype(np.float64),
                                     "F_Q": st["F_Q"][bh][:, :rq_prev].astype(np.float64)})
        check_attention(hv, cfg, TOL_ATTN)
        check_fit_and_apply(hv, cfg)


def test_fused_warm_call_under_gqa_matches_staged():
    """The fused call keeps F_K per K/V head in its workspace and reads the
    centroids per query head: same output as the staged path with the state
    of a staged cold partition."""
    import free_block_sparse_sampled_b200 as S
    from free_block_sparse_sampled_b200 import _abi
    d0, d1 = to_device(WG, _gqa_inputs(0)), to_device(WG, _gqa_inputs(1))
    cold_cfg = _cfg(WG, Hkv=WG.H // G)
    warm_cfg = _cfg(WG, Hkv=WG.H // G, kmeans_iters=2, flags=_abi.FLAG_WARM_START)
    plain_cfg = _cfg(WG, Hkv=WG.H // G, kmeans_iters=2)
    ws = S.alloc_workspace(cold_cfg)
    S.call(cold_cfg, *d0, ws)
    o_warm, _ = S.call(warm_cfg, *d1, ws)
    ws2 = S.alloc_workspace(cold_cfg)
    p0 = S.partition(cold_cfg, *d0, ws2, extras=True)
    state = {n: p0[n].clone() for n in ("F_K", "F_Q", "k_centroid", "q_centroid", "n_groups")}
    part = S.partition(plain_cfg, *d1, ws2, warm=state)
    rt = S.route(plain_cfg, part, ws2)
    O_sp, pd, ps = S.attention(plain_cfg, part, rt, ws2)
    fit = S.probe_fit(plain_cfg, part, rt, ps, pd, ws2)
    o_staged = S.apply(plain_cfg, part, rt, O_sp, pd, fit, ws2)
    torch.cuda.synchronize()
    assert S.device_status(ws) == 0 and S.device_status(ws2) == 0
    assert torch.equal(o_warm, o_staged)
