"""Grouped-query attention (paper §4.3 "Routing and GQA", C.1) on the GPU,
through the C ABI: G = 2 query heads per K/V head share the key metric (the
mean of their sampled metrics), F_K and the K/V groups; query groups,
routing, probes and the fit stay per query head."""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import generate_inputs
from synthetic.workloads import Workload

from gpu_parity_lib import (TOL_ATTN, check_attention, check_fit_and_apply, check_integer_chain, check_kmeans_chain,
                            check_partition_floats, head_view, np64, run_staged, to_device)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

W = Workload("gqa_bf16_d128", 1, 4, 128, (3, 20, 36), "bf16", 24, 128, 0.22, 256, 100, 1.0,
             Cq=12, Ck=48, seed=51)
G = 2


def _inputs():
    q, k, v = generate_inputs(W)
    return q, np.ascontiguousarray(k[:, ::G]), np.ascontiguousarray(v[:, ::G])


def test_gqa_every_stage():
    from free_block_sparse_sampled_b200 import SparsePRConfig
    cfg = SparsePRConfig.from_workload(W, Hkv=W.H // G)
    q, k, v = _inputs()
    res = run_staged(cfg, *to_device(W, (q, k, v)), debug=True)
    assert res["status"] == 0
    p = res["part"]
    for bh in range(cfg.BH):
        b, h = divmod(bh, cfg.H)
        kvh = bh // G
        hv = head_view(res, cfg, bh)
        # K/V-side debug arrays are indexed by K/V head
        hv["debug_kv_scores"] = p["debug_kv_scores"][kvh].cpu().numpy()
        hv["debug_kv_hist"] = p["debug_kv_hist"][kvh].cpu().numpy().astype(np.int64)
        if bh % G:
            prev = head_view(res, cfg, bh - 1)
            assert np.array_equal(hv["kv_label"], prev["kv_label"])
            assert np.array_equal(hv["F_K"], prev["F_K"])
        check_kmeans_chain(hv, cfg, "kv")
        check_kmeans_chain(hv, cfg, "q")
        check_integer_chain(hv, cfg)
        qs = [q[b, (h // G) * G + g].astype(np.float64) for g in range(G)]
        MK = O.key_metric(np.concatenate(qs), O.sample_indices(G * cfg.N, G * cfg.Ms))
        check_partition_floats(hv, cfg, q[b, h].astype(np.float64), k[b, h // G].astype(np.float64),
                               v[b, h // G].astype(np.float64), M_K=MK)
        check_attention(hv, cfg, TOL_ATTN)
        check_fit_and_apply(hv, cfg)


def test_gqa_fused_call_equals_staged():
    import free_block_sparse_sampled_b200 as S
    cfg = S.SparsePRConfig.from_workload(W, Hkv=W.H // G)
    qd, kd, vd = to_device(W, _inputs())
    staged = run_staged(cfg, qd, kd, vd)
    ws = S.alloc_workspace(cfg)
    out, st = S.call(cfg, qd, kd, vd, ws, stats=True)
    torch.cuda.synchronize()
    assert torch.equal(out, staged["out"]) and S.device_status(ws) == 0
    assert st["pairs_exec"] - st["pairs_route"] == cfg.BH * cfg.Mp * cfg.N


def test_gqa_with_one_group_is_the_plain_call():
    """Hkv = H is the call without GQA."""
    import free_block_sparse_sampled_b200 as S
    q, k, v = generate_inputs(W)
    d = to_device(W, (q, k, v))
    a = run_staged(S.SparsePRConfig.from_workload(W), *d)
    b = run_staged(S.SparsePRConfig.from_workload(W, Hkv=W.H), *d)
    assert torch.equal(a["out"], b["out"])


def test_gqa_semantic_partition():
    """GQA with the semantic partition: the K/V head's raw keys are
    clustered once and the groups serve its G query heads."""
    from free_block_sparse_sampled_b200 import SparsePRConfig, _abi
    cfg = SparsePRConfig.from_workload(W, Hkv=W.H // G,
                                       flags=_abi.FLAG_SEMANTIC_KEYS | _abi.FLAG_SEMANTIC_QUERIES)
    q, k, v = _inputs()
    res = run_staged(cfg, *to_device(W, (q, k, v)), debug=True)
    assert res["status"] == 0
    p = res["part"]
    for bh in range(cfg.BH):
        b, h = divmod(bh, cfg.H)
        kvh = bh // G
        hv = head_view(res, cfg, bh)
        hv["debug_kv_scores"] = p["debug_kv_scores"][kvh].cpu().numpy()
        hv["debug_kv_hist"] = p["debug_kv_hist"][kvh].cpu().numpy().astype(np.int64)
        if bh % G:
            assert np.array_equal(hv["kv_label"], head_view(res, cfg, bh - 1)["kv_label"])
        check_kmeans_chain(hv, cfg, "kv")
        check_kmeans_chain(hv, cfg, "q")
        check_integer_chain(hv, cfg)
        check_partition_floats(hv, cfg, q[b, h].astype(np.float64), k[b, h // G].astype(np.float64),
                               v[b, h // G].astype(np.float64), semantic_keys=True, semantic_queries=True)
        check_attention(hv, cfg, TOL_ATTN)
        check_fit_and_apply(hv, cfg)
