"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Integer outputs (labels, compaction, permutation, selected cells, pair
counts, probes) must match bit-exactly when the oracle is fed the GPU's own
upstream fp32 values; floating-point outputs must match within the stated
tolerances: per-row relative L2 <= 2e-3 for bf16 attention with fp32
accumulation, <= 1e-4 for the fp32 ridge fit and corrected output."""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import generate_inputs, get_workload
from synthetic.workloads import Workload

from gpu_parity_lib import (TOL_ATTN, TOL_ATTN_F32, check_attention, check_fit_and_apply, check_integer_chain,
                            check_kmeans_chain, check_partition_floats, head_view, np64, row_rel_l2, run_staged,
                            to_device)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


def _cfg(w, **kw):
    from free_block_sparse_sampled_b200 import SparsePRConfig
    return SparsePRConfig.from_workload(w, **kw)


SMALL = {
    # fp32, d=64: the tiny call exactly (CUDA-core attention)
    "tiny": get_workload("tiny"),
    # bf16, d=128, N=2160 (ragged vs 128), several tiles per group
    "bf16_d128": Workload("bf16_d128", 1, 2, 128, (3, 20, 36), "bf16", 24, 128, 0.22, 256, 100, 1.0,
                          Cq=12, Ck=48, seed=11),
    # bf16, d=64 on the tensor-core kernel
    "bf16_d64": Workload("bf16_d64", 1, 2, 64, (2, 16, 40), "bf16", 16, 128, 0.25, 128, 64, 1.0,
                         Cq=10, Ck=40, seed=12),
    # bf16 with 64-row tiles (CUDA-core attention)
    "bf16_block64": Workload("bf16_block64", 2, 1, 128, (2, 12, 40), "bf16", 16, 64, 0.3, 128, 40, 0.5,
                             Cq=8, Ck=30, seed=13),
}


def _inputs(w):
    q, k, v = generate_inputs(w)
    return (q, k, v), to_device(w, (q, k, v))


@pytest.mark.parametrize("name", list(SMALL))
def test_small_call_every_stage(name):
    w = SMALL[name]
    cfg = _cfg(w)
    (q, k, v), (qd, kd, vd) = _inputs(w)
    res = run_staged(cfg, qd, kd, vd, debug=True)
    assert res["status"] == 0
    tol = TOL_ATTN if w.dtype == "bf16" else TOL_ATTN_F32
    for bh in range(cfg.BH):
        b, h = divmod(bh, cfg.H)
        hv = head_view(res, cfg, bh)
        check_kmeans_chain(hv, cfg, "kv")
        check_kmeans_chain(hv, cfg, "q")
        check_integer_chain(hv, cfg)
        check_partition_floats(hv, cfg, q[b, h].astype(np.float64), k[b, h].astype(np.float64),
                               v[b, h].astype(np.float64))
        check_attention(hv, cfg, tol)
        check_fit_and_apply(hv, cfg)


def test_tensor_core_matches_cuda_core_kernel():
    w = SMALL["bf16_d128"]
    cfg = _cfg(w)
    _, (qd, kd, vd) = _inputs(w)
    a = run_staged(cfg, qd, kd, vd)
    from free_block_sparse_sampled_b200 import _abi
    b = run_staged(_cfg(w, flags=_abi.FLAG_SIMT_ATTENTION), qd, kd, vd)
    assert torch.equal(a["route"]["mask"], b["route"]["mask"])
    err = row_rel_l2(np64(a["O_sp"].reshape(-1, cfg.d)), np64(b["O_sp"].reshape(-1, cfg.d)))
    assert err.max() <= TOL_ATTN
    errp = row_rel_l2(np64(a["probe_dense"].reshape(-1, cfg.d)), np64(b["probe_dense"].reshape(-1, cfg.d)))
    assert errp.max() <= TOL_ATTN


def test_fused_call_equals_staged_and_is_deterministic():
    import free_block_sparse_sampled_b200 as S
    w = SMALL["bf16_d128"]
    cfg = _cfg(w)
    _, (qd, kd, vd) = _inputs(w)
    staged = run_staged(cfg, qd, kd, vd)
    ws = S.alloc_workspace(cfg)
    o1, st = S.call(cfg, qd, kd, vd, ws, stats=True)
    o2, _ = S.call(cfg, qd, kd, vd, ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, staged["out"]) and torch.equal(o1, o2)
    assert st["pairs_route"] == int(staged["route"]["pairs"][:, 0].sum())
    assert st["pairs_exec"] - st["pairs_route"] == cfg.BH * cfg.Mp * cfg.N
    assert st["pairs_visited"] >= st["pairs_route"]
    assert S.device_status(ws) == 0


def test_full_density_is_dense_attention():
    w = SMALL["bf16_d128"]
    cfg = _cfg(w, density=1.0 + w.M / w.N)
    (q, k, v), (qd, kd, vd) = _inputs(w)
    res = run_staged(cfg, qd, kd, vd)
    ref = torch.nn.functional.scaled_dot_product_attention(qd.float(), kd.float(), vd.float())
    for bh in range(cfg.BH):
        hv = head_view(res, cfg, bh)
        assert hv["mask"].all()
        b, h = divmod(bh, cfg.H)
        dense = np64(ref[b, h])[hv["perm_q"]]
        assert row_rel_l2(hv["O_sp"], dense).max() <= TOL_ATTN


@pytest.mark.parametrize("case", ["no_probes", "all_probes", "one_group", "tiny_budget", "small_N",
                                  "more_centres_than_rows", "max_groups"])
def test_edge_cases(case):
    base = SMALL["bf16_d128"]
    over = {
        "no_probes": dict(M=0),
        "all_probes": dict(grid=(2, 8, 8), M=200, Cq=6, Ck=10, Ms=64),
        "one_group": dict(Cq=1, Ck=1),
        "tiny_budget": dict(density=0.001),
        "small_N": dict(grid=(4, 4, 4), M=16, Cq=4, Ck=8, Ms=32),
        "more_centres_than_rows": dict(grid=(1, 8, 12), M=10, Cq=150, Ck=200, Ms=64),
        "max_groups": dict(grid=(4, 32, 32), Cq=2048, Ck=2048, M=128, kmeans_iters=3),
    }[case]
    w = base.replace(name=case, **over)
    cfg = _cfg(w)
    (q, k, v), (qd, kd, vd) = _inputs(w)
    res = run_staged(cfg, qd, kd, vd, debug=case != "max_groups")
    assert res["status"] == 0
    for bh in range(cfg.BH):
        hv = head_view(res, cfg, bh)
        if case != "max_groups":
            check_kmeans_chain(hv, cfg, "kv")
            check_kmeans_chain(hv, cfg, "q")
        check_integer_chain(hv, cfg)
        check_attention(hv, cfg, TOL_ATTN)
        check_fit_and_apply(hv, cfg)
        if case == "all_probes":
            b, h = divmod(bh, cfg.H)
            dense = O.dense_attention(q[b, h].astype(np.float64), k[b, h].astype(np.float64),
                                      v[b, h].astype(np.float64))
            assert row_rel_l2(hv["out"], dense).max() <= TOL_ATTN
        if case == "one_group":
            assert hv["Cq"] == 1 and hv["Ck"] == 1 and hv["mask"].all()
        if case == "tiny_budget":
            assert (hv["sel_count"] == 1).all()


def test_mid_call_every_head():
    w = get_workload("mid")
    cfg = _cfg(w)
    (q, k, v), (qd, kd, vd) = _inputs(w)
    res = run_staged(cfg, qd, kd, vd, debug=True)
    assert res["status"] == 0
    for bh in range(cfg.BH):
        hv = head_view(res, cfg, bh)
        check_kmeans_chain(hv, cfg, "kv")
        check_kmeans_chain(hv, cfg, "q")
        check_integer_chain(hv, cfg)
        if bh < 2:
            check_partition_floats(hv, cfg, q[0, bh].astype(np.float64), k[0, bh].astype(np.float64),
                                   v[0, bh].astype(np.float64))
        check_attention(hv, cfg, TOL_ATTN)
        check_fit_and_apply(hv, cfg)


def test_host_pipeline_matches_device_call():
    """HostPipeline (host buffers, copies overlapped with compute) returns
    exactly what sparsepr_call returns on device-resident inputs."""
    import free_block_sparse_sampled_b200 as S
    w = SMALL["bf16_d128"]
    cfg = _cfg(w)
    q, k, v = generate_inputs(w)
    dq, dk, dv = to_device(w, (q, k, v))
    ws = S.alloc_workspace(cfg)
    ref, _ = S.call(cfg, dq, dk, dv, ws)
    torch.cuda.synchronize()
    hin = [t.cpu().pin_memory() for t in (dq, dk, dv)]
    outs = [torch.empty(ref.shape, dtype=torch.float32, pin_memory=True) for _ in range(3)]
    S.HostPipeline(cfg).run([hin] * 3, outs)
    for o in outs:
        assert torch.equal(o, ref.cpu())
