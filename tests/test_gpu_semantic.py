"""Semantic partition (paper §3 reference partition, Table 2 baseline) and
Table 2's key-response K/V variant on the GPU, through the C ABI: k-means on
the raw key and/or query rows, everything downstream unchanged.  Same checks
as the response-coupled parity tests."""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import generate_inputs
from synthetic.workloads import Workload

from gpu_parity_lib import (TOL_ATTN, TOL_ATTN_F32, check_attention, check_fit_and_apply, check_integer_chain,
                            check_kmeans_chain, check_partition_floats, head_view, run_staged, to_device)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

CASES = {
    "bf16_d128": Workload("sem_bf16_d128", 1, 2, 128, (3, 20, 36), "bf16", 24, 128, 0.22, 256, 100, 1.0,
                          Cq=12, Ck=48, seed=31),
    "bf16_d64": Workload("sem_bf16_d64", 1, 2, 64, (2, 16, 40), "bf16", 16, 128, 0.25, 128, 64, 1.0,
                         Cq=10, Ck=40, seed=32),
    "fp32_d64": Workload("sem_fp32_d64", 1, 2, 64, (4, 16, 16), "fp32", 16, 64, 0.25, 64, 32, 1e-3,
                         Cq=16, Ck=32, seed=33),
}


@pytest.mark.parametrize("variant", ["semantic", "key_response"])
@pytest.mark.parametrize("name", list(CASES))
def test_semantic_partition_every_stage(name, variant):
    from free_block_sparse_sampled_b200 import SparsePRConfig, _abi
    w = CASES[name]
    flags = _abi.FLAG_SEMANTIC_QUERIES | (_abi.FLAG_SEMANTIC_KEYS if variant == "semantic" else 0)
    cfg = SparsePRConfig.from_workload(w, flags=flags)
    q, k, v = generate_inputs(w)
    res = run_staged(cfg, *to_device(w, (q, k, v)), debug=True)
    assert res["status"] == 0
    tol = TOL_ATTN if w.dtype == "bf16" else TOL_ATTN_F32
    for bh in range(cfg.BH):
        b, h = divmod(bh, cfg.H)
        hv = head_view(res, cfg, bh)
        check_kmeans_chain(hv, cfg, "kv")
        check_kmeans_chain(hv, cfg, "q")
        check_integer_chain(hv, cfg)
        check_partition_floats(hv, cfg, q[b, h].astype(np.float64), k[b, h].astype(np.float64),
                               v[b, h].astype(np.float64), semantic_keys=variant == "semantic",
                               semantic_queries=True)
        check_attention(hv, cfg, tol)
        check_fit_and_apply(hv, cfg)


def test_semantic_first_assignment_matches_oracle():
    """bf16 rows are exact in TF32, so the GPU's first semantic assignment
    starts from the oracle's centres (the sampled raw rows): its labels are
    the oracle's except within fp32 rounding of a tie."""
    from free_block_sparse_sampled_b200 import SparsePRConfig, _abi
    w = CASES["bf16_d128"]
    cfg = SparsePRConfig.from_workload(w, flags=_abi.FLAG_SEMANTIC_KEYS | _abi.FLAG_SEMANTIC_QUERIES)
    q, k, v = generate_inputs(w)
    res = run_staged(cfg, *to_device(w, (q, k, v)), debug=True)
    for bh in range(cfg.BH):
        b, h = divmod(bh, cfg.H)
        hv = head_view(res, cfg, bh)
        for X, C, stage, hist in ((k[b, h], cfg.Ck, 0, hv["debug_kv_hist"]), (q[b, h], cfg.Cq, 1, hv["debug_q_hist"])):
            X = X.astype(np.float64)
            init = O.kmeans_init_indices(cfg.seed, bh, stage, C, cfg.N)
            ref, _ = O.kmeans_assign(X, X[init])
            assert (hist[0] == ref).mean() >= 0.999
