"""Parity at the full sizes of the large (N=118800, H=24) and wide (N=75600,
H=40) calls, in the launch configuration the benchmark times: integer chains
for two heads, and outputs on sampled rows that the oracle computes one by one."""

import numpy as np
import pytest
import torch

from synthetic import generate_inputs, get_workload

from gpu_parity_lib import (TOL_ATTN, check_attention_rows, check_fit_and_apply_rows, check_integer_chain,
                            head_view, run_staged, sample_rows, to_device)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)


@pytest.mark.parametrize("name", ["wide", "large"])
def test_full_size_call(name):
    from free_block_sparse_sampled_b200 import SparsePRConfig
    w = get_workload(name)
    cfg = SparsePRConfig.from_workload(w)
    qkv = generate_inputs(w, bits=True)
    dev = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for a in qkv]
    res = run_staged(cfg, *dev)
    assert res["status"] == 0
    ng = res["part"]["n_groups"].cpu().numpy()
    assert (ng[:, 0] >= 1).all() and (ng[:, 1] >= 1).all() and (ng[:, 0] <= w.Cq).all()
    for bh in (0, cfg.BH - 1):
        hv = head_view(res, cfg, bh)
        check_integer_chain(hv, cfg)
        rows = sample_rows(hv, 64, seed=bh)
        check_attention_rows(hv, cfg, rows, TOL_ATTN)
        check_fit_and_apply_rows(hv, cfg, rows)
    pairs = res["route"]["pairs"].cpu().numpy()
    rho = pairs[:, 1].sum() / (cfg.BH * cfg.N * cfg.N)
    assert rho >= w.density - 1e-9


def test_full_size_warm_call():
    """The wide call warm-started from the previous step's state (paper C.1,
    2 k-means assignments), in the configuration the benchmark's warm call
    times: integer chains for two heads and sampled output rows, each fed the
    GPU's own upstream values."""
    import free_block_sparse_sampled_b200 as S
    from synthetic import drift_inputs
    w = get_workload("wide")
    cfg0 = S.SparsePRConfig.from_workload(w)
    x0 = generate_inputs(w, bits=False)
    x1 = drift_inputs(w, x0, step=1)
    d0 = to_device(w, x0)
    ws = S.alloc_workspace(cfg0)
    p0 = S.partition(cfg0, *d0, ws, extras=True)
    state = {n: p0[n].clone() for n in ("F_K", "F_Q", "k_centroid", "q_centroid", "n_groups")}
    del p0, d0
    torch.cuda.synchronize()
    cfg = S.SparsePRConfig.from_workload(w, kmeans_iters=2)
    d1 = to_device(w, x1)
    part = S.partition(cfg, *d1, ws, warm=state)
    rt = S.route(cfg, part, ws)
    O_sp, pd, ps = S.attention(cfg, part, rt, ws)
    fit = S.probe_fit(cfg, part, rt, ps, pd, ws)
    out = S.apply(cfg, part, rt, O_sp, pd, fit, ws)
    torch.cuda.synchronize()
    res = {"part": part, "route": rt, "O_sp": O_sp, "probe_dense": pd, "probe_sparse": ps, "fit": fit, "out": out}
    assert S.device_status(ws) == 0
    assert (part["kmeans_iters_run"].cpu().numpy() <= 2).all()
    for bh in (0, cfg.BH - 1):
        hv = head_view(res, cfg, bh)
        check_integer_chain(hv, cfg)
        rows = sample_rows(hv, 48, seed=bh)
        check_attention_rows(hv, cfg, rows, TOL_ATTN)
        check_fit_and_apply_rows(hv, cfg, rows)
    pairs = rt["pairs"].cpu().numpy()
    assert pairs[:, 1].sum() / (cfg.BH * cfg.N * cfg.N) >= w.density - 1e-9
