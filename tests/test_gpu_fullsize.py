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
