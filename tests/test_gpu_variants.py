"""Table 4 / D.3 / D.4 variants on the GPU through the C ABI: random and
uniform-grid probes, the restricted correction families and the rank-r
residual truncation.  Same checks as the parity tests; probes and fits are
compared with the oracle's variant on the GPU's own upstream values."""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import generate_inputs
from synthetic.workloads import Workload

from gpu_parity_lib import (TOL_ATTN, TOL_ATTN_F32, check_attention, check_fit_and_apply, check_integer_chain,
                            head_view, run_staged, to_device)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

W = Workload("var_bf16_d128", 1, 2, 128, (3, 20, 36), "bf16", 24, 128, 0.22, 256, 100, 1.0,
             Cq=12, Ck=48, seed=41, logit_std=1.5)
W32 = Workload("var_fp32_d64", 1, 2, 64, (4, 16, 16), "fp32", 16, 64, 0.25, 64, 40, 1e-3,
               Cq=16, Ck=32, seed=42)


def _run(w, **kw):
    from free_block_sparse_sampled_b200 import SparsePRConfig
    cfg = SparsePRConfig.from_workload(w, **kw)
    q, k, v = generate_inputs(w)
    res = run_staged(cfg, *to_device(w, (q, k, v)))
    assert res["status"] == 0
    return cfg, res


@pytest.mark.parametrize("w", [W, W32], ids=lambda w: w.name)
@pytest.mark.parametrize("probes", ["random", "uniform"])
def test_probe_variants(w, probes):
    cfg, res = _run(w, probe_select=probes)
    tol = TOL_ATTN if w.dtype == "bf16" else TOL_ATTN_F32
    for bh in range(cfg.BH):
        hv = head_view(res, cfg, bh)
        check_integer_chain(hv, cfg)
        check_attention(hv, cfg, tol)
        check_fit_and_apply(hv, cfg)


@pytest.mark.parametrize("family", ["diagonal", "scalar", "mean"])
def test_correction_families(family):
    cfg, res = _run(W, correction=family)
    for bh in range(cfg.BH):
        hv = head_view(res, cfg, bh)
        check_integer_chain(hv, cfg)
        check_fit_and_apply(hv, cfg)
        B = hv["fit_B"]
        assert not (B - np.diag(np.diag(B))).any()


def test_residual_rank_truncation():
    """Rank r at the widest gap of the weighted residual spectrum (so fp32
    eigenvectors are well conditioned); full rank leaves B unchanged."""
    from free_block_sparse_sampled_b200 import SparsePRConfig
    cfg0, res0 = _run(W)
    hv = head_view(res0, cfg0, 0)
    q_sizes = np.diff(hv["q_offsets"])
    _, alpha, wt = O.coverage_weights(hv["probe_group"], q_sizes, hv["probe_alloc"], cfg0.Mp)
    X, D = hv["probe_sparse"], hv["probe_dense"]
    f = O.ridge_fit(X, D - X, alpha, wt, cfg0.lam, cfg0.eps_std)
    s = np.linalg.svd(np.sqrt(wt)[:, None] * f["Rbar"], compute_uv=False)
    r = int(4 + np.argmax(s[4:32] / s[5:33]))
    cfg, res = _run(W, residual_rank=r)
    for bh in range(cfg.BH):
        hv = head_view(res, cfg, bh)
        check_fit_and_apply(hv, cfg)
    cfg_d, res_d = _run(W, residual_rank=W.d)
    assert torch.equal(res_d["fit"]["B"], res0["fit"]["B"])
