"""Parity on the sweep grid (B=2, H=16, N=32768 on an 8x64x64 grid, d=128,
bf16): executed-pair density 10/22/35/50 %, probe rows 64/256/1024 and
generator clusters 32/128/512.  For the first and last head of every setting
the integer chain must be bit-exact from the GPU's scores, and attention and
the corrected output must match the oracle on sampled rows.  The planted
variant replaces the probes' dense rows by a known rank-8 affine map of their
sparse rows and checks the GPU ridge fit against the oracle's on them."""

import numpy as np
import pytest
import torch

import oracle as O
from synthetic import generate_inputs, get_workload
from synthetic.video_grid import planted_map
from synthetic.workloads import sweep_workloads

from gpu_parity_lib import (TOL_ATTN, TOL_FIT, check_attention_rows, check_fit_and_apply_rows, check_integer_chain,
                            head_view, np64, npi, run_staged, sample_rows)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

SETTINGS = [w.name for w in sweep_workloads() if w.planted_rank == 0]


def _device_inputs(w):
    qkv = generate_inputs(w, bits=True)
    return [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for a in qkv]


@pytest.mark.parametrize("name", SETTINGS)
def test_sweep_setting(name):
    from free_block_sparse_sampled_b200 import SparsePRConfig
    w = get_workload(name)
    cfg = SparsePRConfig.from_workload(w)
    res = run_staged(cfg, *_device_inputs(w))
    assert res["status"] == 0
    for bh in (0, cfg.BH - 1):
        hv = head_view(res, cfg, bh)
        check_integer_chain(hv, cfg)
        rows = sample_rows(hv, 48, seed=bh)
        check_attention_rows(hv, cfg, rows, TOL_ATTN)
        check_fit_and_apply_rows(hv, cfg, rows)
    pairs = res["route"]["pairs"].cpu().numpy()
    assert pairs[:, 1].sum() / (cfg.BH * cfg.N * cfg.N) >= w.density - 1e-9


def test_sweep_planted_affine_fit():
    import free_block_sparse_sampled_b200 as S
    w = get_workload("sweep_planted")
    cfg = S.SparsePRConfig.from_workload(w)
    q, k, v = _device_inputs(w)
    ws = S.alloc_workspace(cfg)
    part = S.partition(cfg, q, k, v, ws)
    rt = S.route(cfg, part, ws)
    _, _, ps = S.attention(cfg, part, rt, ws)
    # planted dense probe rows: O_sp + b* + O_sp U V^T, per head
    X = ps.double().cpu().numpy().reshape(cfg.BH, cfg.Mp, cfg.d)
    D = np.empty_like(X)
    for bh in range(cfg.BH):
        b, h = divmod(bh, cfg.H)
        bstar, U, Vt = planted_map(w, b, h, rank=w.planted_rank)
        D[bh] = X[bh] + bstar + X[bh] @ U @ Vt
    pd = torch.from_numpy(D.astype(np.float32)).cuda()
    fit = S.probe_fit(cfg, part, rt, ps, pd, ws)
    torch.cuda.synchronize()
    assert S.device_status(ws) == 0
    for bh in (0, cfg.BH - 1):
        Cq2 = int(npi(part["n_groups"][bh])[0])
        q_sizes = np.diff(npi(part["q_offsets"][bh])[: Cq2 + 1])
        _, alpha, wt = O.coverage_weights(npi(rt["probe_group"][bh])[: cfg.Mp], q_sizes,
                                          npi(rt["probe_alloc"][bh])[:Cq2], cfg.Mp)
        Xf = X[bh].astype(np.float32).astype(np.float64)
        Df = D[bh].astype(np.float32).astype(np.float64)
        f = O.ridge_fit(Xf, Df - Xf, alpha, wt, cfg.lam, cfg.eps_std)
        Bg = np64(fit["B"][bh])
        assert np.abs(Bg - f["B"]).max() <= TOL_FIT * np.abs(f["B"]).max()
        # the fitted map reproduces the planted residual on the probes (ridge lambda = 1
        # against weights summing to M keeps the shrinkage small)
        Rhat = np64(fit["mu_r"][bh]) + ((Xf - np64(fit["mu_x"][bh])) / np64(fit["sigma"][bh])) @ Bg
        Rtrue = Df - Xf
        assert np.linalg.norm(Rhat - Rtrue) <= 0.05 * np.linalg.norm(Rtrue)
