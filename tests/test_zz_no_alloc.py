"""sparsepr_probe_fit_static: the probe fit with no caller workspace.

Some callers hold the partition and routing results but cannot allocate
device memory where they run the fit: their framework's caching allocator
owns all free HBM, or they must not take the device-wide synchronisation of
cudaMalloc/cudaFree.  This entry point keeps the fit's scratch in a static
device array instead.  These tests call it through the C ABI and compare it
with sparsepr_probe_fit, on two calls in a row on different inputs (the
array keeps the previous call's contents), and check that a call whose scratch
would exceed the array is refused before anything runs.

The file is named so that pytest collects it after every other test file.
"""

import ctypes

import numpy as np
import pytest
import torch

from synthetic import generate_inputs
from synthetic.workloads import Workload

TOL_FIT = 1e-4   # the fp32 ridge-fit tolerance of the parity tests

# bf16, d=128, N=2160, 2 heads: several query groups, 100 probes per head
CASE = Workload("no_alloc_fit", 1, 2, 128, (3, 20, 36), "bf16", 24, 128, 0.22, 256, 100, 1.0,
                Cq=12, Ck=48, seed=21)


def _lib_and_abi():
    from free_block_sparse_sampled_b200 import _abi as A
    return A.lib(), A


def _static_scratch_bytes(BH, d):
    up = lambda b: (b + 255) // 256 * 256
    return 256 + up(4 * BH) + up(24 * BH * d) + 2 * up(8 * BH * d * d)


def test_static_fit_refuses_oversized_call():
    """A call whose scratch would not fit the static array is refused on the
    host with SPARSEPR_UNSUPPORTED and a message naming both sizes."""
    lib, A = _lib_and_abi()
    from free_block_sparse_sampled_b200 import SparsePRConfig
    limit = A.FIT_STATIC_SCRATCH_BYTES
    H = 1
    while _static_scratch_bytes(H, 128) <= limit:
        H += 1
    cfg = SparsePRConfig.from_workload(CASE, H=H)
    p = cfg.c_params()
    fake = ctypes.c_void_p(256)   # never dereferenced: the size check comes first
    part = A.PartitionOut(*([fake] * len(A.PartitionOut._fields_)))
    rt = A.RouteOut(*([fake] * len(A.RouteOut._fields_)))
    fit = A.FitOut(*([fake] * len(A.FIT_FIELDS)))
    s = lib.sparsepr_probe_fit_static(ctypes.byref(p), ctypes.byref(part), ctypes.byref(rt), fake, fake,
                                      ctypes.byref(fit), None, None)
    assert A.STATUS_NAMES[s] == "UNSUPPORTED"
    msg = lib.sparsepr_last_error_string().decode()
    assert "sparsepr_probe_fit_static" in msg and str(limit) in msg


def test_static_fit_limit_matches_header():
    """The binding's copy of the array size is the header's."""
    import os
    import re
    _, A = _lib_and_abi()
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                            "sparsepr.h")).read()
    m = re.search(r"#define SPARSEPR_FIT_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    assert m is not None
    assert A.FIT_STATIC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def _fit_inputs(w):
    """Partition, routing and probe rows of workload ``w`` on the GPU, and the
    workspace fit of the same inputs as the reference."""
    import free_block_sparse_sampled_b200 as S
    from free_block_sparse_sampled_b200 import SparsePRConfig
    from synthetic.video_grid import bf16_bits
    _, A = _lib_and_abi()
    cfg = SparsePRConfig.from_workload(w)
    assert _static_scratch_bytes(cfg.BH, cfg.d) <= A.FIT_STATIC_SCRATCH_BYTES
    q, k, v = generate_inputs(w)
    dev = [torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda() for a in (q, k, v)]
    ws = S.alloc_workspace(cfg)
    part = S.partition(cfg, *dev, ws)
    rt = S.route(cfg, part, ws)
    _, pd, ps = S.attention(cfg, part, rt, ws)
    ref = S.probe_fit(cfg, part, rt, ps, pd, ws)
    torch.cuda.synchronize()
    assert S.device_status(ws) == 0
    return cfg, part, rt, ps, pd, ref


@pytest.mark.gpu
def test_static_fit_matches_workspace_fit_twice():
    """Two calls in a row on different inputs: three heads, then two heads of
    another seed.  Scratch the second call failed to rewrite would still hold
    the first call's values, which belong to other inputs, so each call is
    compared with the workspace fit of its own inputs."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from free_block_sparse_sampled_b200.api import _p, _stream
    lib, A = _lib_and_abi()
    names = ["B", "mu_x", "sigma", "mu_r"]
    for call, w in enumerate([CASE.replace(H=3), CASE.replace(name="no_alloc_fit_2", seed=22)]):
        cfg, part, rt, ps, pd, ref = _fit_inputs(w)
        # outputs start as NaN so that anything left unwritten shows
        out = {n: torch.full_like(ref[n], float("nan")) for n in names}
        st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        s = A.FitOut(*[_p(out[n]) for n in A.FIT_FIELDS])
        p = cfg.c_params()
        A.check("sparsepr_probe_fit_static", lib.sparsepr_probe_fit_static(
            ctypes.byref(p), ctypes.byref(part["_struct"]), ctypes.byref(rt["_struct"]), _p(ps), _p(pd),
            ctypes.byref(s), _p(st), _stream()))
        torch.cuda.synchronize()
        assert int(st.item()) == 0, f"call {call}: device status {int(st.item())}"
        for n in names:
            a, b = out[n].cpu().double().numpy(), ref[n].cpu().double().numpy()
            assert np.isfinite(a).all(), f"call {call}: {n} not finite"
            scale = max(np.abs(b).max(), 1e-30)
            err = np.abs(a - b).max() / scale
            assert err <= TOL_FIT, f"call {call}: {n} max error {err:.3e} of max |ref|"
