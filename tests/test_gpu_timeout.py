"""The device-timeout path of the attention kernel, made to run out without a
fault: the stall hook (sparsepr_debug_stall_attention) has every block first
wait a few polls on an mbarrier nothing signals.  The call must come back with
SPARSEPR_TIMEOUT in the workspace status word, the status read must clear it,
and the next call on the same workspace and context must be correct again."""

import numpy as np
import pytest
import torch

from synthetic.workloads import Workload

from gpu_parity_lib import run_staged, to_device

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

# bf16, d=128, N=2160: the tensor-core attention kernel, a few dozen blocks
CASE = Workload("timeout", 1, 2, 128, (3, 20, 36), "bf16", 24, 128, 0.22, 256, 100, 1.0, Cq=12, Ck=48, seed=31)


def test_timed_out_attention_reports_and_recovers():
    import free_block_sparse_sampled_b200 as S
    from free_block_sparse_sampled_b200 import _abi
    from synthetic import generate_inputs
    cfg = S.SparsePRConfig.from_workload(CASE)
    dev = to_device(CASE, generate_inputs(CASE))
    ref = run_staged(cfg, *dev)
    assert ref["status"] == 0
    ws, part, rt = ref["ws"], ref["part"], ref["route"]
    lib = _abi.lib()
    lib.sparsepr_debug_stall_attention(64)
    try:
        S.attention(cfg, part, rt, ws)
        torch.cuda.synchronize()
    finally:
        lib.sparsepr_debug_stall_attention(0)
    assert S.device_status(ws) == 5                  # SPARSEPR_TIMEOUT
    assert S.device_status(ws) == 0                  # the read cleared it
    O_sp, pd, _ = S.attention(cfg, part, rt, ws)
    torch.cuda.synchronize()
    assert S.device_status(ws) == 0
    assert torch.equal(O_sp, ref["O_sp"]) and torch.equal(pd, ref["probe_dense"])
    out, _ = S.call(cfg, *dev, ws)
    torch.cuda.synchronize()
    assert S.device_status(ws) == 0
    assert torch.equal(out, ref["out"])
