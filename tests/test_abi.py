"""C-ABI checks that need no GPU: the library loads, exports every function
include/sparsepr.h declares, validates arguments on the host, and the ctypes
struct layouts match the C layouts byte for byte."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparsepr.h")


@pytest.fixture(scope="module")
def L():
    from free_block_sparse_sampled_b200 import _abi, build
    if not os.path.exists(_abi.LIB_PATH):
        build.build()
    return _abi.lib()


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const char\*|sparsepr_status|size_t|void)\s+(sparsepr_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["sparsepr_partition", "sparsepr_route", "sparsepr_attention", "sparsepr_probe_fit",
              "sparsepr_apply", "sparsepr_call"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    from free_block_sparse_sampled_b200 import _abi
    names = _declared_functions()
    assert sorted(_abi.EXPORTED) == names
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (sparsepr_\w+)", out))
    assert set(names) <= exported


def _cfg(**kw):
    from free_block_sparse_sampled_b200 import SparsePRConfig
    base = dict(B=1, H=2, N=1024, d=64, T=4, Y=16, X=16, dtype="fp32", density=0.25, M=32, Ms=64, lam=1e-3,
                Cq=16, Ck=32, block=64)
    base.update(kw)
    return SparsePRConfig(**base)


def test_validation_codes(L):
    from free_block_sparse_sampled_b200 import validate
    assert validate(_cfg()) == 0
    assert validate(_cfg(N=1000)) == 1                  # N != T*Y*X
    assert validate(_cfg(d=96, N=1024)) == 2            # head dim not built
    assert validate(_cfg(lam=0.0)) == 1
    assert validate(_cfg(block=32)) == 1
    assert validate(_cfg(Cq=5000)) == 2
    assert validate(_cfg(rK=65)) == 2
    assert validate(_cfg(kmeans_iters=0)) == 1
    assert validate(_cfg(density=float("nan"))) == 1
    assert validate(_cfg(M=-1)) == 1
    # probe / correction variants, rank truncation, GQA
    assert validate(_cfg(probe_select="random")) == 0 and validate(_cfg(correction="mean")) == 0
    assert validate(_cfg(residual_rank=8)) == 0 and validate(_cfg(residual_rank=65)) == 1
    assert validate(_cfg(H=4, Hkv=2)) == 0
    assert validate(_cfg(H=4, Hkv=3)) == 1                    # H not a multiple of Hkv
    assert validate(_cfg(H=4, Hkv=-1)) == 1
    from free_block_sparse_sampled_b200 import _abi
    assert validate(_cfg(H=4, Hkv=2, flags=_abi.FLAG_WARM_START)) == 0


def test_workspace_size_and_host_errors(L):
    from free_block_sparse_sampled_b200 import _abi
    p = _cfg().c_params()
    n = L.sparsepr_workspace_size(ctypes.byref(p))
    assert n > 0 and n % 256 == 0
    bad = _cfg(N=999).c_params()
    assert L.sparsepr_workspace_size(ctypes.byref(bad)) == 0
    # host-side failures return before any CUDA call
    assert L.sparsepr_call(ctypes.byref(p), None, None, None, None, None, None, 0, None) == 1
    fake = ctypes.c_void_p(1 << 20)                     # aligned, never dereferenced
    q = ctypes.c_void_p(1 << 21)
    assert L.sparsepr_call(ctypes.byref(p), q, q, q, q, None, fake, 16, None) == 3
    assert L.sparsepr_call(ctypes.byref(p), q, q, q, q, None, ctypes.c_void_p((1 << 20) + 8), n, None) == 1
    assert L.sparsepr_call(ctypes.byref(bad), q, q, q, q, None, fake, n, None) == 1
    assert L.sparsepr_get_device_status(None, None, None) == 1
    # the warm-started partition checks its previous state before anything runs
    part = _abi.PartitionOut(*[q] * len(_abi.PARTITION_FIELDS))
    assert L.sparsepr_partition_warm(ctypes.byref(p), q, q, q, None, ctypes.byref(part), fake, n, None) == 1
    prev = _abi.WarmState(q, q, q, None, q)
    assert L.sparsepr_partition_warm(ctypes.byref(p), q, q, q, ctypes.byref(prev), ctypes.byref(part), fake, n,
                                     None) == 1
    assert L.sparsepr_partition_warm(ctypes.byref(p), q, q, q, ctypes.byref(prev), ctypes.byref(part), fake, 16,
                                     None) == 3
    # variant parameters change the workspace plan only where they add buffers
    n_rank = L.sparsepr_workspace_size(ctypes.byref(_cfg(residual_rank=8).c_params()))
    n_sem = L.sparsepr_workspace_size(ctypes.byref(_cfg(flags=_abi.FLAG_SEMANTIC_KEYS).c_params()))
    assert n_rank > n and n_sem >= n
    assert L.sparsepr_status_string(6) == b"ridge Gram matrix not positive definite"
    assert _abi.STATUS_NAMES[5] == "TIMEOUT"


def test_gqa_keeps_one_permuted_kv_per_kv_head(L):
    """Under GQA the permuted K and V and the fp16 copy of V are stored once
    per K/V head: the workspace of G = 4 query heads per K/V head is smaller
    by at least (G - 1)/G of those buffers (bf16 K, V and the fp16 V copy)."""
    H, G = 8, 4
    base = _cfg(H=H, dtype="bf16", d=128, block=128)
    n_mha = L.sparsepr_workspace_size(ctypes.byref(base.c_params()))
    n_gqa = L.sparsepr_workspace_size(ctypes.byref(_cfg(H=H, dtype="bf16", d=128, block=128, Hkv=H // G).c_params()))
    kv_bytes = 3 * base.B * H * base.N * base.d * 2   # Kp, Vp and the fp16 V copy per query head
    gqa_only = base.B * (H // G) * base.N * 4 + 256      # raw labels of the K/V heads' k-means
    assert 0 < n_gqa <= n_mha - kv_bytes * (G - 1) // G + gqa_only


def test_ctypes_layouts_match_c(L):
    from free_block_sparse_sampled_b200 import _abi
    structs = {"sparsepr_params": _abi.Params, "sparsepr_partition_out": _abi.PartitionOut,
               "sparsepr_route_out": _abi.RouteOut, "sparsepr_fit_out": _abi.FitOut, "sparsepr_stats": _abi.Stats,
               "sparsepr_warm_state": _abi.WarmState}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "sparsepr.h"', "int main(void) {"]
    for cname, py in structs.items():
        lines.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            cf = "lambda" if fname == "lambda_" else fname
            lines.append(f'printf("{cname}.{fname} %zu\\n", offsetof({cname}, {cf}));')
    lines.append("return 0; }")
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "probe.c")
        exe = os.path.join(td, "probe")
        open(src, "w").write("\n".join(lines))
        subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    got = dict(line.rsplit(" ", 1) for line in out.strip().splitlines())
    for cname, py in structs.items():
        assert int(got[cname]) == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert int(got[f"{cname}.{fname}"]) == getattr(py, fname).offset, (cname, fname)
