"""Python binding of the SparsePR C ABI.

torch supplies device memory and the current CUDA stream; every step of the
call runs in the CUDA library (libsparsepr.so).  There is no CPU path: if the
library is missing the first call raises.
"""

from __future__ import annotations

import ctypes
import dataclasses
from typing import Dict, Optional, Tuple

import torch

from . import _abi as A


@dataclasses.dataclass
class SparsePRConfig:
    """Problem statement of one call (paper §3-§4 notation)."""
    B: int
    H: int
    N: int
    d: int
    T: int
    Y: int
    X: int
    dtype: str = "bf16"          # storage of Q, K, V: "bf16" or "fp32"
    density: float = 0.22        # target executed-pair density incl. probes
    M: int = 64                  # probe rows per head
    Ms: int = 2048               # sampled queries for the key metric
    lam: float = 1.0             # ridge coefficient
    Cq: int = 300
    Ck: int = 1000
    rK: int = 48
    rQ: int = 64
    kmeans_iters: int = 25
    kmeans_tol: float = 1e-4
    seed: int = 1
    block: int = 128
    eps_rms: float = 1e-6
    eps_std: float = 1e-6
    flags: int = 0
    probe_select: str = "stratified"   # "stratified" (A.2), "random" or "uniform" (Table 4)
    correction: str = "full"           # "full", "diagonal", "scalar" or "mean" (D.4)
    residual_rank: int = 0             # 0: no truncation; r: rank-r residual projection (D.3)
    Hkv: int = 0                       # K/V heads (GQA): 0 = H; else a divisor of H

    @classmethod
    def from_workload(cls, w, **kw) -> "SparsePRConfig":
        T, Y, X = w.grid
        c = cls(B=w.B, H=w.H, N=w.N, d=w.d, T=T, Y=Y, X=X, dtype=w.dtype, density=w.density, M=w.M,
                Ms=w.Ms, lam=w.lam, Cq=w.Cq, Ck=w.Ck, rK=w.rK, rQ=w.rQ, kmeans_iters=w.kmeans_iters,
                kmeans_tol=w.kmeans_tol, seed=w.seed, block=w.block, eps_rms=w.eps_rms,
                eps_std=w.eps_std)
        return dataclasses.replace(c, **kw) if kw else c

    @property
    def BH(self) -> int:
        return self.B * self.H

    @property
    def Hk(self) -> int:
        """K/V heads."""
        return self.Hkv if self.Hkv else self.H

    @property
    def Mp(self) -> int:
        return min(self.M, self.N)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def RKp(self) -> int:
        if self.flags & A.FLAG_SEMANTIC_KEYS:
            return self.d
        r = min(self.rK, self.d, min(self.Ms, self.N))
        return max(32, (r + 15) // 16 * 16)

    @property
    def RQp(self) -> int:
        if self.flags & A.FLAG_SEMANTIC_QUERIES:
            return self.d
        return max(32, (min(self.rQ, self.d) + 15) // 16 * 16)

    def c_params(self) -> A.Params:
        return A.Params(self.B, self.H, self.N, self.d, self.T, self.Y, self.X,
                        A.BF16 if self.dtype == "bf16" else A.F32, float(self.density), self.M, self.Ms,
                        float(self.lam), self.Cq, self.Ck, self.rK, self.rQ, self.kmeans_iters,
                        float(self.kmeans_tol), int(self.seed) & ((1 << 64) - 1), self.block,
                        float(self.eps_rms), float(self.eps_std), self.flags, A.PROBES[self.probe_select],
                        A.CORRECTIONS[self.correction], int(self.residual_rank), int(self.Hkv))


def validate(cfg: SparsePRConfig) -> int:
    p = cfg.c_params()
    return A.lib().sparsepr_validate(ctypes.byref(p))


def workspace_bytes(cfg: SparsePRConfig) -> int:
    p = cfg.c_params()
    n = A.lib().sparsepr_workspace_size(ctypes.byref(p))
    if n == 0:
        A.check("sparsepr_workspace_size", A.lib().sparsepr_validate(ctypes.byref(p)) or 1)
    return int(n)


def alloc_workspace(cfg: SparsePRConfig, device="cuda") -> torch.Tensor:
    ws = torch.empty(workspace_bytes(cfg) + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + workspace_bytes(cfg)]


def _p(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check_qkv(cfg: SparsePRConfig, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> None:
    for t, h in ((q, cfg.H), (k, cfg.Hk), (v, cfg.Hk)):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == cfg.torch_dtype and
                tuple(t.shape) == (cfg.B, h, cfg.N, cfg.d)):
            raise ValueError("Q must be [B,H,N,d] and K/V [B,Hkv,N,d]: contiguous CUDA tensors of the config dtype")


def partition(cfg: SparsePRConfig, q, k, v, ws: torch.Tensor, debug: bool = False,
              extras: bool = False, warm: Optional[Dict[str, torch.Tensor]] = None) -> Dict[str, torch.Tensor]:
    """sparsepr_partition (or sparsepr_partition_warm when ``warm`` holds the
    F_K, F_Q, k_centroid, q_centroid and n_groups of an earlier partition of
    the same config): returns the outputs as tensors (per-head slices contiguous)."""
    _check_qkv(cfg, q, k, v)
    dev = q.device
    BH, N, d, Cq, Ck = cfg.BH, cfg.N, cfg.d, cfg.Cq, cfg.Ck
    i32 = dict(dtype=torch.int32, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    o = {
        # permuted K/V: one per K/V head (the G query heads of a K/V head share its groups)
        "Qp": torch.empty_like(q), "Kp": torch.empty_like(k), "Vp": torch.empty_like(v),
        "q_label": torch.empty(BH, N, **i32), "kv_label": torch.empty(BH, N, **i32),
        "perm_q": torch.empty(BH, N, **i32), "perm_kv": torch.empty(BH, N, **i32),
        "pos_q": torch.empty(BH, N, **i32), "q_offsets": torch.empty(BH, Cq + 1, **i32),
        "kv_offsets": torch.empty(BH, Ck + 1, **i32), "n_groups": torch.empty(BH, 2, **i32),
        "kmeans_iters_run": torch.empty(BH, 2, **i32), "q_centroid": torch.empty(BH, Cq, d, **f32),
        "k_centroid": torch.empty(BH, Ck, d, **f32), "v_centroid": torch.empty(BH, Ck, d, **f32),
        "q_dist": torch.empty(BH, N, **f32),
    }
    if extras or debug:
        o.update({"F_K": torch.empty(BH, d, cfg.RKp, **f32), "F_Q": torch.empty(BH, d, cfg.RQp, **f32),
                  "phi_K": torch.empty(BH, N, cfg.RKp, **f32), "phi_Q": torch.empty(BH, N, cfg.RQp, **f32),
                  "kv_centres": torch.empty(BH, Ck, cfg.RKp, **f32),
                  "q_centres": torch.empty(BH, Cq, cfg.RQp, **f32)})
    c = dataclasses.replace(cfg)
    if debug:
        c.flags |= A.FLAG_DEBUG_EXPORT
        o.update({"debug_kv_scores": torch.empty(BH, N, Ck, **f32),
                  "debug_q_scores": torch.empty(BH, N, Cq, **f32),
                  "debug_kv_hist": torch.full((BH, cfg.kmeans_iters, N), -1, **i32),
                  "debug_q_hist": torch.full((BH, cfg.kmeans_iters, N), -1, **i32)})
    s = A.PartitionOut(*[_p(o.get(n)) for n in A.PARTITION_FIELDS])
    p = c.c_params()
    if warm is None:
        A.check("sparsepr_partition", A.lib().sparsepr_partition(ctypes.byref(p), _p(q), _p(k), _p(v),
                                                                 ctypes.byref(s), _p(ws), ws.numel(), _stream()))
    else:
        shapes = {"F_K": (BH, d, cfg.RKp), "F_Q": (BH, d, cfg.RQp), "k_centroid": (BH, Ck, d),
                  "q_centroid": (BH, Cq, d), "n_groups": (BH, 2)}
        for n, shp in shapes.items():
            t = warm[n]
            want = torch.int32 if n == "n_groups" else torch.float32
            if not (t.is_cuda and t.is_contiguous() and t.dtype == want and tuple(t.shape) == shp):
                raise ValueError(f"warm[{n!r}] must be a contiguous CUDA {want} tensor of shape {shp}")
        ws_state = A.WarmState(*[_p(warm[n]) for n in A.WARM_FIELDS])
        A.check("sparsepr_partition_warm", A.lib().sparsepr_partition_warm(
            ctypes.byref(p), _p(q), _p(k), _p(v), ctypes.byref(ws_state), ctypes.byref(s), _p(ws), ws.numel(),
            _stream()))
        o["_warm_struct"] = ws_state
    o["_struct"] = s
    return o


def route(cfg: SparsePRConfig, part: Dict[str, torch.Tensor], ws: torch.Tensor) -> Dict[str, torch.Tensor]:
    dev = ws.device
    BH, Cq, Ck, Mp = cfg.BH, cfg.Cq, cfg.Ck, max(cfg.Mp, 1)
    r = {"score": torch.zeros(BH, Cq, Ck, dtype=torch.float32, device=dev),
         "mask": torch.zeros(BH, Cq, Ck, dtype=torch.uint8, device=dev),
         "sel_count": torch.zeros(BH, Cq, dtype=torch.int32, device=dev),
         "sel_groups": torch.full((BH, Cq, Ck), -1, dtype=torch.int32, device=dev),
         "pairs": torch.zeros(BH, 2, dtype=torch.int64, device=dev),
         "probe_idx": torch.full((BH, Mp), -1, dtype=torch.int32, device=dev),
         "probe_group": torch.full((BH, Mp), -1, dtype=torch.int32, device=dev),
         "probe_weight": torch.zeros(BH, Mp, dtype=torch.float32, device=dev),
         "probe_alloc": torch.zeros(BH, Cq, dtype=torch.int32, device=dev)}
    s = A.RouteOut(*[_p(r[n]) for n in A.ROUTE_FIELDS])
    p = cfg.c_params()
    A.check("sparsepr_route", A.lib().sparsepr_route(ctypes.byref(p), ctypes.byref(part["_struct"]),
                                                     ctypes.byref(s), _p(ws), ws.numel(), _stream()))
    r["_struct"] = s
    return r


def attention(cfg: SparsePRConfig, part, rt, ws: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    dev = ws.device
    BH, N, d, Mp = cfg.BH, cfg.N, cfg.d, max(cfg.Mp, 1)
    O_sp = torch.empty(BH, N, d, dtype=torch.float32, device=dev)
    pd = torch.empty(BH, Mp, d, dtype=torch.float32, device=dev)
    ps = torch.empty(BH, Mp, d, dtype=torch.float32, device=dev)
    p = cfg.c_params()
    A.check("sparsepr_attention", A.lib().sparsepr_attention(
        ctypes.byref(p), ctypes.byref(part["_struct"]), ctypes.byref(rt["_struct"]), _p(O_sp), _p(pd), _p(ps),
        _p(ws), ws.numel(), _stream()))
    return O_sp, pd, ps


def probe_fit(cfg: SparsePRConfig, part, rt, probe_sparse, probe_dense, ws: torch.Tensor) -> Dict[str, torch.Tensor]:
    dev = ws.device
    BH, d = cfg.BH, cfg.d
    f = {"B": torch.empty(BH, d, d, dtype=torch.float32, device=dev),
         "mu_x": torch.empty(BH, d, dtype=torch.float32, device=dev),
         "sigma": torch.empty(BH, d, dtype=torch.float32, device=dev),
         "mu_r": torch.empty(BH, d, dtype=torch.float32, device=dev)}
    s = A.FitOut(*[_p(f[n]) for n in A.FIT_FIELDS])
    p = cfg.c_params()
    A.check("sparsepr_probe_fit", A.lib().sparsepr_probe_fit(
        ctypes.byref(p), ctypes.byref(part["_struct"]), ctypes.byref(rt["_struct"]), _p(probe_sparse),
        _p(probe_dense), ctypes.byref(s), _p(ws), ws.numel(), _stream()))
    f["_struct"] = s
    return f


def probe_fit_static(cfg: SparsePRConfig, part, rt, probe_sparse, probe_dense, fit: Dict[str, torch.Tensor],
                     device_status: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """sparsepr_probe_fit_static: the probe fit with no workspace, for callers
    that cannot allocate device memory where they fit.  ``fit`` holds the
    caller's preallocated outputs (B, mu_x, sigma, mu_r); ``device_status`` an
    optional device int32 that receives the fit's status."""
    s = A.FitOut(*[_p(fit[n]) for n in A.FIT_FIELDS])
    p = cfg.c_params()
    A.check("sparsepr_probe_fit_static", A.lib().sparsepr_probe_fit_static(
        ctypes.byref(p), ctypes.byref(part["_struct"]), ctypes.byref(rt["_struct"]), _p(probe_sparse),
        _p(probe_dense), ctypes.byref(s), _p(device_status), _stream()))
    out = dict(fit)
    out["_struct"] = s
    return out


def apply(cfg: SparsePRConfig, part, rt, O_sp, probe_dense, fit, ws: torch.Tensor) -> torch.Tensor:
    out = torch.empty(cfg.B, cfg.H, cfg.N, cfg.d, dtype=torch.float32, device=ws.device)
    p = cfg.c_params()
    A.check("sparsepr_apply", A.lib().sparsepr_apply(
        ctypes.byref(p), ctypes.byref(part["_struct"]), ctypes.byref(rt["_struct"]), _p(O_sp), _p(probe_dense),
        ctypes.byref(fit["_struct"]), _p(out), _p(ws), ws.numel(), _stream()))
    return out


def call(cfg: SparsePRConfig, q, k, v, ws: torch.Tensor, out: Optional[torch.Tensor] = None,
         stats: bool = False):
    """sparsepr_call: the whole call on the current stream; returns (O, stats or None)."""
    _check_qkv(cfg, q, k, v)
    if out is None:
        out = torch.empty(cfg.B, cfg.H, cfg.N, cfg.d, dtype=torch.float32, device=q.device)
    st = A.Stats() if stats else None
    p = cfg.c_params()
    A.check("sparsepr_call", A.lib().sparsepr_call(
        ctypes.byref(p), _p(q), _p(k), _p(v), _p(out), ctypes.byref(st) if st is not None else None,
        _p(ws), ws.numel(), _stream()))
    if st is None:
        return out, None
    return out, {f: getattr(st, f) for f, _ in A.Stats._fields_}


def device_status(ws: torch.Tensor) -> int:
    v = ctypes.c_int32(0)
    A.check("sparsepr_get_device_status", A.lib().sparsepr_get_device_status(_p(ws), _stream(), ctypes.byref(v)))
    return int(v.value)


class HostPipeline:
    """A sequence of calls whose inputs and outputs live in pinned host memory.

    The inputs of call i + 1 are copied to the device on one stream while call
    i runs on another, and the output of call i is copied back on a third, so
    host<->device traffic overlaps compute.  Device inputs and outputs are
    double-buffered; one workspace serves every call (calls run in order on
    the compute stream)."""

    def __init__(self, cfg: SparsePRConfig, device="cuda"):
        self.cfg = cfg
        dev = torch.device(device)
        shape = (cfg.B, cfg.H, cfg.N, cfg.d)
        shapes = [shape, (cfg.B, cfg.Hk, cfg.N, cfg.d), (cfg.B, cfg.Hk, cfg.N, cfg.d)]
        self.din = [[torch.empty(sh, dtype=cfg.torch_dtype, device=dev) for sh in shapes] for _ in range(2)]
        self.dout = [torch.empty(shape, dtype=torch.float32, device=dev) for _ in range(2)]
        self.ws = alloc_workspace(cfg, dev)
        self.s_in, self.s_run, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev = lambda: [torch.cuda.Event() for _ in range(2)]
        self.in_ready, self.in_free, self.out_ready, self.out_free = ev(), ev(), ev(), ev()

    def run(self, inputs, outputs) -> None:
        """inputs: sequence of (q, k, v) pinned host tensors [B, H, N, d] in the
        call's dtype; outputs: matching pinned fp32 host tensors.  Returns once
        every output is on the host."""
        cur = torch.cuda.current_stream()
        for s in (self.s_in, self.s_run, self.s_out):
            s.wait_stream(cur)
        for i, ((hq, hk, hv), hout) in enumerate(zip(inputs, outputs)):
            b = i & 1
            with torch.cuda.stream(self.s_in):
                if i >= 2:
                    self.s_in.wait_event(self.in_free[b])      # call i - 2 no longer reads this buffer
                for dst, src in zip(self.din[b], (hq, hk, hv)):
                    dst.copy_(src, non_blocking=True)
                self.in_ready[b].record(self.s_in)
            with torch.cuda.stream(self.s_run):
                self.s_run.wait_event(self.in_ready[b])
                if i >= 2:
                    self.s_run.wait_event(self.out_free[b])    # call i - 2's output has left this buffer
                call(self.cfg, *self.din[b], self.ws, self.dout[b])
                self.in_free[b].record(self.s_run)
                self.out_ready[b].record(self.s_run)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.out_ready[b])
                hout.copy_(self.dout[b], non_blocking=True)
                self.out_free[b].record(self.s_out)
        for s in (self.s_in, self.s_run, self.s_out):
            cur.wait_stream(s)
        torch.cuda.synchronize()
