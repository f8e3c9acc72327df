"""Workload shapes and method settings for the SparsePR attention call.

Shapes follow the five synthetic video-grid calls this library is measured on.
Method settings follow Table C.1 of "Partition the Support, Reconstruct the
Residual" (C_q=300, C_k=1000, r_K=48, r_Q=64, lambda=1, 25 k-means iterations,
tolerance 1e-4) for the two calls whose token counts equal the paper's
HunyuanVideo (118,800) and Wan2.2 (75,600) sequence lengths (Table C.2); the
smaller calls scale the group counts down.  Values the paper leaves open
(epsilons, seeds, probe count per call, sample count) are fixed here once.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    grid: Tuple[int, int, int]          # T, Y, X  (N = T*Y*X, row-major (t,y,x))
    dtype: str                          # "fp32" or "bf16" storage of Q/K/V
    gen_clusters: int                   # clusters of the synthetic generator
    block: int                          # attention tile rows
    density: float                      # target executed-pair density incl. probes
    Ms: int                             # sampled queries for the key metric
    M: int                              # exact probe rows per head
    lam: float                          # ridge coefficient
    Cq: int                             # requested query groups
    Ck: int                             # requested K/V groups
    rK: int = 48
    rQ: int = 64
    kmeans_iters: int = 25
    kmeans_tol: float = 1e-4
    eps_rms: float = 1e-6
    eps_std: float = 1e-6
    seed: int = 1                       # generator seed (also k-means seed)
    patch_equals_cluster: bool = False  # tiny call: 4x4x4 patch index is the cluster
    logit_std: float = 3.0
    planted_rank: int = 0               # >0: planted affine residual variant

    @property
    def N(self) -> int:
        T, Y, X = self.grid
        return T * Y * X

    @property
    def BH(self) -> int:
        return self.B * self.H

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # B=1, H=2, d=64, fp32, grid 4x16x16 (N=1024); 16 generator clusters,
    # block 64, density 25% incl. probes, 64 sampled queries, 32 probes, lambda 1e-3.
    "tiny": Workload("tiny", 1, 2, 64, (4, 16, 16), "fp32", 16, 64, 0.25, 64, 32,
                     1e-3, Cq=16, Ck=32, seed=1, patch_equals_cluster=True),
    # B=1, H=8, d=128, bf16, grid 8x32x32 (N=8192); 64 clusters, block 128,
    # density 22%, 256 sampled queries, 128 probes.
    "mid": Workload("mid", 1, 8, 128, (8, 32, 32), "bf16", 64, 128, 0.22, 256, 128,
                    1.0, Cq=32, Ck=128, seed=2),
    # Video-DiT-shaped call: B=1, H=24, grid 33x45x80 (N=118800, ragged vs 128).
    "large": Workload("large", 1, 24, 128, (33, 45, 80), "bf16", 256, 128, 0.22, 1024,
                      512, 1.0, Cq=300, Ck=1000, seed=3),
    # Wide-head call: B=1, H=40, grid 21x45x80 (N=75600).
    "wide": Workload("wide", 1, 40, 128, (21, 45, 80), "bf16", 192, 128, 0.22, 1024,
                     512, 1.0, Cq=300, Ck=1000, seed=4),
    "wide26": Workload("wide26", 1, 40, 128, (21, 45, 80), "bf16", 192, 128, 0.26, 1024,
                       512, 1.0, Cq=300, Ck=1000, seed=4),
    # Sweep base: B=2, H=16, grid 8x64x64 (N=32768); density / probes / generator
    # clusters are varied by sweep_workloads().
    "sweep": Workload("sweep", 2, 16, 128, (8, 64, 64), "bf16", 128, 128, 0.22, 1024,
                      256, 1.0, Cq=128, Ck=384, seed=5),
}


def sweep_workloads():
    """The sweep grid: density x probe rows x generator clusters, plus the
    planted rank-8 affine residual variant."""
    base = WORKLOADS["sweep"]
    out = []
    for dens in (0.10, 0.22, 0.35, 0.50):
        out.append(base.replace(name=f"sweep_rho{int(dens*100)}", density=dens))
    for m in (64, 256, 1024):
        out.append(base.replace(name=f"sweep_M{m}", M=m))
    for c in (32, 128, 512):
        out.append(base.replace(name=f"sweep_C{c}", gen_clusters=c))
    out.append(base.replace(name="sweep_planted", planted_rank=8))
    return out


def get_workload(name: str, **overrides) -> Workload:
    if name in WORKLOADS:
        w = WORKLOADS[name]
    else:
        table = {w.name: w for w in sweep_workloads()}
        w = table[name]
    return w.replace(**overrides) if overrides else w


def scaled(w: Workload, grid: Tuple[int, int, int], H: Optional[int] = None,
           **kw) -> Workload:
    """A smaller call with the same generator recipe (for parity tests)."""
    return w.replace(grid=grid, H=H if H is not None else w.H, **kw)
