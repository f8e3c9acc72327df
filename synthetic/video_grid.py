"""Seeded synthetic Q/K/V on a (T, Y, X) video token grid.

Recipe (one independent stream per (b, h), seeded by (workload seed, b, h)):

* tokens are flattened row-major over (t, y, x);
* per axis, sin and cos at 8 geometric periods from 2 to 64 tokens give 48
  position features, mapped to d by one Gaussian projection scaled 1/sqrt(48);
* every 4x4x4 spatial-temporal patch belongs to one of C generator clusters
  (the patch index itself when ``patch_equals_cluster``, else a uniform draw);
  20% of tokens are then reassigned to a uniformly drawn cluster;
* cluster centres mu_c ~ N(0, I_d) are shared by Q and K;
* Q = s * (proj + mu_c + N(0, 0.5^2)),  K likewise with independent noise,
  where s makes the std of q.k/sqrt(d) over 4096 random pairs equal 3;
* V = N(0, 1) + 0.5 * mu_c.

bf16 workloads round Q, K, V to bf16 (round to nearest even) so that the CUDA
path and the oracle read bit-identical values.
"""

from __future__ import annotations

import concurrent.futures
import os

import numpy as np

from .workloads import Workload

_PERIODS = 2.0 * 32.0 ** (np.arange(8) / 7.0)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # finite inputs: the sum stays below 2^32
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return u.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _positions(grid):
    T, Y, X = grid
    t, y, x = np.meshgrid(np.arange(T), np.arange(Y), np.arange(X), indexing="ij")
    return t.ravel(), y.ravel(), x.ravel()


def _features(grid) -> np.ndarray:
    cols = []
    for pos in _positions(grid):
        ang = 2.0 * np.pi * pos[:, None].astype(np.float64) / _PERIODS[None, :]
        cols.append(np.sin(ang))
        cols.append(np.cos(ang))
    return np.concatenate(cols, axis=1).astype(np.float32)   # [N, 48]


def _clusters(w: Workload, rng) -> np.ndarray:
    T, Y, X = w.grid
    t, y, x = _positions(w.grid)
    nY, nX = -(-Y // 4), -(-X // 4)
    nT = -(-T // 4)
    patch = ((t // 4) * nY + (y // 4)) * nX + (x // 4)
    n_patches = nT * nY * nX
    if w.patch_equals_cluster:
        of_patch = np.arange(n_patches) % w.gen_clusters
    else:
        of_patch = rng.integers(0, w.gen_clusters, n_patches)
    cl = of_patch[patch].astype(np.int64)
    moved = rng.random(w.N) < 0.2
    cl[moved] = rng.integers(0, w.gen_clusters, int(moved.sum()))
    return cl


def generate_head(w: Workload, b: int, h: int):
    """Q, K, V for one head as float32 [N, d] (bf16-exact for bf16 workloads)."""
    rng = np.random.default_rng([int(w.seed), int(b), int(h), int(w.gen_clusters), 20260808])
    N, d = w.N, w.d
    feats = _features(w.grid)
    proj_w = rng.standard_normal((48, d), dtype=np.float32) / np.float32(np.sqrt(48.0))
    proj = feats @ proj_w
    cl = _clusters(w, rng)
    mu = rng.standard_normal((w.gen_clusters, d), dtype=np.float32)
    base = proj + mu[cl]
    q0 = base + np.float32(0.5) * rng.standard_normal((N, d), dtype=np.float32)
    k0 = base + np.float32(0.5) * rng.standard_normal((N, d), dtype=np.float32)
    i = rng.integers(0, N, 4096)
    j = rng.integers(0, N, 4096)
    lg = (q0[i].astype(np.float64) * k0[j].astype(np.float64)).sum(1) / np.sqrt(d)
    s = np.float32(np.sqrt(w.logit_std / lg.std()))
    q = s * q0
    k = s * k0
    v = rng.standard_normal((N, d), dtype=np.float32) + np.float32(0.5) * mu[cl]
    if w.dtype == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    return q.astype(np.float32), k.astype(np.float32), v.astype(np.float32)


def generate_inputs(w: Workload, heads=None, bits: bool = False):
    """Q, K, V as [B, H, N, d].

    ``heads``: optional list of (b, h) to fill (others stay zero) -- used to
    build bounded samples.  ``bits=True`` returns bf16 bit patterns (uint16)
    for bf16 workloads, halving host memory for the large calls.
    """
    use_bits = bits and w.dtype == "bf16"
    dt = np.uint16 if use_bits else np.float32
    out = [np.zeros((w.B, w.H, w.N, w.d), dtype=dt) for _ in range(3)]
    todo = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.H)]

    def fill(bh):
        b, h = bh
        for dst, src in zip(out, generate_head(w, b, h)):
            dst[b, h] = bf16_bits(src) if use_bits else src

    # heads draw from independent streams, so threads do not change the values
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, todo))
    return tuple(out)


def drift_inputs(w: Workload, qkv, step: int = 1, rel: float = 0.05):
    """Inputs of a later call of the same layer (the next denoising step):
    each of Q, K, V plus Gaussian noise of ``rel`` times its own std, from a
    stream seeded by (workload seed, step).  bf16 workloads are re-rounded."""
    rng = np.random.default_rng([int(w.seed), int(step), 515151])
    out = []
    for x in qkv:
        y = x + np.float32(rel) * np.float32(x.std()) * rng.standard_normal(x.shape, dtype=np.float32)
        out.append(bf16_round(y) if w.dtype == "bf16" else y.astype(np.float32))
    return tuple(out)


def planted_map(w: Workload, b: int, h: int, rank: int = 8, scale: float = 0.05):
    """Seeded affine map (b*, U, V^T) of rank ``rank`` for the planted variant:
    planted dense probe rows are  O_sp + b* + O_sp U V^T."""
    rng = np.random.default_rng([int(w.seed), int(b), int(h), 777, rank])
    d = w.d
    bstar = scale * rng.standard_normal(d)
    U = rng.standard_normal((d, rank)) / np.sqrt(d)
    Vt = scale * rng.standard_normal((rank, d))
    return bstar, U, Vt
