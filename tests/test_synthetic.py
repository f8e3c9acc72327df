"""The seeded input recipe does what the design states: deterministic per
(workload, head), bf16-exact for bf16 calls, logits q.k/sqrt(d) with standard
deviation 3 over random pairs, tokens grouped by generator clusters."""

import numpy as np

from synthetic import generate_head, generate_inputs, get_workload
from synthetic.video_grid import bf16_round


def test_heads_are_seeded_and_independent():
    w = get_workload("tiny")
    a = generate_head(w, 0, 0)
    b = generate_head(w, 0, 0)
    c = generate_head(w, 0, 1)
    for x, y, z in zip(a, b, c):
        assert np.array_equal(x, y) and not np.array_equal(x, z)
    q, k, v = generate_inputs(w)
    assert q.shape == (w.B, w.H, w.N, w.d)
    assert np.array_equal(q[0, 1], c[0])


def test_bf16_calls_are_bf16_exact():
    w = get_workload("mid", grid=(2, 8, 8), H=1)
    for x in generate_head(w, 0, 0):
        assert np.array_equal(bf16_round(x), x)


def test_logit_spread_matches_the_recipe():
    w = get_workload("mid", grid=(4, 16, 16), H=1)
    q, k, _ = (x.astype(np.float64) for x in generate_head(w, 0, 0))
    rng = np.random.default_rng(0)
    i, j = rng.integers(0, w.N, 20000), rng.integers(0, w.N, 20000)
    std = ((q[i] * k[j]).sum(1) / np.sqrt(w.d)).std()
    assert abs(std - w.logit_std) < 0.15 * w.logit_std


def test_tokens_of_one_patch_share_a_cluster_mostly():
    """Within a 4x4x4 patch most tokens (80 % before reassignment) share one
    generator cluster, so their keys sit near one centre."""
    w = get_workload("tiny")
    _, k, _ = generate_head(w, 0, 0)
    T, Y, X = w.grid
    kk = k.reshape(T, Y, X, w.d)
    patch = kk[:4, :4, :4].reshape(-1, w.d)
    other = kk[:4, 4:8, :4].reshape(-1, w.d)
    d_in = np.linalg.norm(patch - np.median(patch, axis=0), axis=1).mean()
    d_out = np.linalg.norm(other - np.median(patch, axis=0), axis=1).mean()
    assert d_in < d_out
