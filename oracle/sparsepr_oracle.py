"""fp64 CPU oracle of one SparsePR attention call, one head at a time.

TEST INFRASTRUCTURE.  This module is only imported by ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``.  It does
not import the CUDA library and shares no code with it.

Every function restates one step of "Partition the Support, Reconstruct the
Residual: Training-Free Sparse Attention for Video Generation and World
Models" (Taghavi, Langari, Pandey; arXiv 2608.18484v2), cited as "paper" with
its section and formula.  Steps are plain numpy in float64; library routines
(matmul, eigh, argsort, cholesky/solve, svd) serve as single steps.  There is
no blocking, fusion or reordering beyond what the paper states.

Readings of passages the paper leaves open (each also listed in the design
notes of the repository):

R1  Sampled queries are evenly spaced rows s_t = floor(t N / M_s) (paper C.2:
    "evenly spaced rows", all rows when fewer are available).
R2  The common positive scale of phi_K is 1/sqrt(d), so squared distances are
    mean squared logit differences over the samples (paper §4.1).
R3  k-means: initial centres are rows drawn uniformly with replacement by a
    SplitMix64 stream (paper C.1); assign = argmax_c (x.c - |c|^2/2), ties to
    the lowest c; update = member mean, empty centres keep their value; the
    tolerance 1e-4 (Table C.1) is a fraction of changed labels, so the stop
    test is  changed <= floor(tol N)  after each re-assignment; at most
    ``max_iter`` assignments.  Nonempty groups are renumbered in increasing
    order of centre index (paper §4.1: C_k counts nonempty groups).
R4  mu_K is the unweighted mean of the nonempty K-group centroids; M_Q uses
    the nonempty count (paper §4.1, B.2).  r_Q' = max(1, min(r_Q, d, C_k'-1)).
R5  Routing score: the paper's value-error score (B.3) summed directly, with a
    per-query-group shift m_a subtracted from every exponent; groups are
    ranked by descending score, ties to the lower group index (§4.3).
R6  Key budget beta = (rho - M/N_q) N_k clamped to [0, N_k]; the prefix rule
    "cumulative key count reaches beta" is  cum >= ceil(beta - 1e-6); at
    least one group is always kept (§4.3).
R7  Probe allocation (lost in the extraction of A.2): largest remainder on
    M |G_a| / N_q, remainder ties to larger |G_a| then lower a; inside a group
    the m_a rows with smallest (d_i, i); every row when M >= N_q.
R8  Residual-span projection at full rank is the identity because every row
    of B_lambda lies in the row space of R-bar (§4.2; C.1 default uses none).
R13 Warm start, metric factors (paper C.1: "two subspace iterations
    initialized from the previous factors and using Cholesky factorization"):
    Q_0 = the previous factor; twice  Y = M Q,  Y^T Y = L L^T,  Q = Y L^-T
    (Cholesky QR); then F = Q C with C C^T = Q^T M Q (Cholesky), times
    1/sqrt(d) for the key factor (R2).  F F^T = Q Q^T M Q Q^T, the metric
    restricted to the iterated subspace; at an exact eigenbasis it equals the
    cold factor's F F^T.  The page does not say what happens when the previous
    factor has fewer columns than the current rank or a Cholesky pivot
    vanishes; then the call takes the cold factor (eigendecomposition).  A
    pivot "vanishes" when its square is not above 1e-12 times the largest
    diagonal entry of the matrix being factored.
R14 Warm start, centres (paper C.1: "previous centroids in the original space
    projected into the current response coordinates"): centre b of the key
    k-means is kbar_b F_K, centre a of the query k-means is RMSNorm(qbar_a F_Q),
    for the previous call's nonempty groups; centres past their count are
    drawn as in a cold start (R3).
R15 Later calls run at most 2 k-means assignments (Table C.1, "initial /
    subsequent k means iteration limits 25/2"); the caller passes the limit.
R16 Semantic partition (§3's reference partition, Table 2's baseline): the
    same k-means (initial rows, limit, stop rule) on the raw key rows and on
    the raw query rows, V inheriting its key's group; d_i is the distance to
    the raw-space query-group mean.  Routing, probes, fit and apply are
    unchanged.  Table 2's key-response variant keeps the response K/V groups
    and takes semantic query groups.
R17 Probe variants (Table 4): "random" = M distinct rows drawn uniformly by
    Floyd's sampling algorithm (Bentley & Floyd 1987) from a SplitMix64
    stream seeded by mix(seed xor mix((bh+1) gamma xor 0x50524F4245)): for
    s = 0..M-1, j = N-M+s, draw s+1 gives t = floor(u (j+1) / 2^32) from its
    top 32 bits u, and the sample gains t, or j when t is already in it.
    "uniform" = rows floor((2j+1) N / (2M)), evenly spaced over the
    row-major (t, y, x) grid.  Both keep A.2's coverage weights
    w_p = |G_a| / m_a with m_a the probes that fall in group a, and list
    probes by group, then by index.  With M >= N every variant takes all rows.
R18 Correction families (D.4): with the same standardisation, centring and
    weights, "mean" has B = 0, "scalar" B = a I with
    a = tr(Xbar^T W Rbar) / (tr(Xbar^T W Xbar) + lambda d), "diagonal"
    B = diag(b) with b_j = (Xbar^T W Rbar)_jj / ((Xbar^T W Xbar)_jj + lambda);
    each minimises the weighted squared error plus lambda |B|_F^2 over its
    family.  Rank r truncation (D.3) replaces B by B V_r V_r^T.
R19 GQA (§4.3 "Routing and GQA", C.1): the G query heads of one K/V head
    share the key metric, F_K and the K/V groups.  The metric's rows are
    G M_s evenly spaced rows of the G heads' queries stacked in head order
    (all rows when fewer); the K/V k-means draws its initial rows from the
    K/V head's stream (head index = K/V head).  Query groups, routing,
    probes and the fit stay per query head, with the query head's streams.

Parity unpinned: these functions carry only internal invariants, because no
printed value or closed form fixes them -- routing_score (the prose around
B.3 is lost; it is checked against its own definition), probe_allocation and
probe_select (the A.2 rule is lost), the key_factor scale, kmeans_stop_count,
the key_budget rounding and the mu_K definition.
"""

from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np

# --------------------------------------------------------------------------
# Counter-based generator for the k-means initial centres (paper C.1: "initial
# k means centers are sampled uniformly with replacement from feature rows").
# SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
# generators", OOPSLA 2014): state += golden gamma; output = mix(state).
# --------------------------------------------------------------------------
_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15


def splitmix64_mix(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def splitmix64_outputs(state: int, n: int):
    """First n outputs of a SplitMix64 generator seeded with ``state``."""
    out = []
    for _ in range(n):
        state = (state + _GAMMA) & _M64
        out.append(splitmix64_mix(state))
    return out


def kmeans_init_indices(seed: int, bh: int, stage: int, C: int, N: int) -> np.ndarray:
    """Row indices of the C initial centres for head ``bh`` and ``stage``
    (0 = K/V partition, 1 = query partition).  Draw c is the (c+1)-th output
    of the stream seeded by mix(seed xor mix((2 bh + stage + 1) gamma));
    its top 32 bits u give the row floor(u N / 2^32)."""
    base = splitmix64_mix((seed & _M64) ^ splitmix64_mix(((2 * bh + stage + 1) * _GAMMA) & _M64))
    draws = splitmix64_outputs(base, C)
    return np.array([((x >> 32) * N) >> 32 for x in draws], dtype=np.int64)


# --------------------------------------------------------------------------
# Dense and block-sparse attention (paper §3, "Dense and block-sparse
# attention"; A.1: l_ij = q_i k_j^T / sqrt(d)).
# --------------------------------------------------------------------------
def softmax_rows(logits: np.ndarray) -> np.ndarray:
    z = logits - logits.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


def dense_attention(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """O^dense = softmax(Q K^T / sqrt(d)) V for the given query rows (§3)."""
    d = q_rows.shape[1]
    out = np.empty((q_rows.shape[0], v.shape[1]))
    step = max(1, (1 << 24) // max(1, k.shape[0]))
    for s in range(0, q_rows.shape[0], step):
        out[s:s + step] = softmax_rows(q_rows[s:s + step] @ k.T / math.sqrt(d)) @ v
    return out


def sparse_attention(q, k, v, q_labels, kv_labels, mask) -> np.ndarray:
    """Eq. (2): O_i^sp = softmax(q_i K_a^T / sqrt(d)) V_a, where K_a, V_a are
    the keys/values of every K/V group selected for query group a (§3)."""
    N, d = q.shape
    out = np.empty((N, v.shape[1]))
    for a in range(mask.shape[0]):
        rows = np.nonzero(q_labels == a)[0]
        if rows.size == 0:
            continue
        keys = np.nonzero(mask[a][kv_labels])[0]
        out[rows] = dense_attention(q[rows], k[keys], v[keys])
    return out


# --------------------------------------------------------------------------
# §4.1 Response-coupled partitioning.
# --------------------------------------------------------------------------
def sample_indices(N: int, Ms: int) -> np.ndarray:
    """R1: evenly spaced query rows (C.2), all rows when Ms >= N."""
    if Ms >= N:
        return np.arange(N)
    return (np.arange(Ms, dtype=np.int64) * N) // Ms


def key_metric(q: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """M_K = Q_s^T Q_s / M_s (§4.1, B.1)."""
    Qs = q[idx]
    return Qs.T @ Qs / len(idx)


def eigh_desc(M: np.ndarray):
    """Symmetric eigendecomposition, eigenvalues in descending order."""
    w, U = np.linalg.eigh(M)
    order = np.argsort(-w, kind="stable")
    return w[order], U[:, order]


def key_factor(M_K: np.ndarray, r_K: int, n_samples: int) -> np.ndarray:
    """F_K with phi_K(k) = k F_K (§4.1): leading r_K' eigenpairs of M_K,
    F_K = U_r diag(sqrt(lambda_r)) / sqrt(d)   (R2), r_K' = min(r_K, d, M_s)."""
    d = M_K.shape[0]
    r = min(r_K, d, n_samples)
    w, U = eigh_desc(M_K)
    return U[:, :r] * np.sqrt(np.maximum(w[:r], 0.0))[None, :] / math.sqrt(d)


def kmeans_assign(X: np.ndarray, centres: np.ndarray):
    """Nearest centre by score x.c - |c|^2/2 (equivalently smallest
    |x - c|^2); returns labels and the score matrix."""
    scores = X @ centres.T - 0.5 * (centres * centres).sum(axis=1)[None, :]
    return argmax_rows(scores), scores


def argmax_rows(scores: np.ndarray) -> np.ndarray:
    """Row-wise argmax, ties to the lowest column (np.argmax keeps the first)."""
    return np.argmax(scores, axis=1).astype(np.int64)


def kmeans_update(X: np.ndarray, labels: np.ndarray, centres: np.ndarray) -> np.ndarray:
    """Each centre becomes the mean of its members; empty centres keep their value."""
    C = centres.shape[0]
    counts = np.bincount(labels, minlength=C)
    sums = np.zeros_like(centres)
    np.add.at(sums, labels, X)
    out = centres.copy()
    nz = counts > 0
    out[nz] = sums[nz] / counts[nz][:, None]
    return out


def kmeans_stop_count(tol: float, N: int) -> int:
    """R3: largest changed-label count that ends the iteration."""
    return int(math.floor(tol * N))


def kmeans(X: np.ndarray, init_idx: np.ndarray, max_iter: int, stop_changed: int,
           init_centres: Optional[np.ndarray] = None):
    """Lloyd k-means (§4.1, C.1, Table C.1) under reading R3.  Returns
    (labels, centres used by the last assignment, number of assignments,
    label history).  ``init_centres`` replaces the sampled rows (R14)."""
    centres = (X[init_idx] if init_centres is None else init_centres).copy()
    labels, _ = kmeans_assign(X, centres)
    history = [labels]
    n_assign = 1
    while n_assign < max_iter:
        centres = kmeans_update(X, labels, centres)
        new, _ = kmeans_assign(X, centres)
        changed = int((new != labels).sum())
        labels = new
        history.append(labels)
        n_assign += 1
        if changed <= stop_changed:
            break
    return labels, centres, n_assign, history


WARM_PIVOT_REL = 1e-12


def cholesky_checked(G: np.ndarray) -> Optional[np.ndarray]:
    """Lower Cholesky factor of G, or None when a pivot vanishes (R13)."""
    try:
        L = np.linalg.cholesky(G)
    except np.linalg.LinAlgError:
        return None
    if not np.all(np.diag(L) ** 2 > WARM_PIVOT_REL * np.max(np.diag(G))):
        return None
    return L


def warm_factor(M: np.ndarray, F_prev: np.ndarray, r: int, scale: float,
                iters: int = 2) -> Optional[np.ndarray]:
    """R13: subspace iteration from the previous factor with Cholesky QR, then
    the metric's Cholesky factor on the iterated subspace; d x r, or None
    when the cold factor must be used instead."""
    if F_prev.shape[1] < r:
        return None
    Q = F_prev[:, :r].copy()
    for _ in range(iters):
        Y = M @ Q
        L = cholesky_checked(Y.T @ Y)
        if L is None:
            return None
        Q = np.linalg.solve(L, Y.T).T          # Y L^-T
    C = cholesky_checked(Q.T @ M @ Q)
    if C is None:
        return None
    return (Q @ C) * scale


def warm_centres(Y: np.ndarray, cbar_prev: np.ndarray, F: np.ndarray, C: int, init_idx: np.ndarray,
                 rms_eps: Optional[float] = None) -> np.ndarray:
    """R14: previous centroids (original space) projected into the current
    coordinates, RMS-normalised for the query side; the remaining centres are
    the cold start's rows of Y (the current coordinates)."""
    centres = Y[init_idx].copy()
    n = min(C, cbar_prev.shape[0])
    z = cbar_prev[:n] @ F
    if rms_eps is not None:
        rms = np.sqrt((z * z).sum(axis=1) / F.shape[1])
        z = z / np.maximum(rms, rms_eps)[:, None]
    centres[:n] = z
    return centres


def compact_labels(labels: np.ndarray, C: int):
    """Renumber nonempty groups 0..C'-1 in increasing order of centre index;
    returns (labels, C', sizes)."""
    counts = np.bincount(labels, minlength=C)
    nonempty = counts > 0
    new_id = np.cumsum(nonempty) - 1
    return new_id[labels].astype(np.int64), int(nonempty.sum()), counts[nonempty].astype(np.int64)


def group_means(Y: np.ndarray, labels: np.ndarray, C: int) -> np.ndarray:
    counts = np.bincount(labels, minlength=C)
    sums = np.zeros((C, Y.shape[1]))
    np.add.at(sums, labels, Y)
    return sums / counts[:, None]


def query_metric(k_centroids: np.ndarray) -> np.ndarray:
    """M_Q = K~^T K~ / (C_k d) with K~ rows  kbar_b - mu_K  (§4.1; B.2 shows the
    centring only shifts every logit of a query by one constant).  R4."""
    Ck, d = k_centroids.shape
    mu_K = k_centroids.mean(axis=0)
    Kt = k_centroids - mu_K[None, :]
    return Kt.T @ Kt / (Ck * d)


def query_rank(r_Q: int, d: int, Ck: int) -> int:
    """R4: the centred K-group centroids have rank at most C_k' - 1."""
    return max(1, min(r_Q, d, Ck - 1))


def query_factor(M_Q: np.ndarray, r: int) -> np.ndarray:
    """F_Q = U_r diag(sqrt(lambda_r)) (its scale cancels in the RMSNorm)."""
    w, U = eigh_desc(M_Q)
    return U[:, :r] * np.sqrt(np.maximum(w[:r], 0.0))[None, :]


def query_coords(q: np.ndarray, F_Q: np.ndarray, eps: float) -> np.ndarray:
    """phi_Q(q) = RMSNorm(q F_Q) = q F_Q / max(sqrt(|q F_Q|^2 / r_Q), eps)  (B.2)."""
    z = q @ F_Q
    rms = np.sqrt((z * z).sum(axis=1) / F_Q.shape[1])
    return z / np.maximum(rms, eps)[:, None]


def query_distances(phi: np.ndarray, labels: np.ndarray, C: int):
    """c_a = group mean of phi_Q and d_i = |phi_Q(q_i) - c_a| (A.2)."""
    c = group_means(phi, labels, C)
    return c, np.sqrt(((phi - c[labels]) ** 2).sum(axis=1))


# --------------------------------------------------------------------------
# §4.3 / B.3 routing.
# --------------------------------------------------------------------------
def routing_score(qbar, k, v, kbar, vbar, kv_labels) -> np.ndarray:
    """B.3 value-error score, summed directly (R5):
    s_ab = 1/|G_b| sum_{j in G_b} | e^{qbar_a kbar_b^T/sqrt d} vbar_b
                                    - e^{qbar_a k_j^T/sqrt d} v_j |^2,
    every exponent shifted by m_a = max(max_j l_aj, max_b lbar_ab)."""
    Cq, d = qbar.shape
    Ck = kbar.shape[0]
    sizes = np.bincount(kv_labels, minlength=Ck).astype(np.float64)
    s = np.empty((Cq, Ck))
    for a in range(Cq):
        l_j = k @ qbar[a] / math.sqrt(d)             # [N]
        l_b = kbar @ qbar[a] / math.sqrt(d)          # [Ck]
        m = max(l_j.max(), l_b.max())
        A = np.exp(l_b - m)[:, None] * vbar          # [Ck, d]
        diff = A[kv_labels] - np.exp(l_j - m)[:, None] * v
        sq = (diff * diff).sum(axis=1)
        s[a] = np.bincount(kv_labels, weights=sq, minlength=Ck) / sizes
    return s


def key_budget(density: float, M: int, Nq: int, Nk: int) -> int:
    """R6: per-query key budget after reserving the probes (§4.3)."""
    beta = (density - M / Nq) * Nk
    beta = min(max(beta, 0.0), float(Nk))
    return int(math.ceil(beta - 1e-6))


def route(s: np.ndarray, kv_sizes: np.ndarray, q_sizes: np.ndarray, beta: int):
    """§4.3: per query group rank K/V groups by descending score (ties: lower
    index) and keep the shortest prefix whose key count reaches beta (at least
    one group).  Returns (mask [Cq, Ck] bool, P_route)."""
    Cq, Ck = s.shape
    mask = np.zeros((Cq, Ck), dtype=bool)
    p_route = 0
    for a in range(Cq):
        order = np.lexsort((np.arange(Ck), -s[a]))
        cum = np.cumsum(kv_sizes[order])
        hit = np.nonzero(cum >= beta)[0]
        n_sel = (hit[0] + 1) if hit.size else Ck
        mask[a, order[:n_sel]] = True
        p_route += int(q_sizes[a]) * int(kv_sizes[order[:n_sel]].sum())
    return mask, p_route


def executed_pairs(p_route: int, M: int, Nk: int) -> int:
    """rho_exec = rho_route + M/N_q  in pairs: probes add M N_k (§4.3, B.3)."""
    return p_route + M * Nk


# --------------------------------------------------------------------------
# §4.3 sparse execution: group-major permutation.
# --------------------------------------------------------------------------
def group_permutation(labels: np.ndarray, C: int):
    """Rows in group-major order, stable by original index; offsets[g] is the
    first permuted row of group g."""
    perm = np.argsort(labels, kind="stable")
    sizes = np.bincount(labels, minlength=C)
    offsets = np.concatenate([[0], np.cumsum(sizes)])
    return perm.astype(np.int64), offsets.astype(np.int64)


# --------------------------------------------------------------------------
# §4.2 / A.2 / A.3 probe-fitted residual reconstruction.
# --------------------------------------------------------------------------
def probe_allocation(q_sizes: np.ndarray, M: int, N: int) -> np.ndarray:
    """R7: m_a per query group by largest remainder on M |G_a| / N."""
    q_sizes = np.asarray(q_sizes, dtype=np.int64)
    if M >= N:
        return q_sizes.copy()
    num = M * q_sizes
    base = num // N
    rem = num % N
    extra = M - int(base.sum())
    order = np.lexsort((np.arange(len(q_sizes)), -q_sizes, -rem))
    m = base.copy()
    m[order[:extra]] += 1
    return m


def probe_select(q_labels: np.ndarray, d_i: np.ndarray, m: np.ndarray) -> np.ndarray:
    """R7: inside group a the m_a members with the smallest (d_i, i); probes are
    listed by group, then by (d_i, i)."""
    out = []
    for a in range(len(m)):
        members = np.nonzero(q_labels == a)[0]
        order = np.lexsort((members, d_i[members]))
        out.append(members[order[: int(m[a])]])
    return np.concatenate(out).astype(np.int64) if out else np.zeros(0, np.int64)


PROBE_STREAM = 0x50524F4245


def random_probes(seed: int, bh: int, N: int, M: int) -> np.ndarray:
    """R17: Floyd's algorithm; returns the sampled rows in increasing order."""
    base = splitmix64_mix((seed & _M64) ^ splitmix64_mix((((bh + 1) * _GAMMA) & _M64) ^ PROBE_STREAM))
    draws = splitmix64_outputs(base, M)
    chosen = set()
    for s_, x in enumerate(draws):
        j = N - M + s_
        t = ((x >> 32) * (j + 1)) >> 32
        chosen.add(j if t in chosen else t)
    return np.array(sorted(chosen), dtype=np.int64)


def uniform_probes(N: int, M: int) -> np.ndarray:
    """R17: rows floor((2j+1) N / (2M)), j = 0..M-1."""
    return np.array([((2 * j + 1) * N) // (2 * M) for j in range(M)], dtype=np.int64)


def listed_by_group(rows: np.ndarray, q_labels: np.ndarray, C: int):
    """Probe rows listed by group, then by index, and m_a per group."""
    order = np.lexsort((rows, q_labels[rows]))
    P = rows[order]
    return P, np.bincount(q_labels[P], minlength=C).astype(np.int64)


def coverage_weights(probe_groups: np.ndarray, q_sizes: np.ndarray, m: np.ndarray, M: int):
    """A.2 w_p = |G_a| / m_a;  A.3 alpha_p = w_p / sum w;  w~_p = M w_p / sum w."""
    w = q_sizes[probe_groups] / m[probe_groups]
    alpha = w / w.sum()
    return w, alpha, M * alpha


class NumericError(RuntimeError):
    pass


def ridge_fit(X: np.ndarray, R: np.ndarray, alpha: np.ndarray, wt: np.ndarray,
              lam: float, eps_std: float) -> Dict[str, np.ndarray]:
    """§4.2 / A.3 / D.3: weighted standardisation of X (sigma = sqrt(var + 1e-6)),
    weighted centring of R, and
    B_lambda = argmin |W^{1/2}(Rbar - Xbar B)|_F^2 + lambda |B|_F^2
             = (Xbar^T W Xbar + lambda I)^{-1} Xbar^T W Rbar   (Cholesky)."""
    mu_X = alpha @ X
    var = alpha @ ((X - mu_X[None, :]) ** 2)
    sigma = np.sqrt(var + eps_std)
    Xb = (X - mu_X[None, :]) / sigma[None, :]
    mu_R = alpha @ R
    Rb = R - mu_R[None, :]
    d = X.shape[1]
    G = Xb.T @ (wt[:, None] * Xb) + lam * np.eye(d)
    rhs = Xb.T @ (wt[:, None] * Rb)
    try:
        L = np.linalg.cholesky(G)
    except np.linalg.LinAlgError as e:
        raise NumericError("Gram matrix is not positive definite") from e
    B = np.linalg.solve(L.T, np.linalg.solve(L, rhs))
    return {"mu_X": mu_X, "sigma": sigma, "mu_R": mu_R, "B": B, "Xbar": Xb, "Rbar": Rb}


def restricted_fit(X: np.ndarray, R: np.ndarray, alpha: np.ndarray, wt: np.ndarray, lam: float,
                   eps_std: float, family: str) -> Dict[str, np.ndarray]:
    """R18: the D.4 correction families on ridge_fit's standardised features."""
    f = ridge_fit(X, R, alpha, wt, lam, eps_std)
    if family == "full":
        return f
    Xb, Rb = f["Xbar"], f["Rbar"]
    d = X.shape[1]
    gx = (wt[:, None] * Xb * Xb).sum(axis=0)          # diagonal of Xbar^T W Xbar
    gr = (wt[:, None] * Xb * Rb).sum(axis=0)          # diagonal of Xbar^T W Rbar
    if family == "diagonal":
        B = np.diag(gr / (gx + lam))
    elif family == "scalar":
        B = (gr.sum() / (gx.sum() + lam * d)) * np.eye(d)
    elif family == "mean":
        B = np.zeros((d, d))
    else:
        raise ValueError(family)
    return {**f, "B": B}


def residual_span_projection(B: np.ndarray, Rbar: np.ndarray, wt: np.ndarray,
                             rank: Optional[int] = None, rtol: float = 1e-10) -> np.ndarray:
    """D.3: project onto the leading right singular vectors of W^{1/2} Rbar
    (singular values above rtol * max; the leading ``rank`` when given).  R8:
    at full rank this returns B unchanged up to rounding."""
    Y = np.sqrt(wt)[:, None] * Rbar
    _, S, Vt = np.linalg.svd(Y, full_matrices=False)
    keep = int((S > rtol * S.max()).sum()) if S.size and S.max() > 0 else 0
    if rank is not None:
        keep = min(keep, rank)
    Vr = Vt[:keep].T
    return B @ Vr @ Vr.T


def apply_correction(O_sp: np.ndarray, probes: np.ndarray, O_dense_probes: np.ndarray,
                     fit: Dict[str, np.ndarray]) -> np.ndarray:
    """§4.2: O^_i = O_i^dense for probes, O_i^sp + mu_R + xbar_i B otherwise,
    with xbar_i = (O_i^sp - mu_X) / sigma."""
    xb = (O_sp - fit["mu_X"][None, :]) / fit["sigma"][None, :]
    out = O_sp + fit["mu_R"][None, :] + xb @ fit["B"]
    out[probes] = O_dense_probes
    return out


# --------------------------------------------------------------------------
# Evaluation (D.2 error metric; Table 2 error reduction).
# --------------------------------------------------------------------------
def relative_error(O: np.ndarray, O_dense: np.ndarray, eps: float = 1e-8) -> np.ndarray:
    """|O_i - O_i^dense|_2 / (|O_i^dense|_2 + 1e-8) per row (D.2)."""
    return np.linalg.norm(O - O_dense, axis=1) / (np.linalg.norm(O_dense, axis=1) + eps)


def error_reduction(mean_err_method: float, mean_err_base: float) -> float:
    """1 - err_method / err_base: ratio of mean errors (§5.1, Table 2)."""
    return 1.0 - mean_err_method / mean_err_base


# --------------------------------------------------------------------------
# The whole call for one head.
# --------------------------------------------------------------------------
def sparsepr_head(q, k, v, *, bh: int, seed: int, density: float, M: int, Ms: int,
                  lam: float, Cq: int, Ck: int, rK: int, rQ: int, kmeans_iters: int,
                  kmeans_tol: float, eps_rms: float = 1e-6, eps_std: float = 1e-6,
                  want_dense: bool = False, warm: Optional[Dict[str, np.ndarray]] = None,
                  partition: str = "response", probes: str = "stratified", correction: str = "full",
                  residual_rank: int = 0, metric_rows: Optional[np.ndarray] = None,
                  bh_kv: Optional[int] = None) -> Dict[str, object]:
    """One SparsePR call on one head, steps in the paper's order:
    partition (§4.1) -> route (§4.3, B.3) -> sparse attention (Eq. 2) ->
    probes (A.2) -> weighted ridge (A.3) -> corrected output (§4.2).
    ``warm`` (F_K, F_Q, kbar, qbar of the previous call) selects the warm
    start of R13-R15; the caller also lowers ``kmeans_iters``.
    ``partition``: "response" (§4.1), "semantic" or "key_response" (R16).
    ``probes``: "stratified" (A.2), "random" or "uniform" (R17);
    ``correction``: "full", "diagonal", "scalar" or "mean" (R18);
    ``residual_rank``: 0 (no truncation) or r (D.3).
    ``metric_rows`` / ``bh_kv``: the query rows the key metric samples and
    the head index of the K/V k-means stream (GQA, R19; default q and bh)."""
    if partition not in ("response", "semantic", "key_response"):
        raise ValueError(partition)
    semantic_keys = partition == "semantic"
    semantic_queries = partition in ("semantic", "key_response")
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, d = q.shape
    out: Dict[str, object] = {}

    # 1-2. key-response metric and factor
    mrows = q if metric_rows is None else np.asarray(metric_rows, dtype=np.float64)
    idx = sample_indices(len(mrows), Ms)
    M_K = key_metric(mrows, idx)
    r_k = min(rK, d, len(idx))
    F_K = None if (warm is None or semantic_keys) else warm_factor(M_K, warm["F_K"], r_k, 1.0 / math.sqrt(d))
    warm_K = F_K is not None
    if semantic_keys:
        F_K = np.eye(d)
    elif F_K is None:
        F_K = key_factor(M_K, rK, len(idx))
    phi_K = k @ F_K
    # 3. paired K/V groups
    init_k = kmeans_init_indices(seed, bh if bh_kv is None else bh_kv, 0, Ck, N)
    stop = kmeans_stop_count(kmeans_tol, N)
    cen_k = None if warm is None else warm_centres(phi_K, warm["kbar"], F_K, Ck, init_k)
    kv_raw, _, it_k, _ = kmeans(phi_K, init_k, kmeans_iters, stop, cen_k)
    kv_labels, Ck2, kv_sizes = compact_labels(kv_raw, Ck)
    # 4. centroids, query metric and factor
    kbar = group_means(k, kv_labels, Ck2)
    vbar = group_means(v, kv_labels, Ck2)
    M_Q = query_metric(kbar)
    rq = query_rank(rQ, d, Ck2)
    F_Q = None if (warm is None or semantic_queries) else warm_factor(M_Q, warm["F_Q"], rq, 1.0)
    warm_Q = F_Q is not None
    if semantic_queries:
        F_Q = np.eye(d)
        phi_Q = q.copy()
    else:
        if F_Q is None:
            F_Q = query_factor(M_Q, rq)
        phi_Q = query_coords(q, F_Q, eps_rms)
    # 5. query groups
    init_q = kmeans_init_indices(seed, bh, 1, Cq, N)
    cen_q = None if warm is None else warm_centres(phi_Q, warm["qbar"], F_Q, Cq, init_q,
                                                   None if semantic_queries else eps_rms)
    q_raw, _, it_q, _ = kmeans(phi_Q, init_q, kmeans_iters, stop, cen_q)
    q_labels, Cq2, q_sizes = compact_labels(q_raw, Cq)
    qbar = group_means(q, q_labels, Cq2)
    _, d_i = query_distances(phi_Q, q_labels, Cq2)
    # 6-7. routing
    s = routing_score(qbar, k, v, kbar, vbar, kv_labels)
    beta = key_budget(density, min(M, N), N, N)
    mask, p_route = route(s, kv_sizes, q_sizes, beta)
    # 8. permutation
    perm_q, q_off = group_permutation(q_labels, Cq2)
    perm_k, k_off = group_permutation(kv_labels, Ck2)
    # 9. sparse attention
    O_sp = sparse_attention(q, k, v, q_labels, kv_labels, mask)
    # 10. probes
    Mp = min(M, N)
    if probes == "stratified" or Mp >= N:
        m = probe_allocation(q_sizes, Mp, N)
        P = probe_select(q_labels, d_i, m)
    else:
        rows = random_probes(seed, bh, N, Mp) if probes == "random" else uniform_probes(N, Mp)
        P, m = listed_by_group(rows, q_labels, Cq2)
    w, alpha, wt = coverage_weights(q_labels[P], q_sizes, m, Mp)
    O_dense_P = dense_attention(q[P], k, v)
    # 11. fit and 13. output
    fit = restricted_fit(O_sp[P], O_dense_P - O_sp[P], alpha, wt, lam, eps_std, correction) if Mp > 0 else None
    if fit is not None and residual_rank > 0:
        fit = {**fit, "B": residual_span_projection(fit["B"], fit["Rbar"], wt, residual_rank)}
    O_hat = apply_correction(O_sp, P, O_dense_P, fit) if fit is not None else O_sp.copy()

    out.update(sample_idx=idx, M_K=M_K, F_K=F_K, phi_K=phi_K, kv_labels=kv_labels,
               Ck=Ck2, kv_sizes=kv_sizes, kmeans_iters_k=it_k, kbar=kbar, vbar=vbar,
               M_Q=M_Q, F_Q=F_Q, phi_Q=phi_Q, q_labels=q_labels, Cq=Cq2, q_sizes=q_sizes,
               kmeans_iters_q=it_q, qbar=qbar, d_i=d_i, score=s, beta=beta, mask=mask,
               pairs_route=p_route, pairs_exec=executed_pairs(p_route, Mp, N),
               perm_q=perm_q, q_offsets=q_off, perm_k=perm_k, k_offsets=k_off,
               O_sp=O_sp, m=m, probes=P, w=w, alpha=alpha, wt=wt, O_dense_probes=O_dense_P,
               fit=fit, O=O_hat, warm_factor_used=(warm is not None and warm_K, warm is not None and warm_Q))
    if want_dense:
        out["O_dense"] = dense_attention(q, k, v)
    return out


def sparsepr_gqa(qs, k, v, *, kvh: int, Ms: int, warms=None, **kw):
    """R19: the G query heads qs[g] of K/V head ``kvh`` (query head indices
    kvh G + g); returns one sparsepr_head result per query head.  ``warms``:
    one warm state per query head (their F_K and kbar agree)."""
    G = len(qs)
    stacked = np.concatenate([np.asarray(x, dtype=np.float64) for x in qs], axis=0)
    return [sparsepr_head(qs[g], k, v, bh=kvh * G + g, bh_kv=kvh, metric_rows=stacked, Ms=G * Ms,
                          warm=None if warms is None else warms[g], **kw)
            for g in range(G)]


def warm_state(out: Dict[str, object]) -> Dict[str, np.ndarray]:
    """The state a later call starts from (R13, R14): the metric factors and
    the raw-space centroids of the nonempty groups of ``out``."""
    return dict(F_K=out["F_K"], F_Q=out["F_Q"], kbar=out["kbar"], qbar=out["qbar"])


def workload_kwargs(w) -> Dict[str, object]:
    """Method settings of a ``synthetic.Workload`` as keyword arguments."""
    return dict(seed=w.seed, density=w.density, M=w.M, Ms=w.Ms, lam=w.lam, Cq=w.Cq,
                Ck=w.Ck, rK=w.rK, rQ=w.rQ, kmeans_iters=w.kmeans_iters,
                kmeans_tol=w.kmeans_tol, eps_rms=w.eps_rms, eps_std=w.eps_std)
