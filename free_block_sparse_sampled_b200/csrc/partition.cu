// Response-coupled partitioning ("Partition the Support, Reconstruct the
// Residual", §4.1, B.1, B.2, C.1).
//
//   M_K = Q_s^T Q_s / M_s over evenly spaced sampled queries
//   F_K from an FP32 eigendecomposition (parallel cyclic Jacobi, one block/head)
//   phi_K = K F_K, k-means with C_k requested centres -> paired K/V groups
//   kbar, vbar, mu_K, M_Q = Ktilde^T Ktilde / (C_k' d), F_Q, phi_Q = RMSNorm(q F_Q)
//   k-means with C_q requested centres -> query groups, qbar, c_a, d_i
//
// Variants: a warm start from the previous call's state (C.1; warm.cu), the
// semantic partition on raw key / query rows (§3, Table 2), and GQA, where the
// query heads of one K/V head share M_K, F_K and the K/V groups (§4.3, C.1).
//
// Every reduction that feeds an integer decision runs in a fixed order: the
// k-means centre update sums members in the order of a stable counting sort,
// never through floating-point atomics.
#include "common.cuh"
#include "internal.h"

namespace spr {

// ---------------------------------------------------------------- Gram kernels
// M_K[bh] = (1/Ms) sum_t q_{s_t} q_{s_t}^T with s_t = floor(t N / Ms)  (paper §4.1, C.2).
template <typename T>
__global__ void __launch_bounds__(256) sampled_gram_kernel(const T* __restrict__ X, int N, int d,
                                                           int Ms_eff, float* __restrict__ out) {
    const int bh = blockIdx.z, i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;
    __shared__ float si[32][33], sj[32][33];
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const T* Xh = X + (size_t)bh * N * d;
    for (int t0 = 0; t0 < Ms_eff; t0 += 32) {
        for (int r = ty; r < 32; r += 8) {
            const int t = t0 + r;
            float a = 0.f, b = 0.f;
            if (t < Ms_eff) {
                const long long row = (Ms_eff >= N) ? t : ((long long)t * N) / Ms_eff;
                const T* xr = Xh + row * d;
                a = ldf(xr + i0 + tx);
                b = ldf(xr + j0 + tx);
            }
            si[r][tx] = a;
            sj[r][tx] = b;
        }
        __syncthreads();
#pragma unroll 8
        for (int r = 0; r < 32; ++r) {
            const float bj = sj[r][tx];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] = fmaf(si[r][ty + 8 * u], bj, acc[u]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
        out[(size_t)bh * d * d + (size_t)(i0 + ty + 8 * u) * d + j0 + tx] = acc[u] / (float)Ms_eff;
}

// mu_K = unweighted mean of the C_k' nonempty K-group centroids (paper B.2).
__global__ void centroid_mean_kernel(const float* __restrict__ cen, const int32_t* __restrict__ ng,
                                     int Ck, int d, float* __restrict__ mu) {
    const int bh = blockIdx.x, j = threadIdx.x;
    const int C = ng[bh * 2 + 1];
    float s = 0.f;
    for (int b = 0; b < C; ++b) s += cen[((size_t)bh * Ck + b) * d + j];
    mu[bh * d + j] = s / (float)C;
}

// M_Q[bh] = sum_b (kbar_b - mu_K)(kbar_b - mu_K)^T / (C_k' d)  (paper §4.1).
__global__ void __launch_bounds__(256) centred_gram_kernel(const float* __restrict__ cen,
                                                           const float* __restrict__ mu,
                                                           const int32_t* __restrict__ ng, int Ck,
                                                           int d, float* __restrict__ out) {
    const int bh = blockIdx.z, i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int C = ng[bh * 2 + 1];
    __shared__ float si[32][33], sj[32][33];
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float* base = cen + (size_t)bh * Ck * d;
    const float mi = mu[bh * d + i0 + tx], mj = mu[bh * d + j0 + tx];
    for (int t0 = 0; t0 < C; t0 += 32) {
        for (int r = ty; r < 32; r += 8) {
            const int t = t0 + r;
            si[r][tx] = (t < C) ? base[(size_t)t * d + i0 + tx] - mi : 0.f;
            sj[r][tx] = (t < C) ? base[(size_t)t * d + j0 + tx] - mj : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int r = 0; r < 32; ++r) {
            const float bj = sj[r][tx];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] = fmaf(si[r][ty + 8 * u], bj, acc[u]);
        }
        __syncthreads();
    }
    const float scale = 1.f / ((float)C * (float)d);
#pragma unroll
    for (int u = 0; u < 4; ++u)
        out[(size_t)bh * d * d + (size_t)(i0 + ty + 8 * u) * d + j0 + tx] = acc[u] * scale;
}

// ---------------------------------------------------------------- eigen factor
// Parallel cyclic Jacobi (round-robin pairing: d/2 disjoint rotations per
// round, d-1 rounds per sweep) on one symmetric d x d matrix per block, then
// F[:, c] = u_c sqrt(max(lambda_c, 0)) * scale for the r leading eigenpairs
// (descending, ties to the lower index) and zero columns up to Rp.
// For the query factor (ng != nullptr) r = max(1, min(r_req, d, C_k' - 1)).
// With run_if, only heads whose run_if entry is nonzero are factored.
template <int d>
__global__ void __launch_bounds__(1024) jacobi_factor_kernel(const float* __restrict__ Ain,
                                                            float* __restrict__ F, int Rp,
                                                            int r_req, const int32_t* ng,
                                                            float scale, int32_t* r_out,
                                                            int max_sweeps, const int32_t* run_if) {
    extern __shared__ float sm[];
    const int bh = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    if (run_if != nullptr && run_if[bh] == 0) return;     // factored by the warm start
    const int ld = d + 1, half = d / 2;
    float* A = sm;
    float* V = A + d * ld;
    float4* par = reinterpret_cast<float4*>(V + d * ld);   // per pair: c, s, p, q (int bits)
    float* red = reinterpret_cast<float*>(par + half);      // 64 floats
    int* order = reinterpret_cast<int*>(red + 64);      // d ints

    const float* Ah = Ain + (size_t)bh * d * d;
    for (int e = tid; e < d * d; e += nt) {
        const int i = e / d, j = e % d;
        A[i * ld + j] = 0.5f * (Ah[i * d + j] + Ah[j * d + i]);
        V[i * ld + j] = (i == j) ? 1.f : 0.f;
    }
    __syncthreads();

    float off_prev = INFINITY;
    for (int sweep = 0; sweep < max_sweeps; ++sweep) {
        // convergence: off-diagonal energy vs total energy; stop once it is at
        // fp32 rounding level or a sweep no longer halves it
        float off = 0.f, tot = 0.f;
        for (int e = tid; e < d * d; e += nt) {
            const int i = e / d, j = e % d;
            const float a = A[i * ld + j];
            tot += a * a;
            if (i != j) off += a * a;
        }
        off = warp_sum(off);
        tot = warp_sum(tot);
        if ((tid & 31) == 0) {
            red[tid >> 5] = off;
            red[32 + (tid >> 5)] = tot;
        }
        __syncthreads();
        if (tid == 0) {
            float o = 0.f, t = 0.f;
            for (int w = 0; w < nt / 32; ++w) {
                o += red[w];
                t += red[32 + w];
            }
            red[0] = o;
            red[32] = t;
        }
        __syncthreads();
        const float off_now = red[0];
        const bool converged = !(off_now > 1e-11f * red[32]) || (sweep >= 3 && off_now > 0.5f * off_prev);
        off_prev = off_now;
        __syncthreads();
        if (converged) break;

        for (int round = 0; round < d - 1; ++round) {
            for (int k = tid; k < half; k += nt) {
                int p, q;
                if (k == 0) {
                    p = round;
                    q = d - 1;
                } else {
                    p = (round + k) % (d - 1);
                    q = (round - k + (d - 1)) % (d - 1);
                }
                if (p > q) {
                    const int t = p;
                    p = q;
                    q = t;
                }
                const float apq = A[p * ld + q], app = A[p * ld + p], aqq = A[q * ld + q];
                float c = 1.f, s = 0.f;
                if (apq != 0.f) {
                    const float theta = (aqq - app) / (2.f * apq);
                    const float t = copysignf(1.f, theta) / (fabsf(theta) + sqrtf(theta * theta + 1.f));
                    c = 1.f / sqrtf(t * t + 1.f);
                    s = t * c;
                }
                par[k] = make_float4(c, s, __int_as_float(p), __int_as_float(q));
            }
            __syncthreads();
            // J^T A J in one pass: each thread owns whole 2 x 2 blocks (rows of
            // pair P, columns of pair Q), rotating the rows and then the
            // columns in registers; V J rotates the column pairs of V.  The
            // thread's column pair Q is fixed (nt is a multiple of d / 2), so
            // its rotation is read once.
            {
                const int Q = tid % half;
                const float4 fQ = par[Q];
                const int r = __float_as_int(fQ.z), t = __float_as_int(fQ.w);
                const float cQ = fQ.x, sQ = fQ.y;
                for (int P = tid / half; P < half; P += nt / half) {
                    const float4 fP = par[P];
                    const int p = __float_as_int(fP.z), q = __float_as_int(fP.w);
                    const float cP = fP.x, sP = fP.y;
                    const float apr = A[p * ld + r], apt = A[p * ld + t], aqr = A[q * ld + r], aqt = A[q * ld + t];
                    const float bpr = cP * apr - sP * aqr, bpt = cP * apt - sP * aqt;   // rows p, q
                    const float bqr = sP * apr + cP * aqr, bqt = sP * apt + cP * aqt;
                    A[p * ld + r] = cQ * bpr - sQ * bpt;                                 // columns r, t
                    A[p * ld + t] = sQ * bpr + cQ * bpt;
                    A[q * ld + r] = cQ * bqr - sQ * bqt;
                    A[q * ld + t] = sQ * bqr + cQ * bqt;
                }
                for (int i = tid / half; i < d; i += nt / half) {
                    const float vr = V[i * ld + r], vt = V[i * ld + t];
                    V[i * ld + r] = cQ * vr - sQ * vt;
                    V[i * ld + t] = sQ * vr + cQ * vt;
                }
            }
            __syncthreads();
        }
    }

    // descending eigenvalue order, ties to the lower index
    for (int i = tid; i < d; i += nt) {
        const float li = A[i * ld + i];
        int rank = 0;
        for (int j = 0; j < d; ++j) {
            const float lj = A[j * ld + j];
            rank += (lj > li) || (lj == li && j < i);
        }
        order[rank] = i;
    }
    __syncthreads();
    int r = r_req;
    if (ng != nullptr) r = max(1, min(min(r_req, d), ng[bh * 2 + 1] - 1));
    if (tid == 0 && r_out != nullptr) r_out[bh] = r;
    float* Fh = F + (size_t)bh * d * Rp;
    for (int e = tid; e < d * Rp; e += nt) {
        const int i = e / Rp, c = e % Rp;
        float v = 0.f;
        if (c < r) {
            const int col = order[c];
            v = V[i * ld + col] * sqrtf(fmaxf(A[col * ld + col], 0.f)) * scale;
        }
        Fh[e] = v;
    }
}

// ---------------------------------------------------------------- projections
// phi[i] = x_i F (R columns); with RMS: divided by max(sqrt(|x_i F|^2 / r), eps)
// (paper §4.1 phi_K, B.2 phi_Q).  One thread per row, F in shared memory.
template <typename T, int R, bool RMS>
__global__ void __launch_bounds__(128) project_kernel(const T* __restrict__ X,
                                                      const float* __restrict__ F, int N, int d,
                                                      const int32_t* __restrict__ r_eff, float eps,
                                                      float* __restrict__ phi) {
    extern __shared__ float Fs[];
    const int bh = blockIdx.y;
    for (int e = threadIdx.x; e < d * R; e += blockDim.x) Fs[e] = F[(size_t)bh * d * R + e];
    __syncthreads();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= N) return;
    const T* x = X + ((size_t)bh * N + i) * d;
    float acc[R];
#pragma unroll
    for (int c = 0; c < R; ++c) acc[c] = 0.f;
    for (int t0 = 0; t0 < d; t0 += 8) {
        float v[8];
        load8(x + t0, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float* Fr = Fs + (t0 + u) * R;
#pragma unroll
            for (int c = 0; c < R; ++c) acc[c] = fmaf(v[u], Fr[c], acc[c]);
        }
    }
    if (RMS) {
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < R; ++c) ss = fmaf(acc[c], acc[c], ss);
        const float den = fmaxf(sqrtf(ss / (float)r_eff[bh]), eps);
#pragma unroll
        for (int c = 0; c < R; ++c) acc[c] = acc[c] / den;
    }
    // k-means runs on TF32 coordinates (exact products on the tensor cores)
    float4* out = reinterpret_cast<float4*>(phi + ((size_t)bh * N + i) * R);
#pragma unroll
    for (int c = 0; c < R; c += 4)
        out[c / 4] = make_float4(tf32_round(acc[c]), tf32_round(acc[c + 1]), tf32_round(acc[c + 2]),
                                 tf32_round(acc[c + 3]));
}

// ---------------------------------------------------------------- k-means
// Initial centres: rows drawn uniformly with replacement (paper C.1) by the
// SplitMix64 stream of (seed, head, stage).  One warp per centre.
template <int R>
__global__ void kmeans_init_kernel(const float* __restrict__ phi, int N, int C, uint64_t seed,
                                   int stage, float* __restrict__ cen, float* __restrict__ hn) {
    const int bh = blockIdx.y, lane = threadIdx.x & 31;
    const int c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (c >= C) return;
    const int row = kmeans_init_row(seed, bh, stage, c, N);
    const float* src = phi + ((size_t)bh * N + row) * R;
    float* dst = cen + ((size_t)bh * C + c) * R;
    float ss = 0.f;
    for (int t = lane; t < R; t += 32) {
        const float v = src[t];
        dst[t] = v;
        ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) hn[(size_t)bh * C + c] = 0.5f * ss;
}

// Assignment: label = argmax_c (x.c - |c|^2/2), ties to the lowest c.  Labels
// are updated in place; changed labels are counted per head.
template <int R>
__global__ void __launch_bounds__(128) kmeans_assign_kernel(
    const float* __restrict__ phi, const float* __restrict__ cen, const float* __restrict__ hn,
    int N, int C, int32_t* __restrict__ labels, int32_t* __restrict__ ctl, int first,
    float* __restrict__ dbg_scores, int32_t* __restrict__ dbg_hist, int max_iter) {
    constexpr int CH = 64;
    __shared__ __align__(16) float cs[CH * R];
    __shared__ float hs[CH];
    const int bh = blockIdx.y;
    int32_t* hc = ctl + bh * kCtlStride;
    if (hc[kCtlDone]) return;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const bool valid = i < N;
    float x[R];
    if (valid) {
        const float4* src = reinterpret_cast<const float4*>(phi + ((size_t)bh * N + i) * R);
#pragma unroll
        for (int t = 0; t < R; t += 4) {
            const float4 v = src[t / 4];
            x[t] = v.x; x[t + 1] = v.y; x[t + 2] = v.z; x[t + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int t = 0; t < R; ++t) x[t] = 0.f;
    }
    float best = -INFINITY;
    int bi = 0;
    const float* ch = cen + (size_t)bh * C * R;
    for (int c0 = 0; c0 < C; c0 += CH) {
        const int n = min(CH, C - c0);
        __syncthreads();
        for (int e = threadIdx.x; e < n * R; e += blockDim.x) cs[e] = ch[(size_t)c0 * R + e];
        for (int e = threadIdx.x; e < n; e += blockDim.x) hs[e] = hn[(size_t)bh * C + c0 + e];
        __syncthreads();
        for (int cc = 0; cc < n; ++cc) {
            const float* cr = cs + cc * R;
            float s = 0.f;
#pragma unroll
            for (int t = 0; t < R; ++t) s = fmaf(x[t], cr[t], s);
            const float sc = s - hs[cc];
            if (dbg_scores != nullptr && valid) dbg_scores[((size_t)bh * N + i) * C + c0 + cc] = sc;
            if (sc > best) {
                best = sc;
                bi = c0 + cc;
            }
        }
    }
    int changed = 0;
    if (valid) {
        int32_t* lp = labels + (size_t)bh * N + i;
        changed = (!first) && (*lp != bi);
        *lp = bi;
        if (dbg_hist != nullptr) dbg_hist[((size_t)bh * max_iter + hc[kCtlIters]) * N + i] = bi;
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, changed);
    if ((threadIdx.x & 31) == 0 && ballot) atomicAdd(&hc[kCtlChanged], __popc(ballot));
}

// After each assignment: count it, and stop the head once changed labels <= stop.
__global__ void kmeans_check_kernel(int32_t* ctl, int BH, int stop, int first) {
    const int bh = blockIdx.x * blockDim.x + threadIdx.x;
    if (bh >= BH) return;
    int32_t* hc = ctl + bh * kCtlStride;
    if (hc[kCtlDone]) return;
    hc[kCtlIters] += 1;
    if (!first && hc[kCtlChanged] <= stop) hc[kCtlDone] = 1;
    hc[kCtlChanged] = 0;
}

__global__ void kmeans_reset_kernel(int32_t* ctl, int BH, int save_slot) {
    const int bh = blockIdx.x * blockDim.x + threadIdx.x;
    if (bh >= BH) return;
    int32_t* hc = ctl + bh * kCtlStride;
    if (save_slot >= 0) hc[save_slot] = hc[kCtlIters];
    hc[kCtlChanged] = 0;
    hc[kCtlDone] = 0;
    hc[kCtlIters] = 0;
}

// ---- stable counting sort of labels (group-major order, stable by index)
__global__ void __launch_bounds__(1024) label_hist_kernel(const int32_t* __restrict__ labels, int N,
                                                          int C, int n_tiles,
                                                          int32_t* __restrict__ hist,
                                                          const int32_t* __restrict__ ctl) {
    const int bh = blockIdx.y, tile = blockIdx.x;
    if (ctl != nullptr && ctl[bh * kCtlStride + kCtlDone]) return;
    __shared__ int h[kMaxGroups];
    for (int c = threadIdx.x; c < C; c += blockDim.x) h[c] = 0;
    __syncthreads();
    const int i = tile * kSortTile + threadIdx.x;
    if (i < N) atomicAdd(&h[labels[(size_t)bh * N + i]], 1);
    __syncthreads();
    int32_t* dst = hist + ((size_t)bh * n_tiles + tile) * C;
    for (int c = threadIdx.x; c < C; c += blockDim.x) dst[c] = h[c];
}

// Per label c: exclusive prefix of the per-tile counts over the tiles (in
// place) and the label's total, written to offs[c].  One thread per label.
__global__ void __launch_bounds__(256) label_colscan_kernel(int32_t* __restrict__ hist, int C, int n_tiles,
                                                            int32_t* __restrict__ offs,
                                                            const int32_t* __restrict__ ctl) {
    const int bh = blockIdx.y, c = blockIdx.x * blockDim.x + threadIdx.x;
    if (ctl != nullptr && ctl[bh * kCtlStride + kCtlDone]) return;
    if (c >= C) return;
    int32_t* hh = hist + (size_t)bh * n_tiles * C + c;
    int run = 0;
    int t = 0;
    for (; t + 32 <= n_tiles; t += 32) {   // 32 loads in flight
        int v[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = hh[(size_t)(t + u) * C];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            hh[(size_t)(t + u) * C] = run;
            run += v[u];
        }
    }
    for (; t < n_tiles; ++t) {
        const int v = hh[(size_t)t * C];
        hh[(size_t)t * C] = run;
        run += v;
    }
    offs[(size_t)bh * (C + 1) + c] = run;
}

// Label totals -> group offsets [C+1] (exclusive scan, offs[C] = N).
__global__ void __launch_bounds__(1024) label_offsets_kernel(int32_t* __restrict__ offs, int N, int C,
                                                             const int32_t* __restrict__ ctl) {
    const int bh = blockIdx.x;
    if (ctl != nullptr && ctl[bh * kCtlStride + kCtlDone]) return;
    __shared__ int tot[kMaxGroups];
    __shared__ int scratch[33];
    int32_t* oo = offs + (size_t)bh * (C + 1);
    for (int c = threadIdx.x; c < C; c += blockDim.x) tot[c] = oo[c];
    __syncthreads();
    block_exclusive_scan(tot, C, scratch);
    for (int c = threadIdx.x; c < C; c += blockDim.x) oo[c] = tot[c];
    if (threadIdx.x == 0) oo[C] = N;
}

// Scatter of one tile's points to their sorted positions: the label's group
// offset + the counts of earlier tiles + the rank among equal labels of lower
// index in this tile, so the sort is stable.  The in-tile rank is the count in
// earlier warps (a per-label scan over the warps of per-warp counts, uint16
// table [warp][label] in dynamic shared memory) plus the rank among lower lanes
// of the same warp; three block barriers per tile.
__global__ void __launch_bounds__(kSortTile) label_scatter_kernel(const int32_t* __restrict__ labels, int N,
                                                                  int C, int n_tiles,
                                                                  const int32_t* __restrict__ hist,
                                                                  const int32_t* __restrict__ offs,
                                                                  int32_t* __restrict__ sorted,
                                                                  const int32_t* __restrict__ ctl) {
    constexpr int W = kSortTile / 32;
    const int bh = blockIdx.y, tile = blockIdx.x;
    if (ctl != nullptr && ctl[bh * kCtlStride + kCtlDone]) return;
    extern __shared__ int32_t sort_smem[];
    int32_t* cnt = sort_smem;                                          // [C]: group offset + earlier tiles
    uint16_t* wc = reinterpret_cast<uint16_t*>(sort_smem + C);         // [W][C]: per-warp counts, then prefix
    const int32_t* base = hist + ((size_t)bh * n_tiles + tile) * C;
    const int32_t* go = offs + (size_t)bh * (C + 1);
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        cnt[c] = base[c] + go[c];
#pragma unroll
        for (int w = 0; w < W; ++w) wc[w * C + c] = 0;
    }
    __syncthreads();
    const int i = tile * kSortTile + threadIdx.x;
    const int lab = (i < N) ? labels[(size_t)bh * N + i] : -1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned m = __match_any_sync(0xffffffffu, lab);
    const int rank = __popc(m & ((1u << lane) - 1u));
    if (lab >= 0 && lane == __ffs(m) - 1) wc[warp * C + lab] = (uint16_t)__popc(m);
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {   // exclusive scan over the warps, per label
        int run = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const int v = wc[w * C + c];
            wc[w * C + c] = (uint16_t)run;
            run += v;
        }
    }
    __syncthreads();
    if (lab >= 0) sorted[(size_t)bh * N + cnt[lab] + wc[warp * C + lab] + rank] = i;
}

// ---- exact member sums for the centre updates
// Coordinates of head bh are taken as the integers q = rint(phi * 2^S_bh),
// with S_bh chosen so that a sum of N of them stays below 2^62 in magnitude.
// Integer sums are exact: they do not depend on the order of the members, so
// after the first update only the points whose label changed move their q
// from one centre's sum to the other's.  A centre is the member mean
// (sum * 2^-S / count in fp64, rounded to fp32 and then TF32); empty centres
// keep their value.

// Largest |phi| of each head, as float bits (non-negative floats order as
// unsigned integers): grid (blocks, BH), atomicMax into amax[bh] (zeroed first).
__global__ void coord_absmax_kernel(const float* __restrict__ phi, size_t per_head, uint32_t* __restrict__ amax) {
    const int bh = blockIdx.y;
    const float4* ph = reinterpret_cast<const float4*>(phi + (size_t)bh * per_head);
    float m = 0.f;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < per_head / 4; e += (size_t)gridDim.x * blockDim.x) {
        const float4 v = ph[e];
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) atomicMax(&amax[bh], __float_as_uint(m));
}

// S_bh = 62 - (bits of max |phi|) - (bits of N), from the head's max bits.
__device__ __forceinline__ int fixed_exponent(uint32_t amax_bits, int N) {
    const float m = __uint_as_float(amax_bits);
    const int eb = m > 0.f ? ilogbf(m) + 1 : 0;   // max |phi| < 2^eb
    return 62 - eb - (32 - __clz(N));               // N < 2^(32 - clz(N))
}

// q = rint(x * 2^S): two exact multiplications by powers of two (each factor
// in float range for the S above) and one rounding conversion.
struct FixedScale {
    float s1, s2;
};
__device__ __forceinline__ FixedScale fixed_scale(int S) {
    FixedScale f;
    f.s1 = __int_as_float((S / 2 + 127) << 23);
    f.s2 = __int_as_float((S - S / 2 + 127) << 23);
    return f;
}
__device__ __forceinline__ long long fixed_coord(float x, const FixedScale& f) { return __float2ll_rn((x * f.s1) * f.s2); }

// First update of a run: the member sums and counts from the sorted member
// lists (one warp per centre; lane k holds coordinates k, k + 32, ...; eight
// member rows in flight per step).
template <int R>
__global__ void centre_sums_kernel(const float* __restrict__ phi, const int32_t* __restrict__ sorted,
                                   const int32_t* __restrict__ offs, const uint32_t* __restrict__ amax, int N, int C,
                                   long long* __restrict__ csum, int32_t* __restrict__ ccnt,
                                   const int32_t* __restrict__ ctl) {
    constexpr int KPL = (R + 31) / 32;   // coordinates per lane
    constexpr int U = 8;                 // member rows per step
    const int bh = blockIdx.y, lane = threadIdx.x & 31;
    if (ctl[bh * kCtlStride + kCtlDone]) return;
    const int c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (c >= C) return;
    const int s = offs[(size_t)bh * (C + 1) + c], e = offs[(size_t)bh * (C + 1) + c + 1];
    const FixedScale S = fixed_scale(fixed_exponent(amax[bh], N));
    long long acc[KPL];
#pragma unroll
    for (int k = 0; k < KPL; ++k) acc[k] = 0;
    const float* ph = phi + (size_t)bh * N * R;
    const int32_t* so = sorted + (size_t)bh * N;
    for (int p0 = s; p0 < e; p0 += 32) {
        const int my = (p0 + lane < e) ? so[p0 + lane] : 0;
        const int n = min(32, e - p0);
        for (int q0 = 0; q0 < n; q0 += U) {
            float x[U][KPL];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int row = __shfl_sync(0xffffffffu, my, (q0 + u) & 31);
#pragma unroll
                for (int k = 0; k < KPL; ++k)
                    x[u][k] = (q0 + u < n && 32 * k + lane < R) ? ph[(size_t)row * R + 32 * k + lane] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int k = 0; k < KPL; ++k) acc[k] += fixed_coord(x[u][k], S);
        }
    }
    long long* cs = csum + ((size_t)bh * C + c) * R;
#pragma unroll
    for (int k = 0; k < KPL; ++k)
        if (32 * k + lane < R) cs[32 * k + lane] = acc[k];
    if (lane == 0) ccnt[(size_t)bh * C + c] = e - s;
}

// Later updates: every point whose label differs from the one its sums hold
// (prev) moves its coordinates from the old centre's sum to the new one's.
// One warp per 32 points; the warp takes the moving points one at a time,
// a lane per coordinate.
__global__ void centre_delta_kernel(const float* __restrict__ phi, const int32_t* __restrict__ labels,
                                    int32_t* __restrict__ prev, const uint32_t* __restrict__ amax, int N, int C, int R,
                                    long long* __restrict__ csum, int32_t* __restrict__ ccnt,
                                    const int32_t* __restrict__ ctl) {
    const int bh = blockIdx.y, lane = threadIdx.x & 31;
    if (ctl[bh * kCtlStride + kCtlDone]) return;
    const int p0 = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 32;
    if (p0 >= N) return;
    const int p = p0 + lane;
    const size_t hb = (size_t)bh * N;
    const int nw = p < N ? labels[hb + p] : 0, od = p < N ? prev[hb + p] : 0;
    const bool mv = p < N && nw != od;
    unsigned moving = __ballot_sync(0xffffffffu, mv);
    if (moving == 0u) return;
    if (mv) {
        prev[hb + p] = nw;
        atomicAdd(&ccnt[(size_t)bh * C + nw], 1);
        atomicSub(&ccnt[(size_t)bh * C + od], 1);
    }
    const FixedScale S = fixed_scale(fixed_exponent(amax[bh], N));
    const float* ph = phi + hb * R;
    unsigned long long* cs = reinterpret_cast<unsigned long long*>(csum) + (size_t)bh * C * R;
    while (moving != 0u) {
        const int j = __ffs(moving) - 1;
        moving &= moving - 1u;
        const int n = __shfl_sync(0xffffffffu, nw, j), o = __shfl_sync(0xffffffffu, od, j);
        for (int k = lane; k < R; k += 32) {
            const long long q = fixed_coord(ph[(size_t)(p0 + j) * R + k], S);
            atomicAdd(&cs[(size_t)n * R + k], (unsigned long long)q);
            atomicAdd(&cs[(size_t)o * R + k], (unsigned long long)(-q));
        }
    }
}

// Centres (and -|c|^2/2 halves, hn = |c|^2 / 2) from the sums; one warp per centre.
__global__ void centre_from_sums_kernel(const long long* __restrict__ csum, const int32_t* __restrict__ ccnt,
                                        const uint32_t* __restrict__ amax, int N, int C, int R, float* __restrict__ cen,
                                        float* __restrict__ hn, const int32_t* __restrict__ ctl) {
    const int bh = blockIdx.y, lane = threadIdx.x & 31;
    if (ctl[bh * kCtlStride + kCtlDone]) return;
    const int c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (c >= C) return;
    const int cnt = ccnt[(size_t)bh * C + c];
    if (cnt <= 0) return;   // empty: keeps its value
    const int S = fixed_exponent(amax[bh], N);
    const long long* cs = csum + ((size_t)bh * C + c) * R;
    float* cc = cen + ((size_t)bh * C + c) * R;
    float ss = 0.f;
    for (int k = lane; k < R; k += 32) {
        const float m = tf32_round((float)(scalbn((double)cs[k], -S) / (double)cnt));
        cc[k] = m;
        ss = fmaf(m, m, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) hn[(size_t)bh * C + c] = 0.5f * ss;
}

// ---------------------------------------------------------------- compaction
// Nonempty groups renumbered in increasing order of centre index (paper §4.1:
// C_k counts the nonempty groups).  Writes new ids, compacted offsets (tail
// filled with N) and the count.
__global__ void __launch_bounds__(1024) compact_groups_kernel(const int32_t* __restrict__ offs_raw,
                                                              int C, int N,
                                                              int32_t* __restrict__ new_id,
                                                              int32_t* __restrict__ offs_out,
                                                              int32_t* __restrict__ ng, int which) {
    const int bh = blockIdx.x;
    __shared__ int flag[kMaxGroups];
    __shared__ int scratch[33];
    const int32_t* o = offs_raw + (size_t)bh * (C + 1);
    for (int c = threadIdx.x; c < C; c += blockDim.x) flag[c] = (o[c + 1] - o[c]) > 0;
    __syncthreads();
    const int total = block_exclusive_scan(flag, C, scratch);
    int32_t* oo = offs_out + (size_t)bh * (C + 1);
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        const bool ne = (o[c + 1] - o[c]) > 0;
        new_id[(size_t)bh * C + c] = ne ? flag[c] : -1;
        if (ne) oo[flag[c]] = o[c];
    }
    for (int c = total + threadIdx.x; c <= C; c += blockDim.x) oo[c] = N;
    if (threadIdx.x == 0) ng[bh * 2 + which] = total;
}

__global__ void relabel_kernel(const int32_t* __restrict__ raw, const int32_t* __restrict__ new_id,
                               const int32_t* __restrict__ sorted, int BH, int N, int C,
                               int32_t* __restrict__ label_out, int32_t* __restrict__ perm_out,
                               int32_t* __restrict__ pos_out) {
    const size_t total = (size_t)BH * N;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const int bh = (int)(e / N);
        label_out[e] = new_id[(size_t)bh * C + raw[e]];
        const int src = sorted[e];
        perm_out[e] = src;
        if (pos_out != nullptr) pos_out[(size_t)bh * N + src] = (int)(e - (size_t)bh * N);
    }
}

// Xp[h, r] = X[h, perm[h * perm_mul, r]] in 16-byte chunks (group-major
// gather, paper §4.3).  perm_mul = G gathers each K/V head once, in the order
// of its first query head (all G share the K/V groups under GQA).
__global__ void gather_rows_kernel(const uint4* __restrict__ X, const int32_t* __restrict__ perm,
                                   int BH, int N, int chunks, int perm_mul, uint4* __restrict__ Xp) {
    const size_t total = (size_t)BH * N * chunks;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const size_t row = e / chunks;
        const int ch = (int)(e - row * chunks);
        const size_t bh = row / N, r = row - bh * N;
        const size_t src = bh * N + perm[(bh * perm_mul) * N + r];
        Xp[e] = X[src * chunks + ch];
    }
}

// Mean of the rows of each group in group-major storage (fixed row order).
// The rows of head bh live at head bh / src_div of Xp (the K/V head under GQA).
template <typename T>
__global__ void group_mean_kernel(const T* __restrict__ Xp, const int32_t* __restrict__ offs,
                                  const int32_t* __restrict__ ng, int which, int N, int C, int d, int src_div,
                                  float* __restrict__ out) {
    const int bh = blockIdx.y, g = blockIdx.x, j = threadIdx.x;
    if (g >= ng[bh * 2 + which]) return;
    const int s = offs[(size_t)bh * (C + 1) + g], e = offs[(size_t)bh * (C + 1) + g + 1];
    const T* base = Xp + (size_t)(bh / src_div) * N * d + j;
    float acc = 0.f;
    for (int r = s; r < e; ++r) acc += ldf(base + (size_t)r * d);
    out[((size_t)bh * C + g) * d + j] = acc / (float)(e - s);
}

// c_a: mean of phi_Q over the members of query group a (members in index order).
__global__ void group_mean_indirect_kernel(const float* __restrict__ phi,
                                           const int32_t* __restrict__ perm,
                                           const int32_t* __restrict__ offs,
                                           const int32_t* __restrict__ ng, int N, int C, int R,
                                           float* __restrict__ out) {
    const int bh = blockIdx.y, g = blockIdx.x, j = threadIdx.x;
    if (g >= ng[bh * 2 + 0] || j >= R) return;
    const int s = offs[(size_t)bh * (C + 1) + g], e = offs[(size_t)bh * (C + 1) + g + 1];
    const int32_t* pr = perm + (size_t)bh * N;
    float acc = 0.f;
    for (int r = s; r < e; ++r) acc += phi[((size_t)bh * N + pr[r]) * R + j];
    out[((size_t)bh * C + g) * R + j] = acc / (float)(e - s);
}

// d_i = |phi_Q(q_i) - c_a|  (paper A.2), by original row.  A power-of-two
// group of lanes shares a row (one float4 each, coalesced); their partial
// sums are combined by shuffles in a fixed order.
__global__ void query_dist_kernel(const float* __restrict__ phi, const float* __restrict__ ca,
                                  const int32_t* __restrict__ qlab, int BH, int N, int C, int R,
                                  float* __restrict__ dist) {
    const int nq = R / 4;                  // float4 per row (R a multiple of 16, at most 128)
    int lpr = 4;                           // lanes per row: the power of two >= nq
    while (lpr < nq) lpr <<= 1;
    const int rpw = 32 / lpr;              // rows per warp step
    const int lane = threadIdx.x & 31, part = lane % lpr, slot = lane / lpr;
    const size_t total = (size_t)BH * N;
    const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
    for (size_t base = (blockIdx.x * (size_t)(blockDim.x >> 5) + (threadIdx.x >> 5)) * rpw; base < total;
         base += warps * rpw) {
        const size_t e = base + slot;
        float ss = 0.f;
        if (e < total && part < nq) {
            const int bh = (int)(e / N);
            const float4 x = reinterpret_cast<const float4*>(phi + e * R)[part];
            const float4 c = reinterpret_cast<const float4*>(ca + ((size_t)bh * C + qlab[e]) * R)[part];
            const float d0 = x.x - c.x, d1 = x.y - c.y, d2 = x.z - c.z, d3 = x.w - c.w;
            ss = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, d3 * d3)));
        }
        for (int o = lpr / 2; o > 0; o >>= 1) ss += __shfl_down_sync(0xffffffffu, ss, o, lpr);
        if (part == 0 && e < total) dist[e] = sqrtf(ss);
    }
}

__global__ void iters_out_kernel(const int32_t* __restrict__ ctl, int BH, int32_t* __restrict__ out) {
    const int bh = blockIdx.x * blockDim.x + threadIdx.x;
    if (bh >= BH) return;
    out[bh * 2 + 0] = ctl[bh * kCtlStride + kCtlItersK];
    out[bh * 2 + 1] = ctl[bh * kCtlStride + kCtlItersQ];
}

// GQA (paper §4.3, C.1): the G query heads of a K/V head share its key
// metric, which is the mean of their sampled metrics (G*Ms evenly spaced rows
// of the stacked heads are each head's own Ms rows).
__global__ void mean_heads_kernel(const float* __restrict__ in, int G, size_t per_head, size_t total,
                                  float* __restrict__ out) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        const size_t h = e / per_head, i = e - h * per_head;
        float s = 0.f;
        for (int g = 0; g < G; ++g) s += in[(h * G + g) * per_head + i];
        out[e] = s / (float)G;
    }
}

// dst head bh = src head bh / G (4-byte words, per_head words per head).
__global__ void broadcast_heads_kernel(const uint32_t* __restrict__ src, size_t per_head, size_t total, int G,
                                       uint32_t* __restrict__ dst) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        const size_t h = e / per_head, i = e - h * per_head;
        dst[e] = src[(h / G) * per_head + i];
    }
}

// The K/V k-means count of each K/V head to its query heads (descending, in place).
__global__ void broadcast_iters_kernel(int32_t* ctl, int BH, int G) {
    for (int bh = BH - 1; bh >= 0; --bh) ctl[bh * kCtlStride + kCtlIters] = ctl[(bh / G) * kCtlStride + kCtlIters];
}

// Semantic partition (paper §3 reference partition, Table 2): the k-means
// coordinates are the raw rows, TF32-rounded (exact for bf16 inputs), and
// the factor is the identity.
template <typename T>
__global__ void raw_coords_kernel(const T* __restrict__ X, size_t n8, float* __restrict__ phi) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n8; e += (size_t)gridDim.x * blockDim.x) {
        float v[8];
        load8(X + e * 8, v);
        float4* o = reinterpret_cast<float4*>(phi + e * 8);
        o[0] = make_float4(tf32_round(v[0]), tf32_round(v[1]), tf32_round(v[2]), tf32_round(v[3]));
        o[1] = make_float4(tf32_round(v[4]), tf32_round(v[5]), tf32_round(v[6]), tf32_round(v[7]));
    }
}

__global__ void identity_factor_kernel(float* __restrict__ F, int d, int Rp, int32_t* __restrict__ r_out) {
    const int bh = blockIdx.x;
    float* Fh = F + (size_t)bh * d * Rp;
    for (int e = threadIdx.x; e < d * Rp; e += blockDim.x) Fh[e] = (e / Rp == e % Rp) ? 1.f : 0.f;
    if (threadIdx.x == 0 && r_out != nullptr) r_out[bh] = d;
}

// ================================================================ host side
void launch_jacobi_factor(const float* A, float* F, int Rp, int r, int BH, int d, cudaStream_t st) {
    const size_t jac_smem = (size_t)(2 * d * (d + 1) + 4 * (d / 2) + 64) * sizeof(float) + (size_t)d * sizeof(int);
    auto jacobi = (d == 128) ? jacobi_factor_kernel<128> : jacobi_factor_kernel<64>;
    cudaFuncSetAttribute(jacobi, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)jac_smem);
    count_launch(), jacobi<<<BH, 1024, jac_smem, st>>>(A, F, Rp, r, nullptr, 1.f, nullptr, 16, nullptr);
}

namespace {

// Dynamic shared memory of label_scatter_kernel for C labels: the offsets
// (int32) and the per-warp counts (uint16).
size_t scatter_smem(int C) {
    const size_t bytes = (size_t)C * (4 + 2 * (kSortTile / 32));
    cudaFuncSetAttribute(label_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    return bytes;
}

inline int grid_for(size_t total, int threads) {
    size_t g = (total + threads - 1) / threads;
    return (int)(g > 148 * 64 ? 148 * 64 : (g == 0 ? 1 : g));
}

template <int R>
void kmeans_run(const Plan& pl, const sparsepr_params& p, void* ws, const float* phi, int C,
                int stage, float* cen, float* hn, float* dbg_scores, int32_t* dbg_hist,
                int save_slot, const WarmInit* wi, int nh, int32_t* raw, cudaStream_t st) {
    int32_t* ctl = at<int32_t>(ws, pl.o_ctl);
    int32_t* hist = at<int32_t>(ws, pl.o_hist);
    int32_t* sorted = at<int32_t>(ws, pl.o_sorted);
    int32_t* offs = at<int32_t>(ws, pl.o_offs);
    const int BH = nh, N = pl.N;
    const int bgrid = (BH + 127) / 128;
    count_launch(), kmeans_reset_kernel<<<bgrid, 128, 0, st>>>(ctl, BH, save_slot);
    if (wi != nullptr)
        launch_warm_init(*wi, R, phi, BH, N, C, p.seed, stage, cen, hn, st);
    else
        count_launch(), kmeans_init_kernel<R><<<dim3((C + 7) / 8, BH), 256, 0, st>>>(phi, N, C, p.seed, stage, cen, hn);
    const dim3 agrid((N + 127) / 128, BH);
    const dim3 tgrid(pl.n_sort_tiles, BH), cgrid((C + 255) / 256, BH), wgrid((C + 7) / 8, BH);
    long long* csum = at<long long>(ws, pl.o_csum);
    int32_t* ccnt = at<int32_t>(ws, pl.o_ccnt);
    int32_t* prev = at<int32_t>(ws, pl.o_prev);
    uint32_t* amax = at<uint32_t>(ws, pl.o_cscale);
    if (p.kmeans_iters > 1) {
        cudaMemsetAsync(amax, 0, (size_t)BH * sizeof(uint32_t), st);
        count_launch(), coord_absmax_kernel<<<dim3(16, BH), 512, 0, st>>>(phi, (size_t)N * R, amax);
    }
    for (int it = 0; it < p.kmeans_iters; ++it) {
        const int first = it == 0;
        if (it == 1) {   // first update: sums and counts from the sorted member lists
            count_launch(), label_hist_kernel<<<tgrid, kSortTile, 0, st>>>(raw, N, C, pl.n_sort_tiles, hist, ctl);
            count_launch(), label_colscan_kernel<<<cgrid, 256, 0, st>>>(hist, C, pl.n_sort_tiles, offs, ctl);
            count_launch(), label_offsets_kernel<<<BH, 1024, 0, st>>>(offs, N, C, ctl);
            count_launch(), label_scatter_kernel<<<tgrid, kSortTile, scatter_smem(C), st>>>(raw, N, C, pl.n_sort_tiles,
                                                                                             hist, offs, sorted, ctl);
            count_launch(), centre_sums_kernel<R><<<wgrid, 256, 0, st>>>(phi, sorted, offs, amax, N, C, csum, ccnt, ctl);
            cudaMemcpyAsync(prev, raw, (size_t)BH * N * sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
            count_launch(), centre_from_sums_kernel<<<wgrid, 256, 0, st>>>(csum, ccnt, amax, N, C, R, cen, hn, ctl);
        } else if (it > 1) {   // later updates: only the points whose label changed
            count_launch(), centre_delta_kernel<<<dim3((N + 255) / 256, BH), 256, 0, st>>>(phi, raw, prev, amax, N, C,
                                                                                          R, csum, ccnt, ctl);
            count_launch(), centre_from_sums_kernel<<<wgrid, 256, 0, st>>>(csum, ccnt, amax, N, C, R, cen, hn, ctl);
        }
        if (!launch_kmeans_assign_tc(phi, cen, hn, at<float>(ws, pl.o_hs), BH, N, C, R, raw, ctl, first, dbg_scores, dbg_hist,
                                     p.kmeans_iters, at<DevStatus>(ws, pl.o_status), st))
            count_launch(), kmeans_assign_kernel<R><<<agrid, 128, 0, st>>>(phi, cen, hn, N, C, raw, ctl, first,
                                                                          dbg_scores, dbg_hist, p.kmeans_iters);
        count_launch(), kmeans_check_kernel<<<bgrid, 128, 0, st>>>(ctl, BH, pl.stop_changed, first);
    }
}

void kmeans_dispatch(int R, const Plan& pl, const sparsepr_params& p, void* ws, const float* phi,
                     int C, int stage, float* cen, float* hn, float* dbg_scores, int32_t* dbg_hist,
                     int save_slot, const WarmInit* wi, int nh, int32_t* raw, cudaStream_t st) {
    switch (R) {
        case 16: kmeans_run<16>(pl, p, ws, phi, C, stage, cen, hn, dbg_scores, dbg_hist, save_slot, wi, nh, raw, st); break;
        case 32: kmeans_run<32>(pl, p, ws, phi, C, stage, cen, hn, dbg_scores, dbg_hist, save_slot, wi, nh, raw, st); break;
        case 48: kmeans_run<48>(pl, p, ws, phi, C, stage, cen, hn, dbg_scores, dbg_hist, save_slot, wi, nh, raw, st); break;
        case 64: kmeans_run<64>(pl, p, ws, phi, C, stage, cen, hn, dbg_scores, dbg_hist, save_slot, wi, nh, raw, st); break;
        default: kmeans_run<128>(pl, p, ws, phi, C, stage, cen, hn, dbg_scores, dbg_hist, save_slot, wi, nh, raw, st); break;
    }
}

template <typename T, bool RMS>
void project_dispatch(int R, const T* X, const float* F, int BH, int N, int d, const int32_t* r_eff,
                      float eps, float* phi, DevStatus* status, cudaStream_t st) {
    if (sizeof(T) == 2 && launch_project_tc(X, F, BH, N, d, R, RMS, r_eff, eps, phi, status, st)) return;
    const dim3 grid((N + 127) / 128, BH);
    const size_t smem = (size_t)d * R * sizeof(float);
    switch (R) {
        case 16: count_launch(), project_kernel<T, 16, RMS><<<grid, 128, smem, st>>>(X, F, N, d, r_eff, eps, phi); break;
        case 32: count_launch(), project_kernel<T, 32, RMS><<<grid, 128, smem, st>>>(X, F, N, d, r_eff, eps, phi); break;
        case 48: count_launch(), project_kernel<T, 48, RMS><<<grid, 128, smem, st>>>(X, F, N, d, r_eff, eps, phi); break;
        default: count_launch(), project_kernel<T, 64, RMS><<<grid, 128, smem, st>>>(X, F, N, d, r_eff, eps, phi); break;
    }
}

// Final group sort of raw labels -> compaction -> labels/perm/pos outputs.
void finalize_groups(const Plan& pl, void* ws, int C, int which, int32_t* label_out,
                     int32_t* perm_out, int32_t* pos_out, int32_t* offs_out, int32_t* ng,
                     cudaStream_t st) {
    int32_t* raw = at<int32_t>(ws, pl.o_raw);
    int32_t* hist = at<int32_t>(ws, pl.o_hist);
    int32_t* sorted = at<int32_t>(ws, pl.o_sorted);
    int32_t* offs = at<int32_t>(ws, pl.o_offs);
    int32_t* newid = at<int32_t>(ws, pl.o_newid);
    const int BH = pl.BH, N = pl.N;
    const dim3 tgrid(pl.n_sort_tiles, BH);
    count_launch(), label_hist_kernel<<<tgrid, kSortTile, 0, st>>>(raw, N, C, pl.n_sort_tiles, hist, nullptr);
    count_launch(), label_colscan_kernel<<<dim3((C + 255) / 256, BH), 256, 0, st>>>(hist, C, pl.n_sort_tiles, offs,
                                                                                   nullptr);
    count_launch(), label_offsets_kernel<<<BH, 1024, 0, st>>>(offs, N, C, nullptr);
    count_launch(), label_scatter_kernel<<<tgrid, kSortTile, scatter_smem(C), st>>>(raw, N, C, pl.n_sort_tiles, hist,
                                                                                     offs, sorted, nullptr);
    count_launch(), compact_groups_kernel<<<BH, 1024, 0, st>>>(offs, C, N, newid, offs_out, ng, which);
    count_launch(), relabel_kernel<<<grid_for((size_t)BH * N, 256), 256, 0, st>>>(raw, newid, sorted, BH, N, C,
                                                                  label_out, perm_out, pos_out);
}

// heads: output heads; perm_mul: output head h takes the permutation of head h * perm_mul.
void gather(const void* X, const int32_t* perm, const Plan& pl, int heads, int perm_mul, void* Xp, cudaStream_t st) {
    const int chunks = pl.d * pl.esz / 16;
    const size_t total = (size_t)heads * pl.N * chunks;
    count_launch(), gather_rows_kernel<<<grid_for(total, 256), 256, 0, st>>>(
        static_cast<const uint4*>(X), perm, heads, pl.N, chunks, perm_mul, static_cast<uint4*>(Xp));
}

template <typename T>
sparsepr_status partition_typed(const sparsepr_params& p, const Plan& pl, const T* Q, const T* K,
                                const T* V, const sparsepr_partition_out& out, void* ws,
                                cudaStream_t st, const WarmSource* warm) {
    const int BH = pl.BH, N = pl.N, d = pl.d;
    float* mat = at<float>(ws, pl.o_mat);
    float* FK = at<float>(ws, pl.o_FK);
    float* FQ = at<float>(ws, pl.o_FQ);
    int32_t* rq = at<int32_t>(ws, pl.o_rq);
    float* phiK = at<float>(ws, pl.o_phiK);
    float* phiQ = at<float>(ws, pl.o_phiQ);
    float* cenK = at<float>(ws, pl.o_cenK);
    float* hnK = at<float>(ws, pl.o_hnK);
    float* cenQ = at<float>(ws, pl.o_cenQ);
    float* hnQ = at<float>(ws, pl.o_hnQ);
    float* muK = at<float>(ws, pl.o_muK);
    int32_t* ctl = at<int32_t>(ws, pl.o_ctl);
    const bool dbg = (p.flags & SPARSEPR_FLAG_DEBUG_EXPORT) != 0;

    const size_t jac_smem = (size_t)(2 * d * (d + 1) + 4 * (d / 2) + 64) * sizeof(float) + (size_t)d * sizeof(int);
    auto jacobi = (d == 128) ? jacobi_factor_kernel<128> : jacobi_factor_kernel<64>;
    cudaFuncSetAttribute(jacobi, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)jac_smem);

    const bool sem_k = (p.flags & SPARSEPR_FLAG_SEMANTIC_KEYS) != 0;
    const bool sem_q = (p.flags & SPARSEPR_FLAG_SEMANTIC_QUERIES) != 0;
    const size_t n8 = (size_t)BH * N * d / 8;
    int32_t* coldK = at<int32_t>(ws, pl.o_warm) + 1;
    int32_t* coldQ = coldK + BH;
    // The K/V side runs once per K/V head: BHk = BH / G heads (GQA, §4.3);
    // K and V are [BHk, N, d].
    const int G = pl.G, BHk = BH / G;
    const size_t nk8 = (size_t)BHk * N * d / 8;
    if (sem_k) {
        // semantic K/V groups: k-means on the raw key rows (RKp = d)
        count_launch(), identity_factor_kernel<<<BHk, 256, 0, st>>>(FK, d, pl.RKp, nullptr);
        count_launch(), raw_coords_kernel<T><<<grid_for(nk8, 256), 256, 0, st>>>(K, nk8, phiK);
    } else {
        // 1-2. key-response metric and factor (§4.1); under GQA the mean of
        // the G query heads' sampled metrics
        count_launch(), sampled_gram_kernel<T><<<dim3(d / 32, d / 32, BH), dim3(32, 8), 0, st>>>(Q, N, d, pl.Ms_eff,
                                                                                                mat);
        float* matK = mat;
        if (G > 1) {
            matK = at<float>(ws, pl.o_G);   // fit scratch, free during the partition
            const size_t tot = (size_t)BHk * d * d;
            count_launch(), mean_heads_kernel<<<grid_for(tot, 256), 256, 0, st>>>(mat, G, (size_t)d * d, tot, matK);
        }
        // warm start (C.1): subspace iteration from the previous factor; heads it
        // cannot factor (or every head, without a previous state) take Jacobi
        if (warm)
            launch_warm_factor(matK, warm->F_K, pl.RKp, warm->fk_stride, pl.rK_eff, nullptr, 1.f / sqrtf((float)d),
                               FK, pl.RKp, nullptr, coldK, warm->valid, BHk, d, st);
        count_launch(), jacobi<<<BHk, 1024, jac_smem, st>>>(matK, FK, pl.RKp, pl.rK_eff, nullptr,
                                                           1.f / sqrtf((float)d), nullptr, 16, warm ? coldK : nullptr);
        project_dispatch<T, false>(pl.RKp, K, FK, BHk, N, d, nullptr, 0.f, phiK, at<DevStatus>(ws, pl.o_status), st);
    }
    // 3. paired K/V groups
    WarmInit wiK{}, wiQ{};
    if (warm) {
        wiK = WarmInit{warm->k_centroid, warm->n_groups, 1, G, FK, d, false, nullptr, 0.f, warm->valid};
        wiQ = WarmInit{warm->q_centroid, warm->n_groups, 0, 1, FQ, d, !sem_q, rq, p.eps_rms, warm->valid};
    }
    int32_t* raw = at<int32_t>(ws, pl.o_raw);
    int32_t* rawK = G > 1 ? at<int32_t>(ws, pl.o_rawkv) : raw;
    kmeans_dispatch(pl.RKp, pl, p, ws, phiK, pl.Ck, 0, cenK, hnK, dbg ? out.debug_kv_scores : nullptr,
                    dbg ? out.debug_kv_hist : nullptr, -1, warm ? &wiK : nullptr, BHk, rawK, st);
    auto to_query_heads = [&](const void* src, void* dst, size_t words_per_head) {
        const size_t tot = (size_t)BH * words_per_head;
        count_launch(), broadcast_heads_kernel<<<grid_for(tot, 256), 256, 0, st>>>(
            static_cast<const uint32_t*>(src), words_per_head, tot, G, static_cast<uint32_t*>(dst));
    };
    if (G > 1) {   // the K/V groups of each K/V head serve its G query heads
        to_query_heads(rawK, raw, (size_t)N);
        count_launch(), broadcast_iters_kernel<<<1, 1, 0, st>>>(ctl, BH, G);
        if (out.kv_centres) to_query_heads(cenK, out.kv_centres, (size_t)pl.Ck * pl.RKp);
    } else if (out.kv_centres) {
        cudaMemcpyAsync(out.kv_centres, cenK, (size_t)BH * pl.Ck * pl.RKp * 4, cudaMemcpyDeviceToDevice, st);
    }
    finalize_groups(pl, ws, pl.Ck, 1, out.kv_label, out.perm_kv, nullptr, out.kv_offsets, out.n_groups, st);
    // one permuted K/V per K/V head, in the group order its query heads share (GQA)
    gather(K, out.perm_kv, pl, BHk, G, out.Kp, st);
    gather(V, out.perm_kv, pl, BHk, G, out.Vp, st);
    // 4. centroids, query metric, factor, coordinates (§4.1, B.2)
    count_launch(), group_mean_kernel<T><<<dim3(pl.Ck, BH), d, 0, st>>>(static_cast<const T*>(out.Kp), out.kv_offsets,
                                                        out.n_groups, 1, N, pl.Ck, d, G, out.k_centroid);
    count_launch(), group_mean_kernel<T><<<dim3(pl.Ck, BH), d, 0, st>>>(static_cast<const T*>(out.Vp), out.kv_offsets,
                                                        out.n_groups, 1, N, pl.Ck, d, G, out.v_centroid);
    if (sem_q) {
        // semantic query groups: k-means on the raw query rows (RQp = d)
        count_launch(), identity_factor_kernel<<<BH, 256, 0, st>>>(FQ, d, pl.RQp, rq);
        count_launch(), raw_coords_kernel<T><<<grid_for(n8, 256), 256, 0, st>>>(Q, n8, phiQ);
    } else {
        count_launch(), centroid_mean_kernel<<<BH, d, 0, st>>>(out.k_centroid, out.n_groups, pl.Ck, d, muK);
        count_launch(), centred_gram_kernel<<<dim3(d / 32, d / 32, BH), dim3(32, 8), 0, st>>>(out.k_centroid, muK,
                                                                              out.n_groups, pl.Ck, d, mat);
        if (warm)
            launch_warm_factor(mat, warm->F_Q, pl.RQp, 1, p.rQ, out.n_groups, 1.f, FQ, pl.RQp, rq, coldQ,
                               warm->valid, BH, d, st);
        count_launch(), jacobi<<<BH, 1024, jac_smem, st>>>(mat, FQ, pl.RQp, p.rQ, out.n_groups, 1.f, rq, 16,
                                                          warm ? coldQ : nullptr);
        project_dispatch<T, true>(pl.RQp, Q, FQ, BH, N, d, rq, p.eps_rms, phiQ, at<DevStatus>(ws, pl.o_status), st);
    }
    // 5. query groups
    kmeans_dispatch(pl.RQp, pl, p, ws, phiQ, pl.Cq, 1, cenQ, hnQ, dbg ? out.debug_q_scores : nullptr,
                    dbg ? out.debug_q_hist : nullptr, kCtlItersK, warm ? &wiQ : nullptr, BH, raw, st);
    count_launch(), kmeans_reset_kernel<<<(BH + 127) / 128, 128, 0, st>>>(ctl, BH, kCtlItersQ);
    if (out.q_centres) cudaMemcpyAsync(out.q_centres, cenQ, (size_t)BH * pl.Cq * pl.RQp * 4, cudaMemcpyDeviceToDevice, st);
    finalize_groups(pl, ws, pl.Cq, 0, out.q_label, out.perm_q, out.pos_q, out.q_offsets, out.n_groups, st);
    gather(Q, out.perm_q, pl, BH, 1, out.Qp, st);
    count_launch(), group_mean_kernel<T><<<dim3(pl.Cq, BH), d, 0, st>>>(static_cast<const T*>(out.Qp), out.q_offsets,
                                                        out.n_groups, 0, N, pl.Cq, d, 1, out.q_centroid);
    // c_a (phi_Q space) into the query-centre buffer, then d_i (A.2)
    count_launch(), group_mean_indirect_kernel<<<dim3(pl.Cq, BH), pl.RQp > 64 ? pl.RQp : 64, 0, st>>>(
                                                              phiQ, out.perm_q, out.q_offsets,
                                                              out.n_groups, N, pl.Cq, pl.RQp, cenQ);
    count_launch(), query_dist_kernel<<<grid_for((size_t)BH * N, 256), 256, 0, st>>>(phiQ, cenQ, out.q_label, BH, N,
                                                                     pl.Cq, pl.RQp, out.q_dist);
    count_launch(), iters_out_kernel<<<(BH + 127) / 128, 128, 0, st>>>(ctl, BH, out.kmeans_iters_run);
    if (out.F_K) {
        if (G > 1) to_query_heads(FK, out.F_K, (size_t)d * pl.RKp);
        else cudaMemcpyAsync(out.F_K, FK, (size_t)BH * d * pl.RKp * 4, cudaMemcpyDeviceToDevice, st);
    }
    if (out.F_Q) cudaMemcpyAsync(out.F_Q, FQ, (size_t)BH * d * pl.RQp * 4, cudaMemcpyDeviceToDevice, st);
    if (out.phi_K) {
        if (G > 1) to_query_heads(phiK, out.phi_K, (size_t)N * pl.RKp);
        else cudaMemcpyAsync(out.phi_K, phiK, (size_t)BH * N * pl.RKp * 4, cudaMemcpyDeviceToDevice, st);
    }
    if (out.phi_Q) cudaMemcpyAsync(out.phi_Q, phiQ, (size_t)BH * N * pl.RQp * 4, cudaMemcpyDeviceToDevice, st);
    return cuda_status(cudaGetLastError());
}

}  // namespace

sparsepr_status run_partition(const sparsepr_params& p, const Plan& pl, const void* Q, const void* K,
                              const void* V, const sparsepr_partition_out& out, void* ws,
                              cudaStream_t st, const WarmSource* warm) {
    if (p.dtype == SPARSEPR_BF16)
        return partition_typed<__nv_bfloat16>(p, pl, static_cast<const __nv_bfloat16*>(Q),
                                              static_cast<const __nv_bfloat16*>(K),
                                              static_cast<const __nv_bfloat16*>(V), out, ws, st, warm);
    return partition_typed<float>(p, pl, static_cast<const float*>(Q), static_cast<const float*>(K),
                                  static_cast<const float*>(V), out, ws, st, warm);
}

}  // namespace spr
