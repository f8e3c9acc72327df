// Probe-fitted residual reconstruction ("Partition the Support, Reconstruct
// the Residual", §4.2, A.2, A.3, D.3).
//
//   w_p = |G_a| / m_a,  alpha_p = w_p / sum w,  w~_p = M alpha_p
//   mu_X = sum alpha x_p,  sigma = sqrt(sum alpha (x_p - mu_X)^2 + eps),
//   Xbar = (X - mu_X)/sigma,  mu_R = sum alpha R_p,  Rbar = R - mu_R
//   B = (Xbar^T W Xbar + lambda I)^-1 Xbar^T W Rbar     (Cholesky)
//   O^_i = O^dense_i for probes,  O^sp_i + mu_R + Xbar_i B otherwise.
//
// The fit is small (M x d and d x d per head) and runs in fp64; B and the
// statistics are stored in fp32 for the fp32 apply.  Restricted families
// (D.4: diagonal, scalar, mean-only) replace the solve, and a rank-r
// truncation (D.3) projects B on the leading eigenvectors of Rbar^T W Rbar.
#include "common.cuh"
#include "internal.h"

namespace spr {

__device__ __forceinline__ double probe_alpha(int p, const int32_t* pg, const int32_t* alloc, const int32_t* qo,
                                              double sum_w) {
    const int a = pg[p];
    return ((double)(qo[a + 1] - qo[a]) / (double)alloc[a]) / sum_w;
}

// Weighted statistics; one thread per channel j.
__global__ void fit_stats_kernel(const float* __restrict__ Xs, const float* __restrict__ Xd,
                                 const int32_t* __restrict__ probe_group, const int32_t* __restrict__ alloc,
                                 const int32_t* __restrict__ q_off, const int32_t* __restrict__ ng,
                                 int32_t* __restrict__ psum, int Cq, int Mp, int d, float eps_std,
                                 double* __restrict__ fstat, float* __restrict__ mu_x, float* __restrict__ sigma,
                                 float* __restrict__ mu_r) {
    constexpr int kChunk = 1024;
    __shared__ double alp[kChunk];     // alpha_p of the current chunk of probes
    __shared__ int part[32];
    __shared__ int sum_w;
    const int bh = blockIdx.x, j = threadIdx.x, nt = blockDim.x;
    const int32_t* pg = probe_group + (size_t)bh * Mp;
    const int32_t* al = alloc + (size_t)bh * Cq;
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    {   // sum_p w_p = sum of |G_a| over groups holding probes (fixed-order block sum)
        int s = 0;
        const int Cqp = ng[bh * 2 + 0];
        for (int a = j; a < Cqp; a += nt)
            if (al[a] > 0) s += qo[a + 1] - qo[a];
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if ((j & 31) == 0) part[j >> 5] = s;
        __syncthreads();
        if (j == 0) {
            int t = 0;
            for (int w = 0; w < nt / 32; ++w) t += part[w];
            sum_w = t;
            psum[bh] = t;
        }
        __syncthreads();
    }
    const float* X = Xs + (size_t)bh * Mp * d;
    const float* D = Xd + (size_t)bh * Mp * d;
    const double sw = (double)sum_w;
    double mx = 0.0, mr = 0.0;
    for (int c0 = 0; c0 < Mp; c0 += kChunk) {
        const int n = min(kChunk, Mp - c0);
        __syncthreads();
        for (int e = j; e < n; e += nt) alp[e] = probe_alpha(c0 + e, pg, al, qo, sw);
        __syncthreads();
#pragma unroll 4
        for (int q = 0; q < n; ++q) {
            const double x = X[(size_t)(c0 + q) * d + j];
            mx += alp[q] * x;
            mr += alp[q] * ((double)D[(size_t)(c0 + q) * d + j] - x);
        }
    }
    double var = 0.0;
    for (int c0 = 0; c0 < Mp; c0 += kChunk) {
        const int n = min(kChunk, Mp - c0);
        __syncthreads();
        for (int e = j; e < n; e += nt) alp[e] = probe_alpha(c0 + e, pg, al, qo, sw);
        __syncthreads();
#pragma unroll 4
        for (int q = 0; q < n; ++q) {
            const double c = (double)X[(size_t)(c0 + q) * d + j] - mx;
            var += alp[q] * c * c;
        }
    }
    const double sg = sqrt(var + (double)eps_std);
    double* fs = fstat + (size_t)bh * 3 * d;
    fs[j] = mx;
    fs[d + j] = sg;
    fs[2 * d + j] = mr;
    mu_x[(size_t)bh * d + j] = (float)mx;
    sigma[(size_t)bh * d + j] = (float)sg;
    mu_r[(size_t)bh * d + j] = (float)mr;
}

// Rows i0..i0+7 of G = Xbar^T W Xbar + lambda I and of RHS = Xbar^T W Rbar
// (and, with S, of Rbar^T W Rbar).  Probes are taken kGramChunk at a time:
// their weights times the block's eight standardised rows are staged in
// shared memory, then each thread accumulates its column j (probes in index
// order).
constexpr int kGramChunk = 1024;
__global__ void fit_gram_kernel(const float* __restrict__ Xs, const float* __restrict__ Xd,
                                const int32_t* __restrict__ probe_group, const int32_t* __restrict__ alloc,
                                const int32_t* __restrict__ q_off, const int32_t* __restrict__ psum, int Cq, int Mp,
                                int d, double lambda, const double* __restrict__ fstat, double* __restrict__ G,
                                double* __restrict__ rhs, double* __restrict__ S) {
    constexpr int RI = 8;
    extern __shared__ double xbi[];   // [kGramChunk][RI] W_p * Xbar[p][i0 + u]; then W_p * Rbar (with S)
    double* rbi = xbi + kGramChunk * RI;
    const int bh = blockIdx.y, i0 = blockIdx.x * RI, j = threadIdx.x;
    const float* X = Xs + (size_t)bh * Mp * d;
    const float* Dp = Xd + (size_t)bh * Mp * d;
    const int32_t* pg = probe_group + (size_t)bh * Mp;
    const int32_t* al = alloc + (size_t)bh * Cq;
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    const double* fs = fstat + (size_t)bh * 3 * d;
    const double sw = (double)psum[bh];
    const double mxj = fs[j], sgj = fs[d + j], mrj = fs[2 * d + j];
    double g[RI], h[RI], sr[RI];
#pragma unroll
    for (int u = 0; u < RI; ++u) g[u] = h[u] = sr[u] = 0.0;
    for (int c0 = 0; c0 < Mp; c0 += kGramChunk) {
        const int n = min(kGramChunk, Mp - c0);
        __syncthreads();   // the previous chunk is consumed
        for (int e = j; e < n * RI; e += blockDim.x) {
            const int p = c0 + e / RI, u = e % RI;
            const double wt = (double)Mp * probe_alpha(p, pg, al, qo, sw);
            const double xv = (double)X[(size_t)p * d + i0 + u];
            xbi[e] = wt * ((xv - fs[i0 + u]) / fs[d + i0 + u]);
            if (S != nullptr) rbi[e] = wt * (((double)Dp[(size_t)p * d + i0 + u] - xv) - fs[2 * d + i0 + u]);
        }
        __syncthreads();
        for (int q = 0; q < n; ++q) {
            const int p = c0 + q;
            const double xj = (double)X[(size_t)p * d + j];
            const double xbj = (xj - mxj) / sgj;
            const double rbj = ((double)Dp[(size_t)p * d + j] - xj) - mrj;
#pragma unroll
            for (int u = 0; u < RI; ++u) {
                const double xb = xbi[q * RI + u];
                g[u] += xb * xbj;
                h[u] += xb * rbj;
            }
            if (S != nullptr) {
#pragma unroll
                for (int u = 0; u < RI; ++u) sr[u] += rbi[q * RI + u] * rbj;
            }
        }
    }
#pragma unroll
    for (int u = 0; u < RI; ++u) {
        const int i = i0 + u;
        G[((size_t)bh * d + i) * d + j] = g[u] + (i == j ? lambda : 0.0);
        rhs[((size_t)bh * d + i) * d + j] = h[u];
        if (S != nullptr) S[((size_t)bh * d + i) * d + j] = sr[u];
    }
}

// Restricted families (D.4) from the diagonals of G = Xbar^T W Xbar + lambda I
// and RHS = Xbar^T W Rbar: diagonal b_j = RHS_jj / G_jj, scalar
// a = tr(RHS) / tr(G) (tr G carries lambda d), mean-only B = 0.  One thread per
// channel j.
__global__ void fit_restricted_kernel(const double* __restrict__ G, const double* __restrict__ rhs, int d,
                                      int family, float* __restrict__ Bout) {
    __shared__ double red[2][32];
    const int bh = blockIdx.x, j = threadIdx.x, lane = j & 31, wid = j >> 5;
    const double gjj = G[((size_t)bh * d + j) * d + j];
    const double hjj = rhs[((size_t)bh * d + j) * d + j];
    double sg = gjj, sh = hjj;
    for (int o = 16; o > 0; o >>= 1) {
        sg += __shfl_xor_sync(0xffffffffu, sg, o);
        sh += __shfl_xor_sync(0xffffffffu, sh, o);
    }
    if (lane == 0) {
        red[0][wid] = sg;
        red[1][wid] = sh;
    }
    __syncthreads();
    double tg = 0.0, th = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {   // fixed order
        tg += red[0][w];
        th += red[1][w];
    }
    double bj = 0.0;
    if (family == SPARSEPR_CORRECTION_DIAGONAL) bj = hjj / gjj;
    else if (family == SPARSEPR_CORRECTION_SCALAR) bj = th / tg;
    float* Bh = Bout + (size_t)bh * d * d;
    for (int i = 0; i < d; ++i) Bh[(size_t)i * d + j] = (i == j) ? (float)bj : 0.f;
}

// S (fp64, symmetric) to fp32 for the Jacobi eigen-factor.
__global__ void to_f32_kernel(const double* __restrict__ S, size_t n, float* __restrict__ out) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x)
        out[e] = (float)S[e];
}

// Rank truncation (D.3): B <- B U_r U_r^T, U_r the unit-normalised nonzero
// leading columns of the eigen-factor Fv (d x d, columns u_c sqrt(lambda_c)).
__global__ void fit_project_kernel(const float* __restrict__ Fv, int d, int r, float* __restrict__ Bm) {
    extern __shared__ float pj[];
    float* U = pj;               // [d][r]
    float* T = pj + d * r;       // [d][r] = B U
    __shared__ float inv[128];
    const int bh = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const float* Fh = Fv + (size_t)bh * d * d;
    float* Bh = Bm + (size_t)bh * d * d;
    for (int c = tid; c < r; c += nt) {
        double ss = 0.0;
        for (int k = 0; k < d; ++k) ss += (double)Fh[(size_t)k * d + c] * Fh[(size_t)k * d + c];
        inv[c] = ss > 0.0 ? (float)(1.0 / sqrt(ss)) : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < d * r; e += nt) U[e] = Fh[(size_t)(e / r) * d + (e % r)] * inv[e % r];
    __syncthreads();
    for (int e = tid; e < d * r; e += nt) {
        const int i = e / r, c = e % r;
        double acc = 0.0;
        for (int k = 0; k < d; ++k) acc += (double)Bh[(size_t)i * d + k] * U[k * r + c];
        T[e] = (float)acc;
    }
    __syncthreads();
    for (int e = tid; e < d * d; e += nt) {
        const int i = e / d, j = e % d;
        double acc = 0.0;
        for (int c = 0; c < r; ++c) acc += (double)T[i * r + c] * U[j * r + c];
        Bh[e] = (float)acc;
    }
}

// Cholesky G = L L^T in shared memory, then each thread solves one column
// of B = G^-1 RHS by forward and back substitution (RHS overwritten in place).
__global__ void fit_solve_kernel(const double* __restrict__ G, double* __restrict__ rhs, int d,
                                 float* __restrict__ Bout, DevStatus* status) {
    extern __shared__ double Ls[];
    __shared__ int fail;
    const int bh = blockIdx.x, tid = threadIdx.x;
    const int ld = d + 1;
    const double* Gh = G + (size_t)bh * d * d;
    for (int e = tid; e < d * d; e += blockDim.x) Ls[(e / d) * ld + (e % d)] = Gh[e];
    if (tid == 0) fail = 0;
    __syncthreads();
    for (int k = 0; k < d; ++k) {
        if (tid == 0) {
            const double piv = Ls[k * ld + k];
            if (!(piv > 0.0)) {
                fail = 1;
                record_status(status, SPARSEPR_NUMERIC, 60);
            } else {
                Ls[k * ld + k] = sqrt(piv);
            }
        }
        __syncthreads();
        if (fail) break;
        const double lkk = Ls[k * ld + k];
        for (int i = k + 1 + tid; i < d; i += blockDim.x) Ls[i * ld + k] /= lkk;
        __syncthreads();
        for (int i = k + 1 + tid; i < d; i += blockDim.x) {
            const double lik = Ls[i * ld + k];
            for (int j = k + 1; j <= i; ++j) Ls[i * ld + j] -= lik * Ls[j * ld + k];
        }
        __syncthreads();
    }
    if (fail) {
        for (int e = tid; e < d * d; e += blockDim.x) Bout[(size_t)bh * d * d + e] = 0.f;
        return;
    }
    // Forward and back substitution for 64 right-hand-side columns at a time,
    // staged in shared memory (Ys[i * 65 + c]); thread c < 64 solves column
    // j0 + c on its own (four partial sums in a fixed order break the
    // dependency chain), so no barrier is needed inside a solve.
    const double* R = rhs + (size_t)bh * d * d;
    double* Ys = Ls + d * ld;
    constexpr int W = 64, LDY = W + 1;
    for (int j0 = 0; j0 < d; j0 += W) {
        __syncthreads();
        for (int e = tid; e < d * W; e += blockDim.x) Ys[(e / W) * LDY + (e % W)] = R[(size_t)(e / W) * d + j0 + (e % W)];
        __syncthreads();
        if (tid < W) {
            double* y = Ys + tid;
            for (int i = 0; i < d; ++i) {   // L y = rhs
                const double* li = Ls + i * ld;
                double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
                int k = 0;
                for (; k + 4 <= i; k += 4) {
                    a0 += li[k] * y[k * LDY];
                    a1 += li[k + 1] * y[(k + 1) * LDY];
                    a2 += li[k + 2] * y[(k + 2) * LDY];
                    a3 += li[k + 3] * y[(k + 3) * LDY];
                }
                for (; k < i; ++k) a0 += li[k] * y[k * LDY];
                y[i * LDY] = (y[i * LDY] - ((a0 + a1) + (a2 + a3))) / li[i];
            }
            for (int i = d - 1; i >= 0; --i) {   // L^T b = y
                double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
                int k = i + 1;
                for (; k + 4 <= d; k += 4) {
                    a0 += Ls[k * ld + i] * y[k * LDY];
                    a1 += Ls[(k + 1) * ld + i] * y[(k + 1) * LDY];
                    a2 += Ls[(k + 2) * ld + i] * y[(k + 2) * LDY];
                    a3 += Ls[(k + 3) * ld + i] * y[(k + 3) * LDY];
                }
                for (; k < d; ++k) a0 += Ls[k * ld + i] * y[k * LDY];
                y[i * LDY] = (y[i * LDY] - ((a0 + a1) + (a2 + a3))) / Ls[i * ld + i];
            }
        }
        __syncthreads();
        for (int e = tid; e < d * W; e += blockDim.x)
            Bout[((size_t)bh * d + (e / W)) * d + j0 + (e % W)] = (float)Ys[(e / W) * LDY + (e % W)];
    }
}

// O_out[perm_q[p]] for 64 permuted rows per block: probe rows copy O^dense,
// the others get O^sp + mu_R + ((O^sp - mu_X)/sigma) B.
template <int D>
__global__ void __launch_bounds__(256) apply_kernel(const float* __restrict__ O_sp, const float* __restrict__ Bm,
                                                    const float* __restrict__ mu_x, const float* __restrict__ sigma,
                                                    const float* __restrict__ mu_r, const int32_t* __restrict__ pslot,
                                                    const float* __restrict__ probe_dense,
                                                    const int32_t* __restrict__ perm_q, int N, int Mp,
                                                    float* __restrict__ O_out) {
    constexpr int RT = 64, CG = D / 16;   // rows per block, columns per thread
    extern __shared__ float sm[];
    float* Bs = sm;                 // [D][D]
    float* Xs = Bs + D * D;         // [RT][D+4]
    float* st = Xs + RT * (D + 4);  // mu_x, sigma, mu_r
    const int bh = blockIdx.y, p0 = blockIdx.x * RT, tid = threadIdx.x;
    const float* Bh = Bm + (size_t)bh * D * D;
    for (int e = tid; e < D * D; e += blockDim.x) Bs[e] = Bh[e];
    for (int e = tid; e < D; e += blockDim.x) {
        st[e] = mu_x[(size_t)bh * D + e];
        st[D + e] = sigma[(size_t)bh * D + e];
        st[2 * D + e] = mu_r[(size_t)bh * D + e];
    }
    __syncthreads();
    for (int e = tid; e < RT * D; e += blockDim.x) {
        const int r = e / D, t = e % D;
        const int p = p0 + r;
        Xs[r * (D + 4) + t] = (p < N) ? (O_sp[((size_t)bh * N + p) * D + t] - st[t]) / st[D + t] : 0.f;
    }
    __syncthreads();
    const int rg = tid / 16, cg = tid % 16;
    float acc[4][CG];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < CG; ++v) acc[u][v] = 0.f;
    for (int t = 0; t < D; ++t) {
        float xb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) xb[u] = Xs[(rg * 4 + u) * (D + 4) + t];
        const float* br = Bs + t * D + cg * CG;
#pragma unroll
        for (int v = 0; v < CG; ++v) {
            const float b = br[v];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u][v] = fmaf(xb[u], b, acc[u][v]);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int p = p0 + rg * 4 + u;
        if (p >= N) continue;
        const size_t src = (size_t)bh * N + p;
        const int slot = pslot[src];
        float* dst = O_out + ((size_t)bh * N + perm_q[src]) * D + cg * CG;
        if (slot >= 0) {
            const float* pd = probe_dense + ((size_t)bh * Mp + slot) * D + cg * CG;
#pragma unroll
            for (int v = 0; v < CG; ++v) dst[v] = pd[v];
        } else {
            const float* x = O_sp + src * D + cg * CG;
#pragma unroll
            for (int v = 0; v < CG; ++v) dst[v] = x[v] + st[2 * D + cg * CG + v] + acc[u][v];
        }
    }
}

// pslot[permuted row] = probe slot, for the probe rows.
__global__ void probe_slot_kernel(const int32_t* __restrict__ probe_idx, const int32_t* __restrict__ pos_q, int BH,
                                  int N, int Mp, int32_t* __restrict__ pslot) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= BH * Mp) return;
    const size_t bh = e / Mp;
    pslot[bh * N + pos_q[bh * N + probe_idx[e]]] = e - (int)bh * Mp;
}

__global__ void fill_kernel(float* __restrict__ x, int n, float v) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) x[i] = v;
}

// ================================================================ host side
sparsepr_status run_fit(const sparsepr_params& p, const Plan& pl, const sparsepr_partition_out& part,
                        const sparsepr_route_out& r, const float* probe_sparse, const float* probe_dense,
                        const sparsepr_fit_out& f, void* ws, cudaStream_t st) {
    const int BH = pl.BH, d = pl.d, Mp = pl.Mp;
    double* fstat = at<double>(ws, pl.o_fstat);
    double* G = at<double>(ws, pl.o_G);
    double* rhs = at<double>(ws, pl.o_rhs);
    const int32_t* alloc = r.probe_alloc;
    int32_t* psum = at<int32_t>(ws, pl.o_psum);
    DevStatus* status = at<DevStatus>(ws, pl.o_status);
    if (Mp == 0) {   // no probes: no correction (B = 0, mu = 0, sigma = 1)
        cudaMemsetAsync(f.B, 0, (size_t)BH * d * d * 4, st);
        cudaMemsetAsync(f.mu_x, 0, (size_t)BH * d * 4, st);
        cudaMemsetAsync(f.mu_r, 0, (size_t)BH * d * 4, st);
        count_launch(), fill_kernel<<<(BH * d + 255) / 256, 256, 0, st>>>(f.sigma, BH * d, 1.f);
        return cuda_status(cudaGetLastError());
    }
    count_launch(), fit_stats_kernel<<<BH, d, 0, st>>>(probe_sparse, probe_dense, r.probe_group, alloc, part.q_offsets,
                                       part.n_groups, psum, pl.Cq, Mp, d, p.eps_std, fstat, f.mu_x, f.sigma,
                                       f.mu_r);
    const bool trunc = p.residual_rank > 0 && p.residual_rank < d;
    double* S = trunc ? at<double>(ws, pl.o_S) : nullptr;
    // 8 staged rows per probe of a chunk (twice with S)
    const size_t gsmem = (size_t)kGramChunk * 8 * sizeof(double) * (trunc ? 2 : 1);
    cudaFuncSetAttribute(fit_gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsmem);
    count_launch(), fit_gram_kernel<<<dim3(d / 8, BH), d, gsmem, st>>>(probe_sparse, probe_dense, r.probe_group, alloc,
                                                                       part.q_offsets, psum, pl.Cq, Mp, d, p.lambda,
                                                                       fstat, G, rhs, S);
    if (p.correction == SPARSEPR_CORRECTION_FULL) {
        const size_t smem = (size_t)(d * (d + 1) + d * 65) * sizeof(double);
        cudaFuncSetAttribute(fit_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        count_launch(), fit_solve_kernel<<<BH, d, smem, st>>>(G, rhs, d, f.B, status);
    } else {
        count_launch(), fit_restricted_kernel<<<BH, d, 0, st>>>(G, rhs, d, p.correction, f.B);
    }
    if (trunc) {
        // leading right singular vectors of W^1/2 Rbar = eigenvectors of Rbar^T W Rbar
        float* Sf = at<float>(ws, pl.o_mat);
        float* Fv = reinterpret_cast<float*>(G);       // G is consumed; d x d floats per head fit in it
        count_launch(), to_f32_kernel<<<(BH * d * d + 255) / 256, 256, 0, st>>>(S, (size_t)BH * d * d, Sf);
        launch_jacobi_factor(Sf, Fv, d, p.residual_rank, BH, d, st);
        const size_t psmem = (size_t)2 * d * p.residual_rank * sizeof(float);
        cudaFuncSetAttribute(fit_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psmem);
        count_launch(), fit_project_kernel<<<BH, 256, psmem, st>>>(Fv, d, p.residual_rank, f.B);
    }
    return cuda_status(cudaGetLastError());
}

sparsepr_status run_apply(const sparsepr_params& p, const Plan& pl, const sparsepr_partition_out& part,
                          const sparsepr_route_out& r, const float* O_sp, const float* probe_dense,
                          const sparsepr_fit_out& f, float* O_out, void* ws, cudaStream_t st) {
    (void)p;
    int32_t* pslot = at<int32_t>(ws, pl.o_pslot);
    cudaMemsetAsync(pslot, 0xff, (size_t)pl.BH * pl.N * sizeof(int32_t), st);
    if (pl.Mp > 0)
        count_launch(), probe_slot_kernel<<<(pl.BH * pl.Mp + 255) / 256, 256, 0, st>>>(r.probe_idx, part.pos_q, pl.BH, pl.N, pl.Mp,
                                                                       pslot);
    if (launch_apply_tc(pl, part, O_sp, probe_dense, f, pslot, O_out, at<DevStatus>(ws, pl.o_status), st))
        return cuda_status(cudaGetLastError());
    const int d = pl.d;
    const size_t smem = (size_t)(d * d + 64 * (d + 4) + 3 * d) * sizeof(float);
    const dim3 grid((pl.N + 63) / 64, pl.BH);
    if (d == 128) {
        cudaFuncSetAttribute(apply_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        count_launch(), apply_kernel<128><<<grid, 256, smem, st>>>(O_sp, f.B, f.mu_x, f.sigma, f.mu_r, pslot, probe_dense,
                                                  part.perm_q, pl.N, pl.Mp, O_out);
    } else {
        cudaFuncSetAttribute(apply_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        count_launch(), apply_kernel<64><<<grid, 256, smem, st>>>(O_sp, f.B, f.mu_x, f.sigma, f.mu_r, pslot, probe_dense,
                                                 part.perm_q, pl.N, pl.Mp, O_out);
    }
    return cuda_status(cudaGetLastError());
}

}  // namespace spr
