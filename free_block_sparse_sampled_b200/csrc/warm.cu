// Cross-call warm start of the partition (paper Appendix C.1, "Warm start"
// paragraph, and Table C.1's subsequent k-means iteration limit).
//
//   warm_factor_kernel  metric factor of this call from the previous factor:
//                       two subspace iterations  Y = M Q,  Q = Y L^-T  with
//                       L L^T = Y^T Y (Cholesky QR), then F = Q C scale with
//                       C C^T = Q^T M Q.  F F^T is the metric restricted to
//                       the iterated subspace.  A vanishing pivot (square not
//                       above 1e-12 x the largest diagonal entry) marks the
//                       head for the cold eigen-factor instead.
//   warm_init_kernel    initial k-means centres: the previous call's raw-space
//                       centroids projected with this call's factor
//                       (RMS-normalised for queries), TF32-rounded like every
//                       centre; centres past the previous group count are the
//                       cold start's sampled rows.
//
// One block per head for the factor (d x d metric and d x r bases in shared
// memory, fp64 Gram matrices and triangular solves, fp32 basis); one warp per
// centre for the initialisation.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace spr {

namespace {

constexpr int kWarmThreads = 512;
constexpr int kWarmRW = kMaxRank;            // basis columns held in shared memory
constexpr double kWarmPivotRel = 1e-12;

template <int D>
struct WarmSmem {
    static constexpr int ldM = D + 1;        // fp32 metric, padded rows
    static constexpr int ldY = kWarmRW + 1;  // fp64 rows, odd stride against bank conflicts
    static constexpr size_t bytes_M = (size_t)D * ldM * 4;
    static constexpr size_t bytes_Q = (size_t)D * kWarmRW * 4;
    static constexpr size_t bytes_Y = (size_t)D * ldY * 8;
    static constexpr size_t bytes_G = (size_t)kWarmRW * ldY * 8;
    static constexpr size_t off_Q = bytes_M;
    static constexpr size_t off_Y = (off_Q + bytes_Q + 15) / 16 * 16;
    static constexpr size_t off_G = off_Y + bytes_Y;
    static constexpr size_t off_misc = off_G + bytes_G;
    static constexpr size_t total = off_misc + 64;
};

// In-place lower Cholesky of the r x r leading block of G (row stride ld;
// only the lower triangle is read).  false when a pivot vanishes.
__device__ bool block_cholesky(double* G, int ld, int r, int* sflag, double* sdmax) {
    const int tid = threadIdx.x, nt = blockDim.x;
    if (tid == 0) {
        double m = 0.0;
        for (int j = 0; j < r; ++j) m = fmax(m, G[j * ld + j]);
        *sdmax = m;
        *sflag = 0;
    }
    __syncthreads();
    const double floor_p = kWarmPivotRel * *sdmax;
    for (int j = 0; j < r; ++j) {
        if (tid == 0) {
            const double pv = G[j * ld + j];
            if (pv > floor_p && pv < INFINITY) G[j * ld + j] = sqrt(pv);
            else *sflag = 1;
        }
        __syncthreads();
        if (*sflag) return false;
        const double ljj = G[j * ld + j];
        for (int i = j + 1 + tid; i < r; i += nt) G[i * ld + j] /= ljj;
        __syncthreads();
        const int w = r - j - 1;
        for (int e = tid; e < w * w; e += nt) {
            const int i = j + 1 + e / w, k = j + 1 + e % w;
            if (k <= i) G[i * ld + k] -= G[i * ld + j] * G[k * ld + j];
        }
        __syncthreads();
    }
    return true;
}

// Y = M Q (fp64 accumulation of fp32 operands), d x r.
template <int D>
__device__ void metric_times_basis(const float* Ms, const float* Qs, double* Ys, int r) {
    using S = WarmSmem<D>;
    for (int e = threadIdx.x; e < D * r; e += blockDim.x) {
        const int i = e / r, c = e % r;
        double acc = 0.0;
#pragma unroll 8
        for (int k = 0; k < D; ++k) acc = fma((double)Ms[i * S::ldM + k], (double)Qs[k * kWarmRW + c], acc);
        Ys[i * S::ldY + c] = acc;
    }
}

template <int D>
__global__ void __launch_bounds__(kWarmThreads) warm_factor_kernel(
    const float* __restrict__ Min, const float* Fprev, int ld_prev, int prev_stride, int r_req,
    const int32_t* __restrict__ ng, float scale, float* F, int Rp, int32_t* __restrict__ r_out,
    int32_t* __restrict__ cold, const int32_t* __restrict__ valid) {
    using S = WarmSmem<D>;
    extern __shared__ __align__(16) unsigned char wsm[];
    float* Ms = reinterpret_cast<float*>(wsm);
    float* Qs = reinterpret_cast<float*>(wsm + S::off_Q);
    double* Ys = reinterpret_cast<double*>(wsm + S::off_Y);
    double* Gs = reinterpret_cast<double*>(wsm + S::off_G);
    int* sflag = reinterpret_cast<int*>(wsm + S::off_misc);
    double* sdmax = reinterpret_cast<double*>(wsm + S::off_misc + 8);
    const int bh = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;

    if (valid != nullptr && *valid != kWarmMagic) {       // no previous state: cold factor
        if (tid == 0) cold[bh] = 1;
        return;
    }
    int r = r_req < D ? r_req : D;
    if (ng != nullptr) r = max(1, min(r, ng[bh * 2 + 1] - 1));
    r = min(r, min(Rp, kWarmRW));

    const float* Mh = Min + (size_t)bh * D * D;
    const float* Fp = Fprev + (size_t)bh * prev_stride * D * ld_prev;   // previous factor of head bh * prev_stride
    for (int e = tid; e < D * D; e += nt) {
        const int i = e / D, j = e % D;
        Ms[i * S::ldM + j] = 0.5f * (Mh[i * D + j] + Mh[j * D + i]);
    }
    for (int e = tid; e < D * kWarmRW; e += nt) {
        const int i = e / kWarmRW, c = e % kWarmRW;
        Qs[e] = (c < r && c < ld_prev) ? Fp[(size_t)i * ld_prev + c] : 0.f;
    }
    __syncthreads();

    bool ok = true;
    for (int it = 0; it < 2 && ok; ++it) {
        metric_times_basis<D>(Ms, Qs, Ys, r);
        __syncthreads();
        for (int e = tid; e < r * r; e += nt) {           // Y^T Y, lower triangle
            const int a = e / r, b = e % r;
            if (b > a) continue;
            double acc = 0.0;
            for (int i = 0; i < D; ++i) acc = fma(Ys[i * S::ldY + a], Ys[i * S::ldY + b], acc);
            Gs[a * S::ldY + b] = acc;
        }
        __syncthreads();
        ok = block_cholesky(Gs, S::ldY, r, sflag, sdmax);
        if (!ok) break;
        for (int i = tid; i < D; i += nt) {               // row i of Y L^-T, forward substitution
            double* y = Ys + i * S::ldY;
            for (int j = 0; j < r; ++j) {
                double s = y[j];
                const double* lj = Gs + j * S::ldY;
                for (int k = 0; k < j; ++k) s = fma(-lj[k], y[k], s);
                y[j] = s / lj[j];
            }
        }
        __syncthreads();
        for (int e = tid; e < D * r; e += nt) {
            const int i = e / r, c = e % r;
            Qs[i * kWarmRW + c] = (float)Ys[i * S::ldY + c];
        }
        __syncthreads();
    }
    if (ok) {
        metric_times_basis<D>(Ms, Qs, Ys, r);             // M Q
        __syncthreads();
        for (int e = tid; e < r * r; e += nt) {           // Q^T M Q, lower triangle
            const int a = e / r, b = e % r;
            if (b > a) continue;
            double acc = 0.0;
            for (int i = 0; i < D; ++i) acc = fma((double)Qs[i * kWarmRW + a], Ys[i * S::ldY + b], acc);
            Gs[a * S::ldY + b] = acc;
        }
        __syncthreads();
        ok = block_cholesky(Gs, S::ldY, r, sflag, sdmax);
    }
    if (!ok) {
        if (tid == 0) cold[bh] = 1;
        return;
    }
    float* Fh = F + (size_t)bh * D * Rp;
    for (int e = tid; e < D * Rp; e += nt) {
        const int i = e / Rp, c = e % Rp;
        float v = 0.f;
        if (c < r) {
            double acc = 0.0;
            for (int k = c; k < r; ++k) acc = fma((double)Qs[i * kWarmRW + k], Gs[k * S::ldY + c], acc);
            v = (float)(acc * (double)scale);
        }
        Fh[e] = v;
    }
    if (tid == 0) {
        cold[bh] = 0;
        if (r_out != nullptr) r_out[bh] = r;
    }
}

// One warp per centre c of head bh.
template <int R, bool RMS>
__global__ void __launch_bounds__(256) warm_init_kernel(
    const float* __restrict__ phi, int N, int C, uint64_t seed, int stage, const float* __restrict__ cbar,
    const int32_t* __restrict__ ng_prev, int which, int prev_stride, const float* __restrict__ F, int d,
    const int32_t* __restrict__ r_eff, float eps, const int32_t* __restrict__ valid, float* __restrict__ cen,
    float* __restrict__ hn) {
    constexpr int J = (R + 31) / 32;
    const int bh = blockIdx.y, lane = threadIdx.x & 31;
    const int c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (c >= C) return;
    int n_prev = 0;
    const int ph = bh * prev_stride;   // the previous call's head holding this head's state
    if (valid == nullptr || *valid == kWarmMagic) n_prev = min(max(ng_prev[ph * 2 + which], 0), C);
    float* dst = cen + ((size_t)bh * C + c) * R;
    float ss = 0.f;
    if (c < n_prev) {
        const float* cb = cbar + ((size_t)ph * C + c) * d;
        const float* Fh = F + (size_t)bh * d * R;
        float z[J];
#pragma unroll
        for (int u = 0; u < J; ++u) z[u] = 0.f;
        for (int t = 0; t < d; ++t) {
            const float x = cb[t];
#pragma unroll
            for (int u = 0; u < J; ++u)
                if (lane + 32 * u < R) z[u] = fmaf(x, Fh[(size_t)t * R + lane + 32 * u], z[u]);
        }
        if (RMS) {
            float s2 = 0.f;
#pragma unroll
            for (int u = 0; u < J; ++u) s2 = fmaf(z[u], z[u], s2);
            s2 = warp_sum(s2);
            const float den = fmaxf(sqrtf(s2 / (float)r_eff[bh]), eps);
#pragma unroll
            for (int u = 0; u < J; ++u) z[u] = z[u] / den;
        }
#pragma unroll
        for (int u = 0; u < J; ++u)
            if (lane + 32 * u < R) {
                const float v = tf32_round(z[u]);
                dst[lane + 32 * u] = v;
                ss = fmaf(v, v, ss);
            }
    } else {
        const int row = kmeans_init_row(seed, bh, stage, c, N);
        const float* src = phi + ((size_t)bh * N + row) * R;
        for (int t = lane; t < R; t += 32) {
            const float v = src[t];
            dst[t] = v;
            ss = fmaf(v, v, ss);
        }
    }
    ss = warp_sum(ss);
    if (lane == 0) hn[(size_t)bh * C + c] = 0.5f * ss;
}

template <int R>
void warm_init_r(const WarmInit& w, const float* phi, int BH, int N, int C, uint64_t seed, int stage, float* cen,
                 float* hn, cudaStream_t st) {
    const dim3 grid((C + 7) / 8, BH);
    if (w.rms)
        count_launch(), warm_init_kernel<R, true><<<grid, 256, 0, st>>>(phi, N, C, seed, stage, w.cbar, w.ng_prev,
                                                                        w.which, w.prev_stride, w.F, w.d, w.r_eff, w.eps, w.valid,
                                                                        cen, hn);
    else
        count_launch(), warm_init_kernel<R, false><<<grid, 256, 0, st>>>(phi, N, C, seed, stage, w.cbar, w.ng_prev,
                                                                         w.which, w.prev_stride, w.F, w.d, w.r_eff, w.eps, w.valid,
                                                                         cen, hn);
}

__global__ void set_word_kernel(int32_t* word, int32_t value) { *word = value; }

}  // namespace

void launch_set_word(int32_t* word, int32_t value, cudaStream_t st) {
    count_launch(), set_word_kernel<<<1, 1, 0, st>>>(word, value);
}

size_t warm_factor_smem(int d) { return d == 128 ? WarmSmem<128>::total : WarmSmem<64>::total; }

void launch_warm_factor(const float* M, const float* Fprev, int ld_prev, int prev_stride, int r_req, const int32_t* ng,
                        float scale, float* F, int Rp, int32_t* r_out, int32_t* cold, const int32_t* valid, int BH,
                        int d, cudaStream_t st) {
    const size_t smem = warm_factor_smem(d);
    if (d == 128) {
        cudaFuncSetAttribute(warm_factor_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        count_launch(), warm_factor_kernel<128><<<BH, kWarmThreads, smem, st>>>(M, Fprev, ld_prev, prev_stride, r_req, ng,
                                                                                scale, F, Rp, r_out, cold, valid);
    } else {
        cudaFuncSetAttribute(warm_factor_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        count_launch(), warm_factor_kernel<64><<<BH, kWarmThreads, smem, st>>>(M, Fprev, ld_prev, prev_stride, r_req, ng,
                                                                               scale, F, Rp, r_out, cold, valid);
    }
}

void launch_warm_init(const WarmInit& w, int R, const float* phi, int BH, int N, int C, uint64_t seed, int stage,
                      float* cen, float* hn, cudaStream_t st) {
    switch (R) {
        case 16: warm_init_r<16>(w, phi, BH, N, C, seed, stage, cen, hn, st); break;
        case 32: warm_init_r<32>(w, phi, BH, N, C, seed, stage, cen, hn, st); break;
        case 48: warm_init_r<48>(w, phi, BH, N, C, seed, stage, cen, hn, st); break;
        case 64: warm_init_r<64>(w, phi, BH, N, C, seed, stage, cen, hn, st); break;
        default: warm_init_r<128>(w, phi, BH, N, C, seed, stage, cen, hn, st); break;
    }
}

}  // namespace spr
