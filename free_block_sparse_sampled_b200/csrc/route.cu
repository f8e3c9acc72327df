// Routing and probe selection ("Partition the Support, Reconstruct the
// Residual", §4.3, B.3, A.2, A.3).
//
//   s_ab = 1/|G_b| sum_{j in G_b} | e^{lbar_ab} vbar_b - e^{l_aj} v_j |^2,
//          lbar_ab = qbar_a kbar_b^T / sqrt(d),  l_aj = qbar_a k_j^T / sqrt(d),
//   evaluated as  e^{2 lbar}|vbar|^2 - 2 e^{lbar}/|G_b| sum_j e^{l_aj} (vbar.v_j)
//                 + 1/|G_b| sum_j e^{2 l_aj} |v_j|^2
//   with every exponent shifted by m_a = max(max_j l_aj, max_b lbar_ab).
//   Per query group: rank K/V groups by descending s (ties: lower index) and
//   keep the shortest prefix whose key count reaches the budget beta.
//   Probes: m_a by largest remainder on M|G_a|/N, the m_a rows of smallest
//   (d_i, i) inside each group, coverage weights w~_p = M w_p / sum w; or
//   (Table 4) M random rows or M rows evenly spaced over the grid, with the
//   coverage weights of the counts that fall in each group.
#include "common.cuh"
#include "internal.h"

namespace spr {

// Segment sums per (a, b): the running max M_ab of l_aj over j in G_b and
// t1 = sum e^{l-M}(vbar_b.v_j), t2 = sum e^{2(l-M)}|v_j|^2.  One block per
// (K/V group b, 8 query groups); one warp per query group.
template <typename T>
__global__ void __launch_bounds__(256) route_partial_kernel(
    const T* __restrict__ Kp, const T* __restrict__ Vp, const int32_t* __restrict__ kv_off,
    const int32_t* __restrict__ ng, const float* __restrict__ vbar, const float* __restrict__ qbar,
    int N, int Cq, int Ck, int d, int G, float* __restrict__ t1o, float* __restrict__ t2o,
    float* __restrict__ mloc) {
    constexpr int RB = 64;
    extern __shared__ float sm[];
    const int bh = blockIdx.z, b = blockIdx.x, a0 = blockIdx.y * 8;
    const int Cqp = ng[bh * 2 + 0], Ckp = ng[bh * 2 + 1];
    if (b >= Ckp || a0 >= Cqp) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ld = d + 1;
    float* qs = sm;                 // [8][d]
    float* ks = qs + 8 * d;         // [RB][d+1]
    float* us = ks + RB * ld;       // [RB]
    float* ws = us + RB;            // [RB]
    float* vb = ws + RB;            // [d]
    for (int e = threadIdx.x; e < 8 * d; e += blockDim.x) {
        const int r = e / d, t = e % d;
        qs[e] = (a0 + r < Cqp) ? qbar[((size_t)bh * Cq + a0 + r) * d + t] : 0.f;
    }
    for (int t = threadIdx.x; t < d; t += blockDim.x) vb[t] = vbar[((size_t)bh * Ck + b) * d + t];
    const int s = kv_off[(size_t)bh * (Ck + 1) + b], e = kv_off[(size_t)bh * (Ck + 1) + b + 1];
    const float inv_sqrt_d = 1.f / sqrtf((float)d);
    float M = -INFINITY, t1 = 0.f, t2 = 0.f;
    const float* qw = qs + warp * d;
    for (int r0 = s; r0 < e; r0 += RB) {
        const int n = min(RB, e - r0);
        __syncthreads();
        for (int rr = warp; rr < n; rr += 8) {
            const T* kr = Kp + ((size_t)(bh / G) * N + r0 + rr) * d;   // the K/V head under GQA
            const T* vr = Vp + ((size_t)(bh / G) * N + r0 + rr) * d;
            float uu = 0.f, ww = 0.f;
            for (int t = lane; t < d; t += 32) {
                ks[rr * ld + t] = ldf(kr + t);
                const float vv = ldf(vr + t);
                uu = fmaf(vb[t], vv, uu);
                ww = fmaf(vv, vv, ww);
            }
            uu = warp_sum(uu);
            ww = warp_sum(ww);
            if (lane == 0) {
                us[rr] = uu;
                ws[rr] = ww;
            }
        }
        __syncthreads();
        if (a0 + warp < Cqp) {
            for (int rr = lane; rr < n; rr += 32) {
                const float* kr = ks + rr * ld;
                float l = 0.f;
                for (int t = 0; t < d; ++t) l = fmaf(qw[t], kr[t], l);
                l *= inv_sqrt_d;
                if (l > M) {
                    const float sc = expf(M - l);
                    t1 *= sc;
                    t2 *= sc * sc;
                    M = l;
                }
                const float ex = expf(l - M);
                t1 = fmaf(ex, us[rr], t1);
                t2 = fmaf(ex * ex, ws[rr], t2);
            }
        }
    }
    // combine lanes (commutative combine -> every lane ends with the same value)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float M2 = __shfl_xor_sync(0xffffffffu, M, o);
        const float u2 = __shfl_xor_sync(0xffffffffu, t1, o);
        const float w2 = __shfl_xor_sync(0xffffffffu, t2, o);
        const float Mn = fmaxf(M, M2);
        const float fa = (M == -INFINITY) ? 0.f : expf(M - Mn);
        const float fb = (M2 == -INFINITY) ? 0.f : expf(M2 - Mn);
        t1 = t1 * fa + u2 * fb;
        t2 = t2 * (fa * fa) + w2 * (fb * fb);
        M = Mn;
    }
    const int a = a0 + warp;
    if (lane == 0 && a < Cqp) {
        const size_t idx = ((size_t)bh * Cq + a) * Ck + b;
        mloc[idx] = M;
        t1o[idx] = t1;
        t2o[idx] = t2;
    }
}

// lbar[a][b] = qbar_a kbar_b^T / sqrt(d) for every pair of nonempty groups (32x32 tiles).
__global__ void __launch_bounds__(256) centroid_logits_kernel(const float* __restrict__ qbar,
                                                              const float* __restrict__ kbar,
                                                              const int32_t* __restrict__ ng, int Cq, int Ck, int d,
                                                              float* __restrict__ lbar) {
    const int bh = blockIdx.z, a0 = blockIdx.y * 32, b0 = blockIdx.x * 32;
    const int Cqp = ng[bh * 2 + 0], Ckp = ng[bh * 2 + 1];
    if (a0 >= Cqp || b0 >= Ckp) return;
    const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
    __shared__ float sa[32][33], sb[32][33];
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int t0 = 0; t0 < d; t0 += 32) {
        for (int r = ty; r < 32; r += 8) {
            sa[r][tx] = (a0 + r < Cqp) ? qbar[((size_t)bh * Cq + a0 + r) * d + t0 + tx] : 0.f;
            sb[r][tx] = (b0 + r < Ckp) ? kbar[((size_t)bh * Ck + b0 + r) * d + t0 + tx] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int t = 0; t < 32; ++t) {
            const float bv = sb[tx][t];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] = fmaf(sa[ty + 8 * u][t], bv, acc[u]);
        }
        __syncthreads();
    }
    const float inv = 1.f / sqrtf((float)d);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int a = a0 + ty + 8 * u, b = b0 + tx;
        if (a < Cqp && b < Ckp) lbar[((size_t)bh * Cq + a) * Ck + b] = acc[u] * inv;
    }
}

// |vbar_b|^2, one warp per K/V group.
__global__ void centroid_sqnorm_kernel(const float* __restrict__ vbar, const int32_t* __restrict__ ng, int Ck, int d,
                                       float* __restrict__ vv) {
    const int bh = blockIdx.y, lane = threadIdx.x & 31;
    const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (b >= ng[bh * 2 + 1]) return;
    const float* v = vbar + ((size_t)bh * Ck + b) * d;
    float acc = 0.f;
    for (int t = lane; t < d; t += 32) acc = fmaf(v[t], v[t], acc);
    acc = warp_sum(acc);
    if (lane == 0) vv[(size_t)bh * Ck + b] = acc;
}

// Scores, ranking and the prefix rule for one query group per block.
__global__ void __launch_bounds__(1024) route_select_kernel(
    const float* __restrict__ lbar_in, const float* __restrict__ vv_in,
    const float* __restrict__ t1o, const float* __restrict__ t2o, const float* __restrict__ mloc,
    const int32_t* __restrict__ q_off, const int32_t* __restrict__ kv_off,
    const int32_t* __restrict__ ng, int Cq, int Ck, int d, long long beta,
    float* __restrict__ score, uint8_t* __restrict__ mask, int32_t* __restrict__ sel_count,
    int32_t* __restrict__ sel_groups, unsigned long long* __restrict__ pairs) {
    __shared__ unsigned long long keys[kMaxGroups];
    __shared__ float lb[kMaxGroups];
    __shared__ int sz[kMaxGroups];
    __shared__ float red[32];
    __shared__ int scratch[33];
    __shared__ int cut;
    const int a = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int Cqp = ng[bh * 2 + 0], Ckp = ng[bh * 2 + 1];
    if (a >= Cqp) return;
    if (tid == 0) cut = Ckp - 1;
    __syncthreads();
    const size_t row = ((size_t)bh * Cq + a) * Ck;
    float mx = -INFINITY;
    for (int b = tid; b < Ckp; b += blockDim.x) {
        const float l = lbar_in[row + b];
        lb[b] = l;
        mx = fmaxf(mx, fmaxf(l, mloc[row + b]));
    }
    mx = warp_max(mx);
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    if (tid < 32) {
        float v = (tid < (int)(blockDim.x >> 5)) ? red[tid] : -INFINITY;
        v = warp_max(v);
        if (tid == 0) red[0] = v;
    }
    __syncthreads();
    const float m_a = red[0];
    const int32_t* ko = kv_off + (size_t)bh * (Ck + 1);
    for (int b = tid; b < Ckp; b += blockDim.x) {
        const float vv = vv_in[(size_t)bh * Ck + b];
        const int nb = ko[b + 1] - ko[b];
        const float inv_nb = 1.f / (float)nb;
        const float ea = expf(lb[b] - m_a);
        const float em = expf(mloc[row + b] - m_a);
        float s = ea * ea * vv - 2.f * ea * em * t1o[row + b] * inv_nb + em * em * t2o[row + b] * inv_nb;
        s = s + 0.f;   // -0 -> +0 so equal scores rank by index
        score[row + b] = s;
        keys[b] = ((unsigned long long)(~float_order_key(s)) << 32) | (unsigned)b;
    }
    const int P = next_pow2(max(Ckp, 2));
    for (int b = Ckp + tid; b < P; b += blockDim.x) keys[b] = ~0ull;
    block_bitonic_sort(keys, P);
    for (int k = tid; k < Ckp; k += blockDim.x) {
        const int b = (int)(keys[k] & 0xffffffffu);
        sz[k] = ko[b + 1] - ko[b];
    }
    __syncthreads();
    block_exclusive_scan(sz, Ckp, scratch);
    for (int k = tid; k < Ckp; k += blockDim.x) {
        const int b = (int)(keys[k] & 0xffffffffu);
        const long long incl = (long long)sz[k] + (ko[b + 1] - ko[b]);
        if (incl >= beta) atomicMin(&cut, k);
    }
    __syncthreads();
    const int n_sel = cut + 1;
    // selection flags by group index (reuse sz as flags)
    __syncthreads();
    const int kc = (int)(keys[cut] & 0xffffffffu);
    const long long keys_sel = (long long)sz[cut] + (ko[kc + 1] - ko[kc]);
    __syncthreads();
    for (int b = tid; b < Ckp; b += blockDim.x) sz[b] = 0;
    __syncthreads();
    for (int k = tid; k < n_sel; k += blockDim.x) sz[keys[k] & 0xffffffffu] = 1;
    __syncthreads();
    for (int b = tid; b < Ck; b += blockDim.x) mask[row + b] = (b < Ckp) ? (uint8_t)sz[b] : (uint8_t)0;
    __syncthreads();
    block_exclusive_scan(sz, Ckp, scratch);
    for (int b = tid; b < Ckp; b += blockDim.x) {
        const bool sel = (b + 1 < Ckp) ? (sz[b + 1] != sz[b]) : (sz[b] != n_sel);
        if (sel) sel_groups[row + sz[b]] = b;
    }
    if (tid == 0) {
        sel_count[(size_t)bh * Cq + a] = n_sel;
        const long long qa = q_off[(size_t)bh * (Cq + 1) + a + 1] - q_off[(size_t)bh * (Cq + 1) + a];
        atomicAdd(&pairs[bh * 2 + 0], (unsigned long long)(qa * keys_sel));
    }
}

// m_a by largest remainder on M|G_a|/N (remainder ties: larger |G_a|, then
// lower a); probe offsets; sum of coverage weights; P_exec.
__global__ void __launch_bounds__(1024) probe_alloc_kernel(const int32_t* __restrict__ q_off,
                                                           const int32_t* __restrict__ ng, int Cq,
                                                           int N, int Mp, int32_t* __restrict__ alloc,
                                                           int32_t* __restrict__ poff,
                                                           int32_t* __restrict__ psum,
                                                           unsigned long long* __restrict__ pairs) {
    __shared__ unsigned long long keys[kMaxGroups];
    __shared__ int base[kMaxGroups];
    __shared__ int mm[kMaxGroups];
    __shared__ int scratch[33];
    __shared__ int sum_base, sum_w;
    const int bh = blockIdx.x, tid = threadIdx.x;
    const int Cqp = ng[bh * 2 + 0];
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    if (tid == 0) {
        sum_base = 0;
        sum_w = 0;
    }
    __syncthreads();
    for (int a = tid; a < Cqp; a += blockDim.x) {
        const int size = qo[a + 1] - qo[a];
        const long long num = (long long)Mp * size;
        const int bs = (int)(num / N);
        const int rem = (int)(num % N);
        base[a] = bs;
        atomicAdd(&sum_base, bs);
        keys[a] = ((unsigned long long)(N - rem) << 40) | ((unsigned long long)(N - size) << 20) |
                  (unsigned long long)a;
    }
    const int P = next_pow2(max(Cqp, 2));
    for (int a = Cqp + tid; a < P; a += blockDim.x) keys[a] = ~0ull;
    block_bitonic_sort(keys, P);
    const int extra = Mp - sum_base;
    for (int k = tid; k < Cqp; k += blockDim.x) {
        const int a = (int)(keys[k] & 0xfffffu);
        const int size = qo[a + 1] - qo[a];
        mm[a] = (Mp >= N) ? size : base[a] + (k < extra ? 1 : 0);
    }
    __syncthreads();
    for (int a = tid; a < Cqp; a += blockDim.x) {
        alloc[(size_t)bh * Cq + a] = mm[a];
        if (mm[a] > 0) atomicAdd(&sum_w, qo[a + 1] - qo[a]);
    }
    __syncthreads();
    block_exclusive_scan(mm, Cqp, scratch);
    for (int a = tid; a < Cqp; a += blockDim.x) poff[(size_t)bh * Cq + a] = mm[a];
    if (tid == 0) {
        psum[bh] = sum_w;
        pairs[bh * 2 + 1] = pairs[bh * 2 + 0] + (unsigned long long)Mp * (unsigned long long)N;
    }
}

// Inside group a: the m_a members with the smallest (d_i, i), in that order.
__global__ void __launch_bounds__(256) probe_select_kernel(
    const int32_t* __restrict__ q_off, const int32_t* __restrict__ perm_q,
    const float* __restrict__ qdist,
    const int32_t* __restrict__ ng, const int32_t* __restrict__ alloc,
    const int32_t* __restrict__ poff, const int32_t* __restrict__ psum, int Cq, int N, int Mp,
    int32_t* __restrict__ probe_idx, int32_t* __restrict__ probe_group,
    float* __restrict__ probe_weight) {
    __shared__ float rd[8];
    __shared__ int ri[8];
    const int a = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    if (a >= ng[bh * 2 + 0]) return;
    const int m = alloc[(size_t)bh * Cq + a];
    if (m == 0) return;
    const int s = q_off[(size_t)bh * (Cq + 1) + a], e = q_off[(size_t)bh * (Cq + 1) + a + 1];
    const int size = e - s;
    const double wt = (double)Mp * ((double)size / (double)m) / (double)psum[bh];
    float last_d = -INFINITY;
    int last_i = -1;
    for (int k = 0; k < m; ++k) {
        float bd = INFINITY;
        int bi = 0x7fffffff;
        for (int p = s + tid; p < e; p += blockDim.x) {
            const int i = perm_q[(size_t)bh * N + p];
            const float dd = qdist[(size_t)bh * N + i];
            const bool after = (dd > last_d) || (dd == last_d && i > last_i);
            const bool better = (dd < bd) || (dd == bd && i < bi);
            if (after && better) {
                bd = dd;
                bi = i;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float d2 = __shfl_xor_sync(0xffffffffu, bd, o);
            const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
            if ((d2 < bd) || (d2 == bd && i2 < bi)) {
                bd = d2;
                bi = i2;
            }
        }
        if ((tid & 31) == 0) {
            rd[tid >> 5] = bd;
            ri[tid >> 5] = bi;
        }
        __syncthreads();
        bd = rd[0];
        bi = ri[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            if ((rd[w] < bd) || (rd[w] == bd && ri[w] < bi)) {
                bd = rd[w];
                bi = ri[w];
            }
        __syncthreads();
        if (tid == 0) {
            const int slot = poff[(size_t)bh * Cq + a] + k;
            probe_idx[(size_t)bh * Mp + slot] = bi;
            probe_group[(size_t)bh * Mp + slot] = a;
            probe_weight[(size_t)bh * Mp + slot] = (float)wt;
        }
        last_d = bd;
        last_i = bi;
    }
}

// Random (Floyd's algorithm) or uniform-grid probe rows, then m_a, the sum of
// coverage weights and the probe list by group, then by index.  One block of
// 1024 threads per head; `bits` is this head's membership bitmap.
constexpr uint64_t kProbeStream = 0x50524F4245ull;
__global__ void __launch_bounds__(1024) probe_fixed_kernel(
    int mode, uint64_t seed, const int32_t* __restrict__ q_off, const int32_t* __restrict__ perm_q,
    const int32_t* __restrict__ q_label, const int32_t* __restrict__ ng, int Cq, int N, int Mp,
    uint32_t* __restrict__ bits_all, int32_t* __restrict__ alloc, int32_t* __restrict__ psum,
    unsigned long long* __restrict__ pairs, int32_t* __restrict__ probe_idx, int32_t* __restrict__ probe_group,
    float* __restrict__ probe_weight) {
    __shared__ int hist[kMaxGroups];
    __shared__ int warp_tot[32];
    __shared__ int sum_w, run;
    const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int nwords = (N + 31) / 32;
    uint32_t* bits = bits_all + (size_t)bh * nwords;
    const int Cqp = ng[bh * 2 + 0];
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    const int32_t* lab = q_label + (size_t)bh * N;
    for (int e = tid; e < nwords; e += blockDim.x) bits[e] = 0u;
    for (int a = tid; a < Cqp; a += blockDim.x) hist[a] = 0;
    if (tid == 0) {
        sum_w = 0;
        run = 0;
    }
    __syncthreads();
    if (mode == SPARSEPR_PROBES_RANDOM) {
        if (tid == 0) {
            const uint64_t base = sm64_finalise(seed ^ sm64_finalise(((uint64_t)(bh + 1) * kGoldenGamma) ^ kProbeStream));
            for (int s = 0; s < Mp; ++s) {
                const int j = N - Mp + s;
                const uint64_t x = sm64_finalise(base + (uint64_t)(s + 1) * kGoldenGamma);
                const int t = (int)(((x >> 32) * (uint64_t)(j + 1)) >> 32);
                const int pick = ((bits[t >> 5] >> (t & 31)) & 1u) ? j : t;
                bits[pick >> 5] |= 1u << (pick & 31);
            }
        }
    } else {
        for (int j = tid; j < Mp; j += blockDim.x) {
            const int r = (int)(((2LL * j + 1) * (long long)N) / (2LL * Mp));
            atomicOr(&bits[r >> 5], 1u << (r & 31));
        }
    }
    __syncthreads();
    for (int i = tid; i < N; i += blockDim.x)
        if ((bits[i >> 5] >> (i & 31)) & 1u) atomicAdd(&hist[lab[i]], 1);
    __syncthreads();
    for (int a = tid; a < Cqp; a += blockDim.x) {
        alloc[(size_t)bh * Cq + a] = hist[a];
        if (hist[a] > 0) atomicAdd(&sum_w, qo[a + 1] - qo[a]);
    }
    __syncthreads();
    if (tid == 0) {
        psum[bh] = sum_w;
        pairs[bh * 2 + 1] = pairs[bh * 2 + 0] + (unsigned long long)Mp * (unsigned long long)N;
    }
    // list in permuted order (group-major, stable by index): block-wide compaction
    const int32_t* pq = perm_q + (size_t)bh * N;
    for (int r0 = 0; r0 < N; r0 += blockDim.x) {
        const int r = r0 + tid;
        int i = 0;
        bool f = false;
        if (r < N) {
            i = pq[r];
            f = (bits[i >> 5] >> (i & 31)) & 1u;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        if (lane == 0) warp_tot[wid] = __popc(bal);
        __syncthreads();
        int before = run;
        for (int w2 = 0; w2 < wid; ++w2) before += warp_tot[w2];
        if (f) {
            const int slot = before + __popc(bal & ((1u << lane) - 1u));
            const int a = lab[i];
            probe_idx[(size_t)bh * Mp + slot] = i;
            probe_group[(size_t)bh * Mp + slot] = a;
            probe_weight[(size_t)bh * Mp + slot] =
                (float)((double)Mp * ((double)(qo[a + 1] - qo[a]) / (double)hist[a]) / (double)sum_w);
        }
        __syncthreads();
        if (tid == 0) {
            int t = 0;
            for (int w2 = 0; w2 < (int)(blockDim.x >> 5); ++w2) t += warp_tot[w2];
            run += t;
        }
        __syncthreads();
    }
}

// ================================================================ host side
namespace {

template <typename T>
void route_partial(const Plan& pl, const sparsepr_partition_out& part, float* t1, float* t2,
                   float* ml, cudaStream_t st) {
    const int d = pl.d;
    const size_t smem = (size_t)(8 * d + 64 * (d + 1) + 2 * 64 + d) * sizeof(float);
    cudaFuncSetAttribute(route_partial_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    count_launch(), route_partial_kernel<T><<<dim3(pl.Ck, (pl.Cq + 7) / 8, pl.BH), 256, smem, st>>>(
        static_cast<const T*>(part.Kp), static_cast<const T*>(part.Vp), part.kv_offsets,
        part.n_groups, part.v_centroid, part.q_centroid, pl.N, pl.Cq, pl.Ck, d, pl.G, t1, t2, ml);
}

}  // namespace

sparsepr_status run_route(const sparsepr_params& p, const Plan& pl, const sparsepr_partition_out& part,
                          const sparsepr_route_out& r, void* ws, cudaStream_t st) {
    float* t1 = at<float>(ws, pl.o_t1);
    float* t2 = at<float>(ws, pl.o_t2);
    float* ml = at<float>(ws, pl.o_mloc);
    int32_t* alloc = r.probe_alloc;
    int32_t* poff = at<int32_t>(ws, pl.o_poff);
    int32_t* psum = at<int32_t>(ws, pl.o_psum);
    const int BH = pl.BH;
    cudaMemsetAsync(r.pairs, 0, (size_t)BH * 2 * sizeof(int64_t), st);
    cudaMemsetAsync(r.sel_count, 0, (size_t)BH * pl.Cq * sizeof(int32_t), st);
    if (route_uses_tc(p)) {
        if (!launch_route_tc(pl, part, ws, t1, t2, ml, st)) return SPARSEPR_CUDA_ERROR;
    } else {
        route_partial<float>(pl, part, t1, t2, ml, st);
    }
    float* lbar = at<float>(ws, pl.o_lbar);
    float* vv = at<float>(ws, pl.o_vv);
    count_launch(), centroid_logits_kernel<<<dim3((pl.Ck + 31) / 32, (pl.Cq + 31) / 32, BH), dim3(32, 8), 0, st>>>(
        part.q_centroid, part.k_centroid, part.n_groups, pl.Cq, pl.Ck, pl.d, lbar);
    count_launch(), centroid_sqnorm_kernel<<<dim3((pl.Ck + 7) / 8, BH), 256, 0, st>>>(part.v_centroid, part.n_groups,
                                                                                      pl.Ck, pl.d, vv);
    count_launch(), route_select_kernel<<<dim3(pl.Cq, BH), 1024, 0, st>>>(
        lbar, vv, t1, t2, ml, part.q_offsets,
        part.kv_offsets, part.n_groups, pl.Cq, pl.Ck, pl.d, (long long)pl.beta, r.score, r.mask,
        r.sel_count, r.sel_groups, reinterpret_cast<unsigned long long*>(r.pairs));
    if (p.probe_select != SPARSEPR_PROBES_STRATIFIED && pl.Mp > 0 && pl.Mp < pl.N) {
        count_launch(), probe_fixed_kernel<<<BH, 1024, 0, st>>>(
            p.probe_select, p.seed, part.q_offsets, part.perm_q, part.q_label, part.n_groups, pl.Cq, pl.N, pl.Mp,
            at<uint32_t>(ws, pl.o_pbits), alloc, psum, reinterpret_cast<unsigned long long*>(r.pairs), r.probe_idx,
            r.probe_group, r.probe_weight);
        return cuda_status(cudaGetLastError());
    }
    count_launch(), probe_alloc_kernel<<<BH, 1024, 0, st>>>(part.q_offsets, part.n_groups, pl.Cq, pl.N, pl.Mp, alloc, poff, psum,
                                            reinterpret_cast<unsigned long long*>(r.pairs));
    if (pl.Mp > 0)
        count_launch(), probe_select_kernel<<<dim3(pl.Cq, BH), 256, 0, st>>>(
            part.q_offsets, part.perm_q, part.q_dist, part.n_groups, alloc, poff, psum,
            pl.Cq, pl.N, pl.Mp, r.probe_idx, r.probe_group, r.probe_weight);
    return cuda_status(cudaGetLastError());
}

}  // namespace spr
