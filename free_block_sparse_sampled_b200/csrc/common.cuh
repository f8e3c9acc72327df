// Shared internals of the SparsePR CUDA library: workspace plan, device
// status word, element loads and small warp/block helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "sparsepr.h"

namespace spr {

constexpr int kMaxGroups = 2048;   // C_q, C_k upper limit (one sort of 2048 keys per block)
constexpr int kMaxRank = 64;       // r_K, r_Q upper limit (register-resident coordinates)
constexpr int kSortTile = 1024;    // points per histogram/scatter tile of the group sort
constexpr int kMaxN = (1 << 20) - 1;

// Device status word (first 256 bytes of the workspace).  The first failure
// wins; `where` records which kernel set it.
struct DevStatus {
    int32_t code;
    int32_t where;
    int32_t pad[62];
};

__device__ __forceinline__ void record_status(DevStatus* st, int code, int where) {
    if (atomicCAS(&st->code, 0, code) == 0) st->where = where;
}

// ------------------------------------------------------------------ loads
__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Eight consecutive elements starting at p (16-byte aligned for bf16, 32 for f32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    float4 a = *reinterpret_cast<const float4*>(p);
    float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// ------------------------------------------------------------------ warp helpers
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// Round to TF32 (10 explicit mantissa bits), nearest even.
__device__ __forceinline__ float tf32_round(float x) {
    uint32_t r;
    asm("cvt.rn.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

// Order-preserving map of a float to uint32 (ascending floats -> ascending keys).
__device__ __forceinline__ uint32_t float_order_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------------ SplitMix64
// Steele, Lea, Flood (OOPSLA 2014): the state advances by the golden gamma and
// each output is the state passed through the variant-13 finaliser.
__host__ __device__ __forceinline__ uint64_t sm64_finalise(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}
constexpr uint64_t kGoldenGamma = 0x9E3779B97F4A7C15ull;

// Row of initial centre c for head bh, stage 0 (K/V) or 1 (query).
__device__ __forceinline__ int kmeans_init_row(uint64_t seed, int bh, int stage, int c, int N) {
    uint64_t stream = sm64_finalise((uint64_t)(2 * bh + stage + 1) * kGoldenGamma);
    uint64_t base = sm64_finalise(seed ^ stream);
    uint64_t x = sm64_finalise(base + (uint64_t)(c + 1) * kGoldenGamma);
    return (int)(((x >> 32) * (uint64_t)N) >> 32);
}

// ------------------------------------------------------------------ workspace plan
struct Plan {
    // sizes
    int BH, N, d, Cq, Ck, Cmax, RKp, RQp, rK_eff, Mp, Ms_eff, n_sort_tiles, esz;
    int G;               // query heads per K/V head (GQA; 1 otherwise)
    int BM, n_items_max, n_probe_items;
    int64_t beta;        // key budget per query group
    int stop_changed;    // k-means stop threshold on changed labels
    // internal buffers (byte offsets into the workspace)
    size_t o_status, o_ctl, o_mat, o_FK, o_FQ, o_rq, o_phiK, o_phiQ, o_cenK, o_hnK, o_cenQ, o_hnQ, o_hs,
        o_raw, o_hist, o_sorted, o_offs, o_newid, o_muK, o_t1, o_t2, o_mloc, o_pslot, o_palloc,
        o_poff, o_psum, o_qprobe, o_work, o_fstat, o_G, o_rhs, o_vh, o_vmax, o_vscale, o_qsplit, o_uw, o_lbar, o_vv,
        o_warm,   // [0]: kWarmMagic when the fused call's state is complete; [1 + bh], [1 + BH + bh]: cold K / Q factor
        o_pbits,  // [BH][ceil(N/32)] probe membership bits (random / uniform probes)
        o_S,      // [BH][d][d] fp64 Rbar^T W Rbar (rank truncation)
        o_rawkv,  // [BH/G][N] K/V k-means labels per K/V head (GQA)
        o_csum,   // [BH][Cmax][Rmax] int64 member sums of the k-means centres (fixed point)
        o_ccnt,   // [BH][Cmax] member counts
        o_prev,   // [BH][N] the labels the sums hold
        o_cscale; // [BH] largest |coordinate| of each head (float bits): its fixed-point exponent
    // outputs owned by the workspace for sparsepr_call
    size_t o_Qp, o_Kp, o_Vp, o_qlab, o_kvlab, o_permq, o_permk, o_posq, o_qoff, o_kvoff, o_ng, o_its,
        o_qcen, o_kcen, o_vcen, o_qdist, o_score, o_mask, o_selc, o_selg, o_pairs, o_pidx, o_pgrp,
        o_pw, o_Osp, o_pdense, o_psparse, o_fB, o_fmux, o_fsig, o_fmur;
    size_t total;
};

// Word the fused call stores in the workspace once its partition state
// (factors, centroids, group counts) is complete; a warm start reads that
// state only when it finds the word.
constexpr int32_t kWarmMagic = 0x57524d31;

// ctl layout per head (int32): see kCtl* indices.
constexpr int kCtlStride = 16;
constexpr int kCtlChanged = 0, kCtlDone = 1, kCtlIters = 2, kCtlItersK = 3, kCtlItersQ = 4,
              kCtlWork = 8;

bool make_plan(const sparsepr_params& p, Plan& pl);

// Last CUDA error seen by this host thread (name and message), for
// sparsepr_last_error_string().
inline char* last_error_buffer() {
    static thread_local char buf[256] = "no error";
    return buf;
}
// Records err (if any) and maps it to a status.
inline sparsepr_status cuda_status(cudaError_t err) {
    if (err == cudaSuccess) return SPARSEPR_OK;
    snprintf(last_error_buffer(), 256, "%s: %s", cudaGetErrorName(err), cudaGetErrorString(err));
    return SPARSEPR_CUDA_ERROR;
}

// Kernels launched by this host thread since the counter was last reset.
inline long long& launch_counter() {
    static thread_local long long n = 0;
    return n;
}
inline void count_launch() { ++launch_counter(); }

// Streaming multiprocessors of the current device (cached per host thread).
inline int sm_count() {
    static thread_local int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    }
    return n;
}

template <typename T>
__host__ __device__ inline T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

}  // namespace spr

namespace spr {

// In-place exclusive scan of n <= 2*blockDim.x ints held in shared memory.
// Every thread of the block must call it; `scratch` holds 33 ints.  Returns
// the total.
__device__ __forceinline__ int block_exclusive_scan(int* s, int n, int* scratch) {
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
    const int a = (2 * tid < n) ? s[2 * tid] : 0;
    const int b = (2 * tid + 1 < n) ? s[2 * tid + 1] : 0;
    const int local = a + b;
    int inc = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    __syncthreads();
    if (lane == 31) scratch[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        int v = (lane < nw) ? scratch[lane] : 0;
        int iv = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, iv, o);
            if (lane >= o) iv += y;
        }
        if (lane < nw) scratch[lane] = iv - v;
        if (lane == nw - 1) scratch[32] = iv;
    }
    __syncthreads();
    const int excl = scratch[wid] + inc - local;
    if (2 * tid < n) s[2 * tid] = excl;
    if (2 * tid + 1 < n) s[2 * tid + 1] = excl + a;
    __syncthreads();
    return scratch[32];
}

// Ascending bitonic sort of n (a power of two) 64-bit keys in shared memory.
__device__ __forceinline__ void block_bitonic_sort(unsigned long long* k, int n) {
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int t = threadIdx.x; t < n / 2; t += blockDim.x) {
                const int i = 2 * stride * (t / stride) + (t % stride);
                const int j = i + stride;
                const bool up = (i & size) == 0;
                const unsigned long long x = k[i], y = k[j];
                if ((x > y) == up) {
                    k[i] = y;
                    k[j] = x;
                }
            }
        }
    }
    __syncthreads();
}

__host__ __device__ inline int round_up(int x, int m) { return (x + m - 1) / m * m; }
__host__ __device__ inline int next_pow2(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

}  // namespace spr
