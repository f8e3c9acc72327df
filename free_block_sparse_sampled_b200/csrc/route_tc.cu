// Routing-score segment sums on the tensor cores ("Partition the Support,
// Reconstruct the Residual", B.3).
//
// For query group a and key j of K/V group b:
//   l_aj = qbar_a k_j^T / sqrt(d),
//   t1_ab = sum_{j in G_b} e^{l_aj - M_ab} (vbar_b . v_j),   t2_ab = sum e^{2(l_aj - M_ab)} |v_j|^2,
// with a reference M_ab >= every l_aj of the group (the running maximum over
// the key tiles seen so far).  The logits are one GEMM of the query-group
// centroids (128 per block, TMEM lanes) against 128-key tiles of the
// group-major keys; qbar is split into three bf16 pieces (hi + mid + lo) so
// the three exact bf16 products reproduce an fp32 logit.  A block covers a
// run of whole K/V groups, so every (a, b) partial is finished in one block.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace spr {
namespace rtc {
constexpr int BA = 128;        // query groups per block
constexpr int BK = 128;        // keys per tile
constexpr int GPB = 64;        // K/V groups per block
constexpr int RING = 4;
constexpr uint32_t kSpin = 1u << 20;
enum { B_A = 0, B_BF = 1, B_BE = 3, B_DF = 5, B_DE = 7, B_MF = 9, B_ME = B_MF + RING, B_DR = B_ME + RING,
       N_BAR = B_DR + 1 };

template <int D>
struct Layout {
    static constexpr int AB = BA * D * 2;           // one bf16 piece of the centroids
    static constexpr int KB = BK * D * 2;           // one key stage
    static constexpr int oA = 0;                    // 3 pieces
    static constexpr int oK = oA + 3 * AB;          // 2 stages
    static constexpr int oMeta = oK + 2 * KB;       // RING x {u[128], w[128], end mask[4]}
    static constexpr int META = (2 * BK + 4) * 4;
    static constexpr int oBar = oMeta + RING * META;
    static constexpr int oMisc = oBar + N_BAR * 8;
    static constexpr int smem = oMisc + 64 + 1024;
};

struct Maps {
    CUtensorMap a;     // [BH * 3 * CqPad, D] bf16 pieces, box 64 x 128
    CUtensorMap k;     // [BH * N, D] bf16 keys, box 64 x 128
};
}  // namespace rtc

// qbar split: piece 0 = bf16(q), 1 = bf16(q - p0), 2 = bf16(q - p0 - p1); rows >= C_q' are zero.
__global__ void route_qsplit_kernel(const float* __restrict__ qbar, const int32_t* __restrict__ ng, int Cq, int CqPad,
                                    int d, __nv_bfloat16* __restrict__ out) {
    const int bh = blockIdx.y;
    const int Cqp = ng[bh * 2 + 0];
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < CqPad * d; e += gridDim.x * blockDim.x) {
        const int a = e / d, t = e % d;
        const float q = (a < Cqp) ? qbar[((size_t)bh * Cq + a) * d + t] : 0.f;
        const __nv_bfloat16 p0 = __float2bfloat16_rn(q);
        const float r1 = q - __bfloat162float(p0);
        const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
        __nv_bfloat16* o = out + (size_t)bh * 3 * CqPad * d + (size_t)a * d + t;
        o[0] = p0;
        o[(size_t)CqPad * d] = p1;
        o[(size_t)2 * CqPad * d] = p2;
    }
}

// u_j = vbar_b . v_j and w_j = |v_j|^2 for every permuted key row j (b its
// group), once per K/V head: under GQA the G query heads of a K/V head share
// its groups, centroids and rows, so head kh reads query head kh * G's.
template <typename T>
__global__ void route_uw_kernel(const T* __restrict__ Vp, const float* __restrict__ vbar,
                                const int32_t* __restrict__ kv_label, const int32_t* __restrict__ perm_kv, int BHk,
                                int N, int Ck, int d, int G, float2* __restrict__ uw) {
    const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
    const int lane = threadIdx.x & 31;
    for (size_t row = blockIdx.x * (size_t)(blockDim.x >> 5) + (threadIdx.x >> 5); row < (size_t)BHk * N; row += warps) {
        const size_t kh = row / N, qh = kh * G, r = row - kh * N;
        const int b = kv_label[qh * N + perm_kv[qh * N + r]];
        const T* v = Vp + row * d;
        const float* vb = vbar + (qh * Ck + b) * d;
        float u = 0.f, w = 0.f;
        for (int t = lane; t < d; t += 32) {
            const float x = ldf(v + t);
            u = fmaf(vb[t], x, u);
            w = fmaf(x, x, w);
        }
        u = warp_sum(u);
        w = warp_sum(w);
        if (lane == 0) uw[row] = make_float2(u, w);
    }
}

template <int D>
__global__ void __launch_bounds__(192, 1) route_tc_kernel(
    const __grid_constant__ rtc::Maps maps, const float2* __restrict__ uw, const int32_t* __restrict__ kv_off,
    const int32_t* __restrict__ ng, int N, int Cq, int Ck, int CqPad, int G, float* __restrict__ t1o,
    float* __restrict__ t2o, float* __restrict__ mloc, DevStatus* status) {
    using namespace rtc;
    using namespace sm100;
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int bh = blockIdx.z, at = blockIdx.y, g0 = blockIdx.x * GPB;
    const int Cqp = ng[bh * 2 + 0], Ckp = ng[bh * 2 + 1];
    if (g0 >= Ckp || at * BA >= Cqp) return;
    if (*reinterpret_cast<volatile const int32_t*>(&status->code) != 0) return;
    const int g1 = min(g0 + GPB, Ckp);
    const int32_t* ko = kv_off + (size_t)bh * (Ck + 1);
    const int j_begin = ko[g0], j_end = ko[g1];
    const int n_tiles = (j_end - j_begin + BK - 1) / BK;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t s_base = smem_u32(sm);
    auto bar = [&](int i) -> uint32_t { return s_base + L::oBar + 8 * i; };
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::oMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    if (tid == 0) {
        mbar_init(bar(B_A), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_BF + s), 1);
            mbar_init(bar(B_BE + s), 1);
            mbar_init(bar(B_DF + s), 1);
            mbar_init(bar(B_DE + s), 128);
        }
        for (int s = 0; s < RING; ++s) {
            mbar_init(bar(B_MF + s), 1);
            mbar_init(bar(B_ME + s), 128);
        }
        mbar_init(bar(B_DR), 1);
        fence_barrier_init();
        misc[1] = 0;
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(misc), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == 4) {
        // ------------------------------------------------ producer: centroid pieces, key tiles, per-tile metadata
        if (lane == 0) {
            prefetch_tmap(&maps.a);
            prefetch_tmap(&maps.k);
            mbar_arrive_expect_tx(bar(B_A), 3 * L::AB);
            for (int pc = 0; pc < 3; ++pc)
                for (int hh = 0; hh < D / 64; ++hh)
                    tma_load_2d(s_base + L::oA + pc * L::AB + hh * BA * 128, &maps.a, bar(B_A), hh * 64,
                                (bh * 3 + pc) * CqPad + at * BA);
        }
        // the block's key-group ends, two per lane (GPB = 64), read once
        static_assert(GPB == 64, "two group ends per lane");
        const int ge0 = (g0 + lane < g1) ? ko[g0 + lane + 1] : -1;
        const int ge1 = (g0 + lane + 32 < g1) ? ko[g0 + lane + 33] : -1;
        int issued = 0;
        for (int t = 0; t < n_tiles; ++t) {
            const int stage = t & 1, ring = t % RING, j0 = j_begin + t * BK;
            int ok = 1;
            if (lane == 0) {
                if (t >= RING && !mbar_wait(bar(B_ME + ring), ((t / RING) - 1) & 1, abort_flag, kSpin)) ok = 0;
                if (ok && t >= 2 && !mbar_wait(bar(B_BE + stage), ((t >> 1) - 1) & 1, abort_flag, kSpin)) ok = 0;
                if (!ok) {
                    record_status(status, SPARSEPR_TIMEOUT, 30);
                    *abort_flag = 1;
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            float* meta = reinterpret_cast<float*>(sm + L::oMeta + ring * L::META);
            uint32_t* endm = reinterpret_cast<uint32_t*>(meta + 2 * BK);
            if (lane < 4) endm[lane] = 0u;
            __syncwarp();
            for (int c = lane; c < BK; c += 32) {
                const int j = j0 + c;
                const float2 v = (j < j_end) ? uw[(size_t)(bh / G) * N + j] : make_float2(0.f, 0.f);
                meta[c] = v.x;
                meta[BK + c] = v.y;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {   // key-group ends that fall in this tile
                const int e = h ? ge1 : ge0;
                if (e > j0 && e <= j0 + BK) atomicOr(&endm[(e - 1 - j0) >> 5], 1u << ((e - 1 - j0) & 31));
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(B_MF + ring));
                mbar_arrive_expect_tx(bar(B_BF + stage), L::KB);
                for (int hh = 0; hh < D / 64; ++hh)
                    tma_load_2d(s_base + L::oK + stage * L::KB + hh * BK * 128, &maps.k, bar(B_BF + stage), hh * 64,
                                (bh / G) * N + j0);
            }
            issued = t + 1;
        }
        if (lane == 0) {
            mbar_wait(bar(B_A), 0, nullptr, kSpin);
            for (int t = max(0, issued - 2); t < issued; ++t) mbar_wait(bar(B_BF + (t & 1)), (t >> 1) & 1, nullptr, kSpin);
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA: D[stage] = sum over pieces of A_piece K^T
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f32acc(BA, BK, kFmtBF16, false);
            // descriptors built once; each MMA adds a compile-time offset (>> 4) to
            // the start-address field, which never carries out (shared < 2^18)
            const uint64_t dA = smem_desc(s_base + L::oA, 16, 1024), dK = smem_desc(s_base + L::oK, 16, 1024);
            bool ok = mbar_wait(bar(B_A), 0, abort_flag, kSpin);
            for (int t = 0; ok && t < n_tiles; ++t) {
                const int stage = t & 1;
                if (!mbar_wait(bar(B_BF + stage), (t >> 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                if (t >= 2 && !mbar_wait(bar(B_DE + stage), ((t >> 1) - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                tc_fence_after();
                const uint64_t b0 = dK + (uint64_t)((stage * L::KB) >> 4);
#pragma unroll
                for (int pc = 0; pc < 3; ++pc)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t oa = (uint64_t)((pc * L::AB + (kk / 4) * BA * 128 + (kk % 4) * 32) >> 4);
                        const uint64_t ob = (uint64_t)(((kk / 4) * BK * 128 + (kk % 4) * 32) >> 4);
                        mma_f16_ss(tmem + stage * BK, dA + oa, b0 + ob, idesc, (pc | kk) ? 1u : 0u);
                    }
                mma_commit(bar(B_DF + stage));
                mma_commit(bar(B_BE + stage));
            }
            if (!ok) {
                record_status(status, SPARSEPR_TIMEOUT, 31);
                *abort_flag = 1;
            }
            mma_commit(bar(B_DR));
            mbar_wait(bar(B_DR), 0, nullptr, kSpin);
        }
    } else {
        // ------------------------------------------------ epilogue: one query group per thread
        const int r = tid, a = at * BA + r;
        const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);
        const float cs = 1.4426950408889634f / sqrtf((float)D);   // logits in log2 units
        float Mr = -INFINITY, t1 = 0.f, t2 = 0.f;                 // open group: reference and sums
        int b = g0;
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            const int stage = t & 1, ring = t % RING, j0 = j_begin + t * BK;
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DF + stage), (t >> 1) & 1, abort_flag, kSpin));
            if (!ok) break;
            tc_fence_after();
            const int ncol = min(BK, j_end - j0);
            // pass 1: the tile's maximum logit (log2 units) moves the open group's reference
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c4 = 0; c4 < BK / 32; ++c4) {
                float v[32];
                tmem_ld32(t_row + stage * BK + c4 * 32, v);
                tmem_wait_ld(v);
                const int nv = ncol - c4 * 32;   // valid columns of the chunk (uniform)
#pragma unroll
                for (int i = 0; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], i < nv ? v[i] * cs : -INFINITY);
            }
            const float Mn = fmaxf(Mr, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
            if (Mn > Mr) {
                const float f = (Mr == -INFINITY) ? 0.f : ex2_approx(Mr - Mn);
                t1 *= f;
                t2 *= f * f;
                Mr = Mn;
            }
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_MF + ring), (t / RING) & 1, abort_flag, kSpin));
            if (!ok) break;
            const float* meta = reinterpret_cast<const float*>(sm + L::oMeta + ring * L::META);
            const uint32_t* endm = reinterpret_cast<const uint32_t*>(meta + 2 * BK);
            // pass 2, one 32-key chunk at a time (a rolled loop keeps the code small):
            // the chunk's exponentials first (all independent), then the segment
            // sums in key order, flushed at every key-group end.  Columns past the
            // tile's keys give e = 0 and carry no group end, so no test branches.
            const size_t row_idx = ((size_t)bh * Cq + a) * Ck;
            const float m_nat = Mr * 0.6931471805599453f;   // back to natural-log units
#pragma unroll 1
            for (int c4 = 0; c4 < BK / 32; ++c4) {
                float v[32];
                tmem_ld32(t_row + stage * BK + c4 * 32, v);
                tmem_wait_ld(v);
                const int nv = ncol - c4 * 32;
                const uint32_t em = endm[c4];   // group ends at these keys (same for every row)
                const float4* u4 = reinterpret_cast<const float4*>(meta + c4 * 32);
                const float4* w4 = reinterpret_cast<const float4*>(meta + BK + c4 * 32);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = i < nv ? ex2_approx(fmaf(v[i], cs, -Mr)) : 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 uq = u4[q], wq = w4[q];
                    const float uu[4] = {uq.x, uq.y, uq.z, uq.w}, ww[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int i = 4 * q + k;
                        const float e = v[i];
                        t1 = fmaf(e, uu[k], t1);
                        t2 = fmaf(e * e, ww[k], t2);
                        if ((em >> i) & 1u) {   // uniform: group b ends at this key
                            if (a < Cqp) {
                                mloc[row_idx + b] = m_nat;
                                t1o[row_idx + b] = t1;
                                t2o[row_idx + b] = t2;
                            }
                            ++b;
                            t1 = 0.f;
                            t2 = 0.f;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bar(B_DE + stage));
            mbar_arrive(bar(B_ME + ring));
        }
        if (!ok) {
            record_status(status, SPARSEPR_TIMEOUT, 32);
            *abort_flag = 1;
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ================================================================ host side
namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn_rt() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}
bool make_bf16_rows(CUtensorMap* m, const void* base, uint64_t rows, int d) {
    EncodeTiledFn fn = encode_fn_rt();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

bool route_uses_tc(const sparsepr_params& p) { return p.dtype == SPARSEPR_BF16; }

bool launch_route_tc(const Plan& pl, const sparsepr_partition_out& part, void* ws, float* t1, float* t2, float* ml,
                     cudaStream_t st) {
    const int BH = pl.BH, N = pl.N, d = pl.d;
    const int CqPad = round_up(pl.Cq, rtc::BA);
    __nv_bfloat16* qs = at<__nv_bfloat16>(ws, pl.o_qsplit);
    float2* uw = at<float2>(ws, pl.o_uw);
    DevStatus* status = at<DevStatus>(ws, pl.o_status);
    count_launch(), route_qsplit_kernel<<<dim3(64, BH), 256, 0, st>>>(part.q_centroid, part.n_groups, pl.Cq, CqPad, d, qs);
    const int G = pl.G, BHk = BH / G;
    count_launch(), route_uw_kernel<__nv_bfloat16><<<148 * 8, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(part.Vp), part.v_centroid, part.kv_label, part.perm_kv, BHk, N, pl.Ck, d, G,
        uw);
    rtc::Maps maps;
    if (!make_bf16_rows(&maps.a, qs, (uint64_t)BH * 3 * CqPad, d)) return false;
    if (!make_bf16_rows(&maps.k, part.Kp, (uint64_t)BHk * N, d)) return false;
    const dim3 grid((pl.Ck + rtc::GPB - 1) / rtc::GPB, CqPad / rtc::BA, BH);
    if (d == 128) {
        cudaFuncSetAttribute(route_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, rtc::Layout<128>::smem);
        count_launch(), route_tc_kernel<128><<<grid, 192, rtc::Layout<128>::smem, st>>>(
            maps, uw, part.kv_offsets, part.n_groups, N, pl.Cq, pl.Ck, CqPad, G, t1, t2, ml, status);
    } else {
        cudaFuncSetAttribute(route_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, rtc::Layout<64>::smem);
        count_launch(), route_tc_kernel<64><<<grid, 192, rtc::Layout<64>::smem, st>>>(
            maps, uw, part.kv_offsets, part.n_groups, N, pl.Cq, pl.Ck, CqPad, G, t1, t2, ml, status);
    }
    return true;
}

}  // namespace spr
