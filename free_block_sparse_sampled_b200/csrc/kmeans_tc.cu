// k-means assignment on the tensor cores ("Partition the Support, Reconstruct
// the Residual", §4.1, C.1): label = argmax_c (x.c - |c|^2/2), ties to the
// lowest c, for 128 points per block against every centre.
//
// Coordinates and centres are stored TF32-rounded (round to nearest even),
// so the tcgen05 kind::tf32 products are exact and the scores carry only fp32
// accumulation error.  The -|c|^2/2 term joins the product as one more K step:
// a constant tile of ones (two columns) against each centre's -|c|^2/2 split
// into TF32 hi and lo parts, so the tensor core returns the score itself.
// Coordinates and centres move through shared memory as 16-float column
// chunks (TMA, 64-byte swizzle, sized to the rank): the points of an item in
// two buffers, the centres in blocks of up to 256 in two stages, with their
// split half-norms 32-byte swizzled.  The scores of a block land in TMEM (two
// buffers) and eight epilogue warps (two per TMEM lane quadrant, each owning
// half of the columns) take the running argmax while the next block
// multiplies.  All waits are bounded.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace spr {
namespace kmtc {
constexpr int BP = 128;                 // points per item (TMEM lanes)
constexpr uint32_t kSpin = 1u << 20;
enum { B_AF = 0, B_AE = 2, B_BF = 4, B_DF = 6, B_DE = 8, B_DR = 10, N_BAR = 11 };
constexpr int kKeepStride = 144;        // bytes per lane of the best-chunk copy (32 floats + 16: no bank conflicts)

// Shared-memory plan for rank R and centre blocks of NB (every tile 1024-aligned):
//   A: 2 buffers x R/16 chunks x 128 rows x 64 B; B: 2 stages x R/16 chunks x NB rows x 64 B;
//   a 128 x 8 TF32 ones tile and 2 stages x NB x 8 TF32 split half-norms (32-byte swizzle);
//   per epilogue lane a copy of its best 32-score chunk; barriers; the half merge.
struct Layout {
    int a_buf, b_stage, oA, oB, oOnes, oH, oKeep, oBar, oRed, oMisc, bytes;
    __host__ __device__ Layout(int R, int NB) {
        a_buf = BP * R * 4;
        b_stage = NB * R * 4;
        oA = 0;
        oB = oA + 2 * a_buf;
        oOnes = oB + 2 * b_stage;
        oH = oOnes + BP * 32;
        oKeep = oH + 2 * NB * 32;
        oBar = oKeep + 8 * 32 * kKeepStride;
        oRed = oBar + N_BAR * 8;
        oMisc = oRed + BP * 8;
        bytes = oMisc + 64 + 1024;
    }
};
// largest centre block for rank R that keeps the plan within 227 KB
__host__ __device__ constexpr int nb_max(int R) { return R > 48 ? 192 : 256; }

struct Maps {
    CUtensorMap pts;       // [BH*N, R] fp32, box 16 x 128, 64-byte swizzle
    CUtensorMap cen;       // [BH*C, R] fp32, box 16 x NB, 64-byte swizzle
    CUtensorMap hs;        // [BH*C, 8] fp32, box 8 x NB, 32-byte swizzle
};

// Byte offset of element (row, k) of a [rows x 8] fp32 tile in the 32-byte
// swizzled K-major layout (16-byte unit index XOR bit 2 of the row).
__device__ __forceinline__ uint32_t sw32(int row, int k) {
    return (uint32_t)(row * 32 + ((((k >> 2) ^ (row >> 2)) & 1) << 4) + (k & 3) * 4);
}

// -|c|^2/2 of every centre as (hi, lo, 0, 0, 0, 0, 0, 0) with hi the TF32
// rounding and lo the TF32 rounding of the remainder.
__global__ void half_norm_split_kernel(const float* __restrict__ hn, size_t n, float* __restrict__ hs) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const float h = -hn[e], hi = tf32_round(h), lo = tf32_round(h - hi);
        float4* o = reinterpret_cast<float4*>(hs + e * 8);
        o[0] = make_float4(hi, lo, 0.f, 0.f);
        o[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}
// Maximum of 32 scores as a tree of three-way maxima.
__device__ __forceinline__ float max32(const float (&s)[32]) {
    using sm100::fmax3;
    float m3[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) m3[i] = fmax3(s[3 * i], s[3 * i + 1], s[3 * i + 2]);
    m3[10] = fmaxf(s[30], s[31]);
    return fmaxf(fmax3(fmax3(m3[0], m3[1], m3[2]), fmax3(m3[3], m3[4], m3[5]), fmax3(m3[6], m3[7], m3[8])),
                 fmaxf(m3[9], m3[10]));
}

// Stores a chunk of 32 scores at a shared-window address.
__device__ __forceinline__ void st_chunk(uint32_t a, const float (&v)[32]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) sm100::st_shared_v4(a + 16 * j, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

// One 64-column pair of an epilogue lane: the chunks of 32 scores at columns
// cb0 and cb0 + 32, of which the columns below lim take part.  MODE 0: both
// chunks whole; 1: the first whole and the second past lim; 2: columns at or
// past lim masked to -inf.  Both chunk maxima are taken before either updates
// the running first maximum (best, the base column bcb of its chunk); a lane
// whose maximum moved then rewrites its copy of the best chunk at `keep`.
template <int MODE, bool DBG>
__device__ __forceinline__ void pair_update(float (&v)[2][32], int cb0, int lim, float& best, int& bcb, uint32_t keep,
                                            float* dbg_row) {
    if (MODE == 2) {
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int i = 0; i < 32; ++i) v[q][i] = (cb0 + 32 * q + i < lim) ? v[q][i] : -INFINITY;
    }
    if (DBG && dbg_row != nullptr) {
#pragma unroll
        for (int q = 0; q < (MODE == 1 ? 1 : 2); ++q)
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (cb0 + 32 * q + i < lim) dbg_row[cb0 + 32 * q + i] = v[q][i];
    }
    const float m0 = max32(v[0]);
    if (MODE == 1) {
        const bool up0 = m0 > best;   // a later chunk only wins with a strictly larger score
        best = up0 ? m0 : best;
        bcb = up0 ? cb0 : bcb;
        if (up0) st_chunk(keep, v[0]);
        return;
    }
    const float m1 = max32(v[1]);
    const bool up0 = m0 > best;
    const float b0 = up0 ? m0 : best;
    const bool up1 = m1 > b0;
    best = up1 ? m1 : b0;
    bcb = up1 ? cb0 + 32 : (up0 ? cb0 : bcb);
    // divergent branches after both maxima: only the lanes that move store
    // (predicated stores cost shared-memory bandwidth for every lane)
    if (up1) st_chunk(keep, v[1]);
    else if (up0) st_chunk(keep, v[0]);
}
// The K steps of one centre block: D = A B^T over R/8 TF32 steps of 8, then
// + ones x (hi, lo) for the -|c|^2/2 term.  Descriptors advance by the
// 64-byte chunk stride (512 units for the points, cb for the centres) every
// second step and by 32 bytes inside a chunk.
template <int KS>
__device__ __forceinline__ void mma_block(uint32_t d, uint64_t a0, uint64_t b0, uint32_t cb, uint64_t ones, uint64_t h,
                                          uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
        const uint64_t oa = (uint64_t)((kk >> 1) * ((BP * 64) >> 4) + (kk & 1) * 2);
        const uint64_t ob = (uint64_t)((kk >> 1) * cb + (kk & 1) * 2);
        sm100::mma_tf32_ss(d, a0 + oa, b0 + ob, idesc, kk > 0 ? 1u : 0u);
    }
    sm100::mma_tf32_ss(d, ones, h, idesc, 1u);
}
}  // namespace kmtc

// Persistent: block k handles items k, k + grid, ... where an item is 128
// points of one head; heads whose k-means has stopped are skipped by every role.
template <bool DBG>
__global__ void __launch_bounds__(320, 1) kmeans_assign_tc_kernel(
    const __grid_constant__ kmtc::Maps maps, int BH, int N, int C, int R, int NB,
    int nblk, int32_t* __restrict__ labels, int32_t* __restrict__ ctl, int first, float* __restrict__ dbg_scores,
    int32_t* __restrict__ dbg_hist, int max_iter, DevStatus* status) {
    using namespace kmtc;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    if (*reinterpret_cast<volatile const int32_t*>(&status->code) != 0) return;
    const int tiles_per_head = (N + BP - 1) / BP;
    const int n_items = BH * tiles_per_head;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t s_base = smem_u32(sm);
    const Layout L(R, NB);
    auto bar = [&](int i) -> uint32_t { return s_base + L.oBar + 8 * i; };
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L.oMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    const int nchunk = R / 16;                  // 16 fp32 per 64-byte row chunk
    const int ksteps = R / 8;                   // kind::tf32 K = 8 per instruction
    // a head's stop flag is set between launches: each role reads it once per head
    int live_bh = -1;
    bool live = false;
    auto item_live = [&](int w) -> bool {
        const int bh = w / tiles_per_head;
        if (bh != live_bh) {
            live_bh = bh;
            live = ctl[bh * kCtlStride + kCtlDone] == 0;
        }
        return live;
    };

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_AF + s), 1);
            mbar_init(bar(B_AE + s), 1);
            mbar_init(bar(B_BF + s), 1);
            mbar_init(bar(B_DF + s), 1);
            mbar_init(bar(B_DE + s), 256);
        }
        mbar_init(bar(B_DR), 1);
        fence_barrier_init();
        misc[1] = 0;
    }
    {   // the ones tile of the half-norm K step: columns 0 and 1 of every row
        float* ones = reinterpret_cast<float*>(sm + L.oOnes);
        for (int e = tid; e < BP * 8; e += blockDim.x) {
            const int row = e >> 3, k = e & 7;
            ones[sw32(row, k) >> 2] = k < 2 ? 1.f : 0.f;
        }
        fence_proxy_async_smem();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(misc), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == 8) {
        if (lane == 0) {   // TMA producer
            prefetch_tmap(&maps.pts);
            prefetch_tmap(&maps.cen);
            prefetch_tmap(&maps.hs);
            int li = 0, gb = 0;           // local item count, global centre-block count
            bool ok = true;
            for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
                if (!item_live(w)) continue;
                const int bh = w / tiles_per_head, p0 = (w % tiles_per_head) * BP, ab = li & 1;
                if (li >= 2 && !mbar_wait(bar(B_AE + ab), ((li >> 1) - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                mbar_arrive_expect_tx(bar(B_AF + ab), L.a_buf);
                for (int ch = 0; ch < nchunk; ++ch)
                    tma_load_2d(s_base + L.oA + ab * L.a_buf + ch * BP * 64, &maps.pts, bar(B_AF + ab), ch * 16,
                                bh * N + p0);
                for (int blk = 0; blk < nblk; ++blk, ++gb) {
                    const int stage = gb & 1;
                    // the stage is free once the products of block gb - 2 are done (the
                    // commit that also hands their scores to the epilogue)
                    if (gb >= 2 && !mbar_wait(bar(B_DF + stage), ((gb >> 1) - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                    mbar_arrive_expect_tx(bar(B_BF + stage), L.b_stage + NB * 32);
                    for (int ch = 0; ch < nchunk; ++ch)
                        tma_load_2d(s_base + L.oB + stage * L.b_stage + ch * NB * 64, &maps.cen, bar(B_BF + stage),
                                    ch * 16, bh * C + blk * NB);
                    tma_load_2d(s_base + L.oH + stage * NB * 32, &maps.hs, bar(B_BF + stage), 0, bh * C + blk * NB);
                }
                ++li;
            }
            if (!ok) {
                record_status(status, SPARSEPR_TIMEOUT, 20);
                *abort_flag = 1;
            }
            for (int t = max(0, li - 2); t < li; ++t) mbar_wait(bar(B_AF + (t & 1)), (t >> 1) & 1, nullptr, kSpin);
            for (int t = max(0, gb - 2); t < gb; ++t) mbar_wait(bar(B_BF + (t & 1)), (t >> 1) & 1, nullptr, kSpin);
        }
    } else if (warp == 9) {
        if (lane == 0) {   // MMA issuer
            const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(NB >> 3) << 17) |
                                   ((uint32_t)(BP >> 4) << 24);   // F32 <- TF32 x TF32, K-major both
            // descriptors built once; each MMA adds its offset (>> 4) to the
            // start-address field, which never carries out (shared < 2^18)
            const uint64_t dA = smem_desc_sw64(s_base + L.oA), dB = smem_desc_sw64(s_base + L.oB);
            const uint64_t dOnes = smem_desc_sw32(s_base + L.oOnes), dH = smem_desc_sw32(s_base + L.oH);
            int li = 0, gb = 0;
            bool ok = true;
            for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
                if (!item_live(w)) continue;
                const int ab = li & 1;
                if (!mbar_wait(bar(B_AF + ab), (li >> 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                const uint64_t a0 = dA + (uint64_t)((ab * L.a_buf) >> 4);
                for (int blk = 0; blk < nblk; ++blk, ++gb) {
                    const int stage = gb & 1;
                    if (!mbar_wait(bar(B_BF + stage), (gb >> 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                    if (gb >= 2 && !mbar_wait(bar(B_DE + stage), ((gb >> 1) - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t b0 = dB + (uint64_t)((stage * L.b_stage) >> 4);
                    const uint32_t d = tmem + stage * NB;
                    const uint64_t h0 = dH + (uint64_t)((stage * NB * 32) >> 4);
                    switch (ksteps) {
                        case 4: mma_block<4>(d, a0, b0, (uint32_t)((NB * 64) >> 4), dOnes, h0, idesc); break;
                        case 6: mma_block<6>(d, a0, b0, (uint32_t)((NB * 64) >> 4), dOnes, h0, idesc); break;
                        default: mma_block<8>(d, a0, b0, (uint32_t)((NB * 64) >> 4), dOnes, h0, idesc); break;
                    }
                    mma_commit(bar(B_DF + stage));
                }
                mma_commit(bar(B_AE + ab));
                ++li;
            }
            if (!ok) {
                record_status(status, SPARSEPR_TIMEOUT, 21);
                *abort_flag = 1;
            }
            mma_commit(bar(B_DR));
            mbar_wait(bar(B_DR), 0, nullptr, kSpin);
        }
    } else {
        // epilogue: warps 0-3 take the lower half of each centre block, 4-7 the upper half
        const int half = warp >> 2, row = (warp & 3) * 32 + lane;
        const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const int hw = NB / 2;
        float* red_s = reinterpret_cast<float*>(sm + L.oRed);
        int* red_i = reinterpret_cast<int*>(sm + L.oRed + BP * 4);
        // this lane's copy of its best chunk
        const uint32_t keep = s_base + L.oKeep + (uint32_t)(warp * 32 + lane) * kKeepStride;
        int gb = 0;
        bool ok = true;
        for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
            if (!item_live(w)) continue;
            const int bh = w / tiles_per_head, p = (w % tiles_per_head) * BP + row;
            const bool valid = p < N;
            int32_t* hc = ctl + bh * kCtlStride;
            // previous label, read now and used after the last centre block
            const int old_label = (valid && !first) ? labels[(size_t)bh * N + p] : 0;
            // running first maximum over this half's columns, in column order: the
            // best value, the base column of the chunk holding it and, in shared
            // memory, a copy of that chunk's scores (eight vector stores by the
            // lanes that move, instead of a per-chunk index search, which every
            // chunk would run: some lane of the warp almost always improves); the
            // index is searched once per item
            float best = -INFINITY;
            int bcb = 0;
            float* dbg_row = (DBG && valid) ? dbg_scores + ((size_t)bh * N + p) * C : nullptr;
            for (int blk = 0; blk < nblk; ++blk, ++gb) {
                const int db = gb & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DF + db), (gb >> 1) & 1, abort_flag, kSpin));
                if (!ok) break;
                tc_fence_after();
                // the columns of this half that hold centres of this head
                const int lim = min(C, blk * NB + (half + 1) * hw);
                for (int c0 = 0; c0 < hw; c0 += 64) {
                    const int cb0 = blk * NB + half * hw + c0;   // warp-uniform
                    if (cb0 >= lim) break;
                    // 64 columns (those past the half stay inside the allocation and are masked)
                    float v[2][32];
                    tmem_ld32(t_row + db * NB + half * hw + c0, v[0]);
                    tmem_ld32(t_row + db * NB + half * hw + c0 + 32, v[1]);
                    tmem_wait_ld(v[0]);
                    tmem_wait_ld(v[1]);
                    if (cb0 + 64 <= lim) pair_update<0, DBG>(v, cb0, lim, best, bcb, keep, dbg_row);
                    else if (cb0 + 32 == lim) pair_update<1, DBG>(v, cb0, lim, best, bcb, keep, dbg_row);
                    else pair_update<2, DBG>(v, cb0, lim, best, bcb, keep, dbg_row);
                }
                tc_fence_before();
                mbar_arrive(bar(B_DE + db));
            }
            if (!ok) break;
            int bi = 0x7fffffff;
            if (best > -INFINITY) {
                float kv[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) ld_shared_v4(keep + 16 * j, kv[4 * j], kv[4 * j + 1], kv[4 * j + 2], kv[4 * j + 3]);
                int idx = 31;
#pragma unroll
                for (int i = 30; i >= 0; --i) idx = (kv[i] == best) ? i : idx;
                bi = bcb + idx;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (half == 1) {
                red_s[row] = best;
                red_i[row] = bi;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (half == 0) {
                const float b1 = red_s[row];
                const int i1 = red_i[row];
                if (b1 > best || (b1 == best && i1 < bi)) {
                    best = b1;
                    bi = i1;
                }
                if (bi == 0x7fffffff) bi = 0;
                int changed = 0;
                if (valid) {
                    int32_t* lp = labels + (size_t)bh * N + p;
                    changed = (!first) && (old_label != bi);
                    *lp = bi;
                    if (dbg_hist != nullptr) dbg_hist[((size_t)bh * max_iter + hc[kCtlIters]) * N + p] = bi;
                }
                const unsigned ballot = __ballot_sync(0xffffffffu, changed);
                if (lane == 0 && ballot) atomicAdd(&hc[kCtlChanged], __popc(ballot));
            }
        }
        if (!ok) {
            record_status(status, SPARSEPR_TIMEOUT, 22);
            *abort_flag = 1;
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ================================================================ host side
namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn_km() {
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
bool make_f32_map(CUtensorMap* m, const void* base, uint64_t rows, int R, int box_rows, int box_cols = 32,
                  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn_km();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)R, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)R * 4};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

void kmeans_centre_blocks(int C, int R, int& NB, int& nblk) {
    const int nbm = kmtc::nb_max(R);
    nblk = (C + nbm - 1) / nbm;
    NB = round_up((C + nblk - 1) / nblk, 64);
    if (NB > nbm) NB = nbm;
}

bool launch_kmeans_assign_tc(const float* phi, const float* cen, const float* hn, float* hs, int BH, int N, int C,
                             int R, int32_t* labels, int32_t* ctl, int first, float* dbg_scores, int32_t* dbg_hist,
                             int max_iter, DevStatus* status, cudaStream_t st) {
    if (R > kMaxRank || R % 16 != 0) return false;   // 16-float chunks of rows of up to 64 floats
    int NB, nblk;
    kmeans_centre_blocks(C, R, NB, nblk);
    const kmtc::Layout L(R, NB);
    kmtc::Maps maps;
    if (!make_f32_map(&maps.pts, phi, (uint64_t)BH * N, R, kmtc::BP, 16, CU_TENSOR_MAP_SWIZZLE_64B)) return false;
    if (!make_f32_map(&maps.cen, cen, (uint64_t)BH * C, R, NB, 16, CU_TENSOR_MAP_SWIZZLE_64B)) return false;
    if (!make_f32_map(&maps.hs, hs, (uint64_t)BH * C, 8, NB, 8, CU_TENSOR_MAP_SWIZZLE_32B)) return false;
    {
        const size_t n = (size_t)BH * C;
        const int g = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
        count_launch(), kmtc::half_norm_split_kernel<<<g, 256, 0, st>>>(hn, n, hs);
    }
    const int items = BH * ((N + kmtc::BP - 1) / kmtc::BP);
    const int grid = items < sm_count() ? items : sm_count();
    if (dbg_scores != nullptr) {
        cudaFuncSetAttribute(kmeans_assign_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, L.bytes);
        count_launch(), kmeans_assign_tc_kernel<true><<<grid, 320, L.bytes, st>>>(
            maps, BH, N, C, R, NB, nblk, labels, ctl, first, dbg_scores, dbg_hist, max_iter, status);
    } else {
        cudaFuncSetAttribute(kmeans_assign_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, L.bytes);
        count_launch(), kmeans_assign_tc_kernel<false><<<grid, 320, L.bytes, st>>>(
            maps, BH, N, C, R, NB, nblk, labels, ctl, first, dbg_scores, dbg_hist, max_iter, status);
    }
    return true;
}

}  // namespace spr
