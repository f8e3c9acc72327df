// Block-sparse attention over group-permuted Q/K/V and exact probe rows
// ("Partition the Support, Reconstruct the Residual", §3 Eq. (2), §4.3).
//
// Work items are query tiles of at most 128 rows that never cross a query
// group, plus tiles of probe rows.  A sparse item attends to the rows of
// every K/V group selected for its query group; a probe item attends to all N
// keys.  Softmax is renormalised over exactly those keys.
//
// bf16, block 128: tcgen05 kernel.  Warps 0-3 own the 128 query rows (TMEM
// lanes) and run the online softmax; warp 4 streams K/V with TMA in 8-row
// slots (one 1 KB box per 8 keys x 64 channels, 128-byte swizzle) so ragged
// K/V groups pack into 128-key tiles with little padding (partially used
// slots are masked); warp 5 issues S = Q K^T and O += P V into TMEM.
// Every wait is bounded; on timeout the kernel records SPARSEPR_TIMEOUT, lets
// in-flight copies and MMAs finish, frees TMEM and returns.
//
// fp32 inputs (or the SIMT flag): CUDA-core kernel with the same work items.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace spr {

// ---------------------------------------------------------------- work items
// Items never cross a query group.  pair == 0: one tile of BM rows per item
// (w = rows).  pair == 1: two consecutive 128-row tiles per item
// (w = rows of tile 0 | rows of tile 1 << 16).
__global__ void __launch_bounds__(1024) build_work_kernel(const int32_t* __restrict__ q_off,
                                                          const int32_t* __restrict__ ng, int Cq, int BM, int pair,
                                                          int4* __restrict__ items,
                                                          int32_t* __restrict__ counter) {
    __shared__ int cnt[kMaxGroups];
    __shared__ int scratch[33];
    __shared__ int base;
    const int bh = blockIdx.x;
    const int Cqp = ng[bh * 2 + 0];
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    const int span = pair ? 2 * BM : BM;
    for (int a = threadIdx.x; a < Cqp; a += blockDim.x) cnt[a] = (qo[a + 1] - qo[a] + span - 1) / span;
    __syncthreads();
    const int total = block_exclusive_scan(cnt, Cqp, scratch);
    if (threadIdx.x == 0) base = atomicAdd(counter, total);
    __syncthreads();
    for (int a = threadIdx.x; a < Cqp; a += blockDim.x) {
        const int s = qo[a], size = qo[a + 1] - qo[a];
        const int n = (size + span - 1) / span;
        for (int t = 0; t < n; ++t) {
            const int rest = size - t * span;
            const int w = pair ? (min(BM, rest) | (max(0, min(BM, rest - BM)) << 16)) : min(BM, rest);
            items[base + cnt[a] + t] = make_int4(bh, a, s + t * span, w);
        }
    }
}

struct Item {
    int bh, a, row0, nrows;
};

__device__ __forceinline__ bool decode_item(int item, const int4* items, const int32_t* counter,
                                            int n_probe_items, int BM, int Mp, Item& it) {
    if (item < n_probe_items) {
        const int per = (Mp + BM - 1) / BM;
        it.bh = item / per;
        it.a = -1;
        it.row0 = (item % per) * BM;
        it.nrows = min(BM, Mp - it.row0);
        return true;
    }
    const int k = item - n_probe_items;
    if (k >= *counter) return false;
    const int4 w = items[k];
    it.bh = w.x;
    it.a = w.y;
    it.row0 = w.z;
    it.nrows = w.w;
    return true;
}


// Walks the 8-row key slots of an item: every selected K/V group (or all N
// keys for a probe item) is cut into slots of 8 rows; the last slot of a
// group holds fewer valid rows.  Slots past the end are padding (v = 0).
struct SlotCursor {
    const int32_t* sg;
    const int32_t* ko;
    int n_groups, gi, r_start, r_len, r_off, probe_next, N;
    bool probe, have;
    __device__ __forceinline__ SlotCursor(const Item& it, const int32_t* sel_groups, const int32_t* sel_count,
                                          const int32_t* kv_off, int Cq, int Ck, int N_)
        : gi(0), r_start(0), r_len(0), r_off(0), probe_next(0), N(N_), have(false) {
        probe = it.a < 0;
        sg = sel_groups + ((size_t)it.bh * Cq + (probe ? 0 : it.a)) * Ck;
        ko = kv_off + (size_t)it.bh * (Ck + 1);
        n_groups = probe ? 0 : sel_count[(size_t)it.bh * Cq + it.a];
    }
    __device__ __forceinline__ void next(int& row, int& v) {
        row = -1;
        v = 0;
        if (probe) {
            if (probe_next < N) {
                row = probe_next;
                v = min(8, N - probe_next);
                probe_next += 8;
            }
            return;
        }
        while (!have && gi < n_groups) {
            const int b = sg[gi++];
            r_start = ko[b];
            r_len = ko[b + 1] - r_start;
            r_off = 0;
            have = r_len > 0;
        }
        if (have) {
            row = r_start + r_off;
            v = min(8, r_len - r_off);
            r_off += 8;
            if (r_off >= r_len) have = false;
        }
    }
};

// ---------------------------------------------------------------- gathers
template <typename T>
__global__ void gather_probe_rows_kernel(const T* __restrict__ src, const int32_t* __restrict__ probe_idx,
                                         const int32_t* __restrict__ pos_q, int BH, int N, int Mp, int d,
                                         T* __restrict__ dst) {
    const int chunks = d * (int)sizeof(T) / 16;
    const size_t total = (size_t)BH * Mp * chunks;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const size_t r = e / chunks;
        const int c = (int)(e - r * chunks);
        const size_t bh = r / Mp;
        const size_t p = bh * N + pos_q[bh * N + probe_idx[r]];
        reinterpret_cast<uint4*>(dst)[r * chunks + c] = reinterpret_cast<const uint4*>(src)[p * chunks + c];
    }
}

// ---------------------------------------------------------------- SIMT kernel
// Two threads per query row (each owns half of the channels); keys staged
// 32 at a time in shared memory; online softmax in the log2 domain.
template <typename T, int D>
__global__ void __launch_bounds__(256) attention_simt_kernel(
    const T* __restrict__ Qp, const T* __restrict__ Kp, const T* __restrict__ Vp,
    const T* __restrict__ Qprobe, const int4* __restrict__ items, const int32_t* __restrict__ counter,
    int n_probe_items, int BM, int N, int Mp, int Cq, int Ck, const int32_t* __restrict__ kv_off,
    const int32_t* __restrict__ sel_count, const int32_t* __restrict__ sel_groups,
    float* __restrict__ O_sp, float* __restrict__ probe_dense, unsigned long long* __restrict__ visited,
    float scale_log2, int G) {
    constexpr int H = D / 2, KC = 32;
    __shared__ float ks[KC][D];
    __shared__ float vs[KC][D];
    Item it;
    if (!decode_item(blockIdx.x, items, counter, n_probe_items, BM, Mp, it)) return;
    const int r = threadIdx.x >> 1, h = threadIdx.x & 1;
    const bool active = r < it.nrows;
    const T* qrow = (it.a < 0) ? Qprobe + ((size_t)it.bh * Mp + it.row0 + r) * D
                               : Qp + ((size_t)it.bh * N + it.row0 + r) * D;
    float q[H], o[H];
#pragma unroll
    for (int t = 0; t < H; ++t) {
        q[t] = active ? ldf(qrow + h * H + t) * scale_log2 : 0.f;
        o[t] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    const int n_ranges = (it.a < 0) ? 1 : sel_count[(size_t)it.bh * Cq + it.a];
    const int32_t* sg = sel_groups + ((size_t)it.bh * Cq + (it.a < 0 ? 0 : it.a)) * Ck;
    const int32_t* ko = kv_off + (size_t)it.bh * (Ck + 1);
    for (int g = 0; g < n_ranges; ++g) {
        int s, e;
        if (it.a < 0) {
            s = 0;
            e = N;
        } else {
            const int b = sg[g];
            s = ko[b];
            e = ko[b + 1];
        }
        for (int c0 = s; c0 < e; c0 += KC) {
            const int n = min(KC, e - c0);
            __syncthreads();
            for (int x = threadIdx.x; x < KC * D; x += blockDim.x) {
                const int j = x / D, t = x % D;
                const bool ok = j < n;
                const size_t kr = (size_t)(it.bh / G) * N + c0 + j;   // the K/V head under GQA
                ks[j][t] = ok ? ldf(Kp + kr * D + t) : 0.f;
                vs[j][t] = ok ? ldf(Vp + kr * D + t) : 0.f;
            }
            __syncthreads();
            float sc[KC];
            float cm = -INFINITY;
#pragma unroll
            for (int j = 0; j < KC; ++j) {
                float part = 0.f;
#pragma unroll
                for (int t = 0; t < H; ++t) part = fmaf(q[t], ks[j][h * H + t], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                sc[j] = (j < n) ? part : -INFINITY;
                cm = fmaxf(cm, sc[j]);
            }
            const float mn = fmaxf(m, cm);
            const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - mn);
            l *= alpha;
#pragma unroll
            for (int t = 0; t < H; ++t) o[t] *= alpha;
            m = mn;
#pragma unroll
            for (int j = 0; j < KC; ++j) {
                if (j < n) {
                    const float p = exp2f(sc[j] - m);
                    l += p;
#pragma unroll
                    for (int t = 0; t < H; ++t) o[t] = fmaf(p, vs[j][h * H + t], o[t]);
                }
            }
        }
    }
    if (threadIdx.x == 0) {
        unsigned long long keys = 0;
        for (int g = 0; g < n_ranges; ++g)
            keys += (it.a < 0) ? (unsigned long long)N : (unsigned long long)(ko[sg[g] + 1] - ko[sg[g]]);
        atomicAdd(visited, keys * (unsigned long long)BM);
    }
    if (!active) return;
    float* out = (it.a < 0) ? probe_dense + ((size_t)it.bh * Mp + it.row0 + r) * D
                            : O_sp + ((size_t)it.bh * N + it.row0 + r) * D;
    const float inv = 1.f / l;
#pragma unroll
    for (int t = 0; t < H; ++t) out[h * H + t] = o[t] * inv;
}

// ---------------------------------------------------------------- tcgen05 kernel
// One block handles up to two 128-row query tiles of the same query group
// (or two tiles of probe rows) against the same key sequence.
//   warps 0-3 / 4-7: online softmax of Q tile 0 / 1 (one TMEM lane per row)
//   warp 8: TMA producer (whole warp), warp 9: MMA issuer, warps 10-11 idle
// TMEM: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).  P_t
// (fp16, two per column) overwrites the first 64 columns of S_t and feeds
// O_t += P_t V as a TMEM-operand MMA.  The MMA thread issues PV_t(j-1)
// before S_t(j), so the commit that publishes S_t(j) also certifies that O_t
// is quiescent for the softmax's lazy rescale.
namespace tc {
constexpr int BM = 128, BN = 128, NS = 2, RING = 4, NBOX = 5;   // boxes of 8 << k rows, k < NBOX
constexpr int kThreads = 384;   // 3 warpgroups: softmax tile 0, softmax tile 1, producer + MMA
constexpr int kLaunchRegs = 168, kRegsSoftmax = 224, kRegsOther = 56;
// what the softmax warpgroups take, the third gives back: per block and per
// SM sub-partition (which holds one warp of each warpgroup)
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther == kThreads * kLaunchRegs, "register split");
static_assert(2 * kRegsSoftmax + kRegsOther == 3 * kLaunchRegs, "register split per sub-partition");
constexpr uint32_t kSpin = 1u << 20;   // polls of mbarrier.try_wait before giving up
#ifndef SPR_SOFT_PAIRS
#define SPR_SOFT_PAIRS 2
#endif
// exponential pairs, of every 16, computed on the FMA pipe instead of the MUFU
constexpr int kSoftPairs = SPR_SOFT_PAIRS;
static_assert(kSoftPairs >= 0 && kSoftPairs <= 16, "soft pairs per 16");
enum { B_Q = 0, B_KF = 1, B_KE = B_KF + NS, B_VF = B_KE + NS, B_VE = B_VF + NS, B_SF = B_VE + NS,
       B_PF = B_SF + 2, B_OF = B_PF + 2, B_DR = B_OF + 1, B_MF = B_DR + 1, B_ME = B_MF + RING,
       B_ST = B_ME + RING,   // never signalled: the stall hook's wait (sparsepr_debug_stall_attention)
       N_BAR = B_ST + 1 };

template <int D>
struct Layout {
    static constexpr int QB = BM * D * 2;          // one Q tile
    static constexpr int KB = BN * D * 2;          // one K (or V) stage
    static constexpr int oQ = 0;                   // two Q tiles
    static constexpr int oK = oQ + 2 * QB;
    static constexpr int oV = oK + NS * KB;
    static constexpr int oBar = oV + NS * KB;
    static constexpr int oMeta = (oBar + N_BAR * 8 + 15) / 16 * 16;   // RING x 16 valid-row counts (read as uint4)
    static constexpr int oRun = oMeta + RING * 16;  // 16 x (first row, slot count) of the tile being loaded
    static constexpr int oMisc = oRun + 16 * 8;
    static constexpr int bytes = oMisc + 64;
    static constexpr int smem = bytes + 1024;      // slack for 1024-byte alignment
    static_assert(oK % 1024 == 0 && oV % 1024 == 0, "swizzled tiles need 1024-byte alignment");
    static_assert(oMeta % 16 == 0 && oRun % 8 == 0, "vector accesses need aligned offsets");
};

// Tensor maps: K (bf16) and V (fp16) rows in boxes of 8, 16, 32, 64, 128 rows x
// 64 channels; Q and probe-Q in boxes of 128 rows.  All 128-byte swizzled.
struct Maps {
    CUtensorMap k[NBOX];
    CUtensorMap v[NBOX];
    CUtensorMap q;
    CUtensorMap qp;
};
}  // namespace tc

struct Item2 {
    int bh, a, row0, n0, n1;
};

__device__ __forceinline__ bool decode_item2(int item, const int4* items, const int32_t* counter, int n_probe_items,
                                             int Mp, Item2& it) {
    if (item < n_probe_items) {
        const int per = (Mp + 255) / 256;
        it.bh = item / per;
        it.a = -1;
        it.row0 = (item % per) * 256;
        it.n0 = min(128, Mp - it.row0);
        it.n1 = max(0, min(128, Mp - it.row0 - 128));
        return true;
    }
    const int k = item - n_probe_items;
    if (k >= *counter) return false;
    const int4 w = items[k];
    it.bh = w.x;
    it.a = w.y;
    it.row0 = w.z;
    it.n0 = w.w & 0xffff;
    it.n1 = w.w >> 16;
    return true;
}

template <int D>
__global__ void __launch_bounds__(384, 1) attention_tc_kernel(
    const __grid_constant__ tc::Maps maps, const int4* __restrict__ items, const int32_t* __restrict__ counter,
    int n_probe_items, int N, int Mp, int Cq, int Ck, int total_rows, const int32_t* __restrict__ kv_off,
    const int32_t* __restrict__ sel_count, const int32_t* __restrict__ sel_groups, const float* __restrict__ vscale,
    float* __restrict__ O_sp, float* __restrict__ probe_dense, DevStatus* status,
    unsigned long long* __restrict__ visited, float scale_log2, uint32_t stall_polls, int G) {
    using namespace tc;
    using namespace sm100;
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    Item2 it;
    if (!decode_item2(blockIdx.x, items, counter, n_probe_items, Mp, it)) return;
    // once any block has given up, the rest of the launch returns at once
    if (*reinterpret_cast<volatile const int32_t*>(&status->code) != 0) return;
    const int nq = it.n1 > 0 ? 2 : 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t s_base = smem_u32(sm);
    const uint32_t sQ = s_base + L::oQ, sK = s_base + L::oK, sV = s_base + L::oV;
    auto bar = [&](int i) -> uint32_t { return s_base + L::oBar + 8 * i; };
    uint8_t* meta = sm + L::oMeta;
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::oMisc);   // [0] tmem, [1] abort, [2] n_tiles
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    if (tid == 0) {
        mbar_init(bar(B_Q), 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(B_KF + s), 1);
            mbar_init(bar(B_KE + s), 1);
            mbar_init(bar(B_VF + s), 1);
            mbar_init(bar(B_VE + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_SF + s), 1);
            mbar_init(bar(B_PF + s), 128);
        }
        mbar_init(bar(B_OF), 1);
        mbar_init(bar(B_DR), 1);
        mbar_init(bar(B_ST), 1);
        for (int s = 0; s < RING; ++s) {
            mbar_init(bar(B_MF + s), 1);
            mbar_init(bar(B_ME + s), 128 * nq);
        }
        fence_barrier_init();
        misc[1] = 0;
    }
    if (warp == 0) {   // number of 128-key tiles = ceil(slots / 16)
        long long slots = 0;
        if (it.a < 0) {
            slots = lane == 0 ? (N + 7) / 8 : 0;
        } else {
            const int cnt = sel_count[(size_t)it.bh * Cq + it.a];
            const int32_t* sg = sel_groups + ((size_t)it.bh * Cq + it.a) * Ck;
            const int32_t* ko = kv_off + (size_t)it.bh * (Ck + 1);
            for (int g = lane; g < cnt; g += 32) {
                const int b = sg[g];
                slots += (ko[b + 1] - ko[b] + 7) / 8;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) slots += __shfl_xor_sync(0xffffffffu, slots, o);
        if (lane == 0) {
            misc[2] = (uint32_t)((slots + 15) / 16);
            atomicAdd(visited, (unsigned long long)((slots + 15) / 16) * (unsigned long long)(BM * BN * nq));
        }
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(misc), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int n_tiles = (int)misc[2];

    // Register split (the host launches only when the kernel was built with
    // kLaunchRegs registers per thread): warpgroup 2 (producer, MMA, two idle
    // warps) drops to kRegsOther, the two softmax warpgroups rise to
    // kRegsSoftmax, which keeps the S row of 128 fp32 values in registers.
    if (warp >= 8) {
        setmaxnreg_dec<kRegsOther>();
        if (warp == 8) {
            // ------------------------------------------------ TMA producer (whole warp)
            // A window of 32 selected K/V groups is held one per lane; a warp
            // prefix sum of their 8-row slot counts places every group in the
            // item's slot sequence.  For each 128-key tile the lanes whose group
            // overlaps it record one run (first row, slot count) and the valid
            // row count of each slot; runs are then issued by their own lanes as
            // the fewest power-of-two boxes.
            const CUtensorMap* tq = (it.a < 0) ? &maps.qp : &maps.q;
            if (lane == 0) {
                prefetch_tmap(tq);
                for (int k = 0; k < NBOX; ++k) {
                    prefetch_tmap(&maps.k[k]);
                    prefetch_tmap(&maps.v[k]);
                }
                const int qrow = (it.a < 0) ? it.bh * Mp + it.row0 : it.bh * N + it.row0;
                mbar_arrive_expect_tx(bar(B_Q), nq * L::QB);
                for (int t = 0; t < nq; ++t)
                    for (int hh = 0; hh < D / 64; ++hh)
                        tma_load_2d(sQ + t * L::QB + hh * BM * 128, tq, bar(B_Q), hh * 64, qrow + t * BM);
            }
            const bool probe = it.a < 0;
            const int kv_head = it.bh / G;   // permuted K/V rows of the K/V head (GQA)
            const int32_t* sg = sel_groups + ((size_t)it.bh * Cq + (probe ? 0 : it.a)) * Ck;
            const int32_t* ko = kv_off + (size_t)it.bh * (Ck + 1);
            const int n_groups = probe ? 1 : sel_count[(size_t)it.bh * Cq + it.a];
            int2* runs = reinterpret_cast<int2*>(sm + L::oRun);
            int gbase = 0, w_begin = 0, w_end = 0, my_rs = 0, my_len = 0, my_sb = 0, my_se = 0;
            auto load_window = [&]() {
                const int g = gbase + lane;
                my_rs = 0;
                my_len = 0;
                if (g < n_groups) {
                    if (probe) {
                        my_len = N;
                    } else {
                        const int b = sg[g];
                        my_rs = ko[b];
                        my_len = ko[b + 1] - my_rs;
                    }
                }
                const int ns = (my_len + 7) >> 3;
                int incl = ns;
    #pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                my_sb = w_begin + incl - ns;
                my_se = w_begin + incl;
                w_end = w_begin + __shfl_sync(0xffffffffu, incl, 31);
            };
            load_window();
            int issued_k = 0, issued_v = 0;
            auto lane0_wait = [&](uint32_t b, uint32_t parity, int where) -> bool {
                int ok = 1;
                if (lane == 0 && !mbar_wait(b, parity, abort_flag, kSpin)) {
                    record_status(status, SPARSEPR_TIMEOUT, where);
                    *abort_flag = 1;
                    ok = 0;
                }
                return __shfl_sync(0xffffffffu, ok, 0) != 0;
            };
            auto issue = [&](uint32_t dst, const CUtensorMap* mp, uint32_t b) {
                if (lane < 16) {
                    const int2 rn = runs[lane];   // (first global row, slots) of a run starting at slot lane
                    int done = 0;
                    while (done < rn.y) {
                        int k = 31 - __clz(rn.y - done);
                        if (k > NBOX - 1) k = NBOX - 1;
                        const int y = (rn.x == total_rows) ? total_rows : rn.x + 8 * done;
                        for (int hh = 0; hh < D / 64; ++hh)
                            tma_load_2d(dst + hh * BN * 128 + (lane + done) * 1024, &mp[k], b, hh * 64, y);
                        done += 1 << k;
                    }
                }
            };
            for (int j = 0; j < n_tiles; ++j) {
                const int stage = j % NS, use = j / NS, ring = j % RING;
                const int T0 = 16 * j;
                if (j >= RING && !lane0_wait(bar(B_ME + ring), ((j / RING) - 1) & 1, 40)) break;
                uint8_t* vm = meta + ring * 16;
                if (lane < 16) {
                    vm[lane] = 0;
                    runs[lane] = make_int2(0, 0);
                }
                __syncwarp();
                while (true) {
                    const int lo = max(my_sb, T0), hi = min(my_se, T0 + 16);
                    if (lo < hi) {
                        const int o = lo - my_sb;
                        runs[lo - T0] = make_int2(kv_head * N + my_rs + 8 * o, hi - lo);
                        for (int t = lo; t < hi; ++t) vm[t - T0] = (uint8_t)min(8, my_len - 8 * (t - my_sb));
                    }
                    if (w_end >= T0 + 16 || gbase + 32 >= n_groups) break;
                    gbase += 32;
                    w_begin = w_end;
                    load_window();
                }
                if (lane == 0 && w_end < T0 + 16) {   // past the last group: zero-filled padding slots
                    const int ps = max(w_end, T0);
                    runs[ps - T0] = make_int2(total_rows, T0 + 16 - ps);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_MF + ring));
                if (j >= NS && !lane0_wait(bar(B_KE + stage), (use - 1) & 1, 41)) break;
                if (lane == 0) mbar_arrive_expect_tx(bar(B_KF + stage), L::KB);
                __syncwarp();
                issue(sK + stage * L::KB, maps.k, bar(B_KF + stage));
                issued_k = j + 1;
                if (j >= NS && !lane0_wait(bar(B_VE + stage), (use - 1) & 1, 42)) break;
                if (lane == 0) mbar_arrive_expect_tx(bar(B_VF + stage), L::KB);
                __syncwarp();
                issue(sV + stage * L::KB, maps.v, bar(B_VF + stage));
                issued_v = j + 1;
                __syncwarp();
            }
            // every copy this CTA issued lands before the CTA can exit (abort or not)
            if (lane == 0) {
                mbar_wait(bar(B_Q), 0, nullptr, kSpin);
                for (int t = max(0, issued_k - NS); t < issued_k; ++t)
                    mbar_wait(bar(B_KF + t % NS), (t / NS) & 1, nullptr, kSpin);
                for (int t = max(0, issued_v - NS); t < issued_v; ++t)
                    mbar_wait(bar(B_VF + t % NS), (t / NS) & 1, nullptr, kSpin);
            }
        } else if (warp == 9) {
            // ------------------------------------------------ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idesc_qk = idesc_f32acc(128, 128, kFmtBF16, false);
                constexpr uint32_t idesc_pv = idesc_f32acc(128, D, kFmtF16, true);
                // Descriptors are built once; every MMA adds a compile-time offset
                // (its start address, >> 4, sits in the low bits and never carries
                // out: shared addresses are below 2^18).  Rebuilding them per MMA
                // costs more issue cycles than the 64 an M=128, N=128, K=16 MMA takes.
                const uint64_t dq = smem_desc(sQ, 16, 1024), dk = smem_desc(sK, 16, 1024);
                const uint64_t dv = smem_desc(sV, BN * 128, 1024);
                auto issue_s = [&](int t, int stage) {
                    const uint64_t a0 = dq + (uint64_t)((t * L::QB) >> 4), b0 = dk + (uint64_t)((stage * L::KB) >> 4);
                    const uint32_t d = tmem + 128 * t;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t off = (uint64_t)((((kk / 4) * BM * 128) + (kk % 4) * 32) >> 4);
                        const uint64_t offb = (uint64_t)((((kk / 4) * BN * 128) + (kk % 4) * 32) >> 4);
                        mma_f16_ss(d, a0 + off, b0 + offb, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                };
                auto issue_pv = [&](int t, int jj) {
                    const uint64_t b0 = dv + (uint64_t)(((jj % NS) * L::KB) >> 4);
                    const uint32_t d = tmem + 256 + D * t, a = tmem + 128 * t;
                    const uint32_t acc0 = jj > 0 ? 1u : 0u;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_f16_ts(d, a + kk * 8, b0 + (uint64_t)((kk * 2048) >> 4), idesc_pv, kk > 0 ? 1u : acc0);
                };
                // Stall hook (testing the timeout path): a bounded wait on a
                // barrier nothing signals runs out before any MMA is issued.
                bool ok = stall_polls == 0 || mbar_wait(bar(B_ST), 0, abort_flag, stall_polls);
                ok = ok && mbar_wait(bar(B_Q), 0, abort_flag, kSpin);
                for (int j = 0; ok && j < n_tiles; ++j) {
                    const int stage = j % NS;
                    if (!mbar_wait(bar(B_KF + stage), (j / NS) & 1, abort_flag, kSpin)) { ok = false; break; }
                    if (j >= 1 && !mbar_wait(bar(B_VF + (j - 1) % NS), ((j - 1) / NS) & 1, abort_flag, kSpin)) { ok = false; break; }
                    for (int t = 0; t < nq; ++t) {
                        if (j >= 1) {
                            if (!mbar_wait(bar(B_PF + t), (j - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                            tc_fence_after();
                            issue_pv(t, j - 1);
                        }
                        tc_fence_after();
                        issue_s(t, stage);
                        mma_commit(bar(B_SF + t));
                    }
                    if (!ok) break;
                    mma_commit(bar(B_KE + stage));
                    if (j >= 1) mma_commit(bar(B_VE + (j - 1) % NS));
                }
                if (ok && n_tiles > 0) {
                    const int jl = n_tiles - 1;
                    if (!mbar_wait(bar(B_VF + jl % NS), (jl / NS) & 1, abort_flag, kSpin)) ok = false;
                    for (int t = 0; ok && t < nq; ++t) {
                        if (!mbar_wait(bar(B_PF + t), jl & 1, abort_flag, kSpin)) { ok = false; break; }
                        tc_fence_after();
                        issue_pv(t, jl);
                    }
                    if (ok) {
                        mma_commit(bar(B_VE + jl % NS));
                        mma_commit(bar(B_OF));
                    }
                }
                if (!ok) {
                    record_status(status, SPARSEPR_TIMEOUT, 43);
                    *abort_flag = 1;
                }
                // every MMA issued above completes before TMEM is released
                mma_commit(bar(B_DR));
                mbar_wait(bar(B_DR), 0, nullptr, kSpin);
            }
        }
    } else {
        setmaxnreg_inc<kRegsSoftmax>();
        if (warp < 4 * nq) {
            // ------------------------------------------------ softmax of Q tile t (rows = TMEM lanes)
            // The whole 128-key row of S is held in registers: one TMEM read, the
            // row maximum, then P = exp2(s * scale - m_ref) as fp16 pairs.
            const int t = warp >> 2, r = tid - 128 * t;
            const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
            const uint32_t tS = t_row + 128 * t, tO = t_row + 256 + D * t;
            float m_ref = -INFINITY;
            float2 l2 = make_float2(0.f, 0.f);
            bool ok = true;
            // Keys past a group's end in a partial 8-key slot, and padding slots,
            // get -inf.  w holds the valid counts of the chunk's four slots; a
            // chunk of full slots (the common case) takes one uniform test.
            auto mask_chunk = [&](float (&v)[32], uint32_t w) {
                if (w != 0x08080808u) {
                    uint32_t valid = 0;
#pragma unroll
                    for (int q = 0; q < 4; ++q) valid |= ((1u << ((w >> (8 * q)) & 0xffu)) - 1u) << (8 * q);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = ((valid >> i) & 1u) ? v[i] : -INFINITY;
                }
            };
            for (int j = 0; j < n_tiles; ++j) {
                const int ring = j % RING;
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SF + t), j & 1, abort_flag, kSpin));
                if (!ok) break;
                tc_fence_after();
                float sv[4][32];
    #pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sv[c]);
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_MF + ring), (j / RING) & 1, abort_flag, kSpin));
                tmem_wait_ld();
                if (!ok) break;
                const uint4 vw = *reinterpret_cast<const uint4*>(meta + ring * 16);
                mbar_arrive(bar(B_ME + ring));
                const uint32_t vwa[4] = {vw.x, vw.y, vw.z, vw.w};
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    #pragma unroll
                for (int c = 0; c < 4; ++c) {
                    mask_chunk(sv[c], vwa[c]);
    #pragma unroll
                    for (int i = 0; i < 16; ++i) mx4[i & 3] = fmax3(mx4[i & 3], sv[c][2 * i], sv[c][2 * i + 1]);
                }
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale_log2;
                const float m_new = fmaxf(m_ref, mx);
                const bool need = (j > 0) && (m_new > m_ref + 8.f);
                if (j == 0) m_ref = m_new;
                if (__any_sync(0xffffffffu, need)) {   // O_t is quiescent: PV_t(j-1) completed before S_t(j)
                    const float alpha = need ? ex2_approx(m_ref - m_new) : 1.f;
                    if (need) {
                        m_ref = m_new;
                        l2.x *= alpha;
                        l2.y *= alpha;
                    }
    #pragma unroll
                    for (int c4 = 0; c4 < D / 32; ++c4) {
                        float v[32];
                        tmem_ld32(tO + c4 * 32, v);
                        tmem_wait_ld(v);
    #pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= alpha;
                        tmem_st32(tO + c4 * 32, v);
                    }
                    tmem_wait_st();
                }
                // P = exp2(s * scale - m_ref) <= 2^8 as fp16, keys 2i and 2i+1 in
                // column i of S's first 64 columns (all of S is already read).
                // kSoftPairs of every 16 pairs, evenly spread, take the FMA-pipe
            // exponential, which relieves the MUFU (two exponentials per pair).
                const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_ref, -m_ref);
                float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
    #pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t w[16];
    #pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 x = ffma2(make_float2(sv[c][2 * i], sv[c][2 * i + 1]), sc2, nm2);
                        float2 pr;
                        if ((i * kSoftPairs) % 16 < kSoftPairs) {
                            pr = exp2_fma2(x);
                        } else {
                            pr.x = ex2_approx(x.x);
                            pr.y = ex2_approx(x.y);
                        }
                        if (i & 1) lb = fadd2(lb, pr);
                        else la = fadd2(la, pr);
                        const __half2 h = __floats2half2_rn(pr.x, pr.y);
                        w[i] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                    tmem_st16(tS + 16 * c, w);
                }
                l2 = fadd2(l2, fadd2(la, lb));
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_PF + t));
            }
            if (ok && n_tiles > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OF), 0, abort_flag, kSpin));
                if (ok) {
                    tc_fence_after();
                    const int nrows = t == 0 ? it.n0 : it.n1;
                    const int row = it.row0 + BM * t + r;
                    float* out = (it.a < 0) ? probe_dense + ((size_t)it.bh * Mp + row) * D
                                            : O_sp + ((size_t)it.bh * N + row) * D;
                    const float inv = vscale[it.bh / G] / (l2.x + l2.y);
    #pragma unroll
                    for (int c4 = 0; c4 < D / 32; ++c4) {
                        float v[32];
                        tmem_ld32(tO + c4 * 32, v);
                        tmem_wait_ld(v);
                        if (r < nrows) {
                            float4* o4 = reinterpret_cast<float4*>(out + c4 * 32);
    #pragma unroll
                            for (int i = 0; i < 8; ++i)
                                o4[i] = make_float4(v[4 * i] * inv, v[4 * i + 1] * inv, v[4 * i + 2] * inv,
                                                    v[4 * i + 3] * inv);
                        }
                    }
                }
            }
            if (!ok) {
                record_status(status, SPARSEPR_TIMEOUT, 44);
                *abort_flag = 1;
            }
            tc_fence_before();
        }
    }
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- V for the tensor-core kernel
// The P V product runs in fp16 (P <= 2^8 keeps 11 mantissa bits).  V is
// copied to fp16 with an exact per-head power-of-two scale that keeps
// |v| <= 2^14; the output is multiplied back by that power of two.
__global__ void vmax_kernel(const __nv_bfloat16* __restrict__ V, size_t per_head, unsigned* __restrict__ vmax) {
    const int bh = blockIdx.y;
    const __nv_bfloat16* v = V + (size_t)bh * per_head;
    float m = 0.f;
    for (size_t e = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; e < per_head;
         e += (size_t)gridDim.x * blockDim.x * 8) {
        float x[8];
        load8(v + e, x);
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
    }
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) atomicMax(&vmax[bh], __float_as_uint(m));
}

__global__ void vconvert_kernel(const __nv_bfloat16* __restrict__ V, size_t per_head, const unsigned* __restrict__ vmax,
                                __half* __restrict__ VH, float* __restrict__ vscale) {
    const int bh = blockIdx.y;
    const float mx = __uint_as_float(vmax[bh]);
    int k = 0;
    if (mx > 16384.f && isfinite(mx)) {
        int e;
        frexpf(mx, &e);
        k = e - 14;
    }
    const float s = ldexpf(1.f, -k);
    if (blockIdx.x == 0 && threadIdx.x == 0) vscale[bh] = ldexpf(1.f, k);
    const __nv_bfloat16* v = V + (size_t)bh * per_head;
    __half* h = VH + (size_t)bh * per_head;
    for (size_t e = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; e < per_head;
         e += (size_t)gridDim.x * blockDim.x * 8) {
        float x[8];
        load8(v + e, x);
        __align__(16) __half2 o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = __floats2half2_rn(x[2 * i] * s, x[2 * i + 1] * s);
        *reinterpret_cast<uint4*>(h + e) = *reinterpret_cast<const uint4*>(o);
    }
}

// ================================================================ host side
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// [rows, d] row-major 16-bit elements, boxes of box_rows rows x 64 channels, 128-byte swizzle.
bool make_rows_map(CUtensorMap* m, const void* base, uint64_t rows, int d, int box_rows, bool fp16) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr || rows == 0) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
              dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The kernel's register split assumes kLaunchRegs registers per thread at
// launch: with fewer, the softmax warpgroups' increase could never be met.
bool tc_register_split_ok(int d) {
    cudaFuncAttributes a;
    const cudaError_t e = d == 128 ? cudaFuncGetAttributes(&a, attention_tc_kernel<128>)
                                   : cudaFuncGetAttributes(&a, attention_tc_kernel<64>);
    if (e != cudaSuccess) {
        cuda_status(e);
        return false;
    }
    if (a.numRegs != tc::kLaunchRegs || a.maxThreadsPerBlock < tc::kThreads) {
        snprintf(last_error_buffer(), 256, "attention_tc_kernel<%d>: built with %d registers per thread, %d expected",
                 d, a.numRegs, tc::kLaunchRegs);
        return false;
    }
    return true;
}

std::atomic<uint32_t> g_stall_polls{0};

inline int grid_for(size_t total, int threads) {
    size_t g = (total + threads - 1) / threads;
    return (int)(g > 148 * 64 ? 148 * 64 : (g == 0 ? 1 : g));
}

}  // namespace

bool attention_uses_tc(const sparsepr_params& p) {
    return p.dtype == SPARSEPR_BF16 && p.block == 128 && (p.d == 64 || p.d == 128) &&
           !(p.flags & SPARSEPR_FLAG_SIMT_ATTENTION);
}

sparsepr_status run_attention(const sparsepr_params& p, const Plan& pl, const sparsepr_partition_out& part,
                              const sparsepr_route_out& r, float* O_sp, float* probe_dense,
                              float* probe_sparse, void* ws, cudaStream_t st) {
    const int BH = pl.BH, N = pl.N, d = pl.d, Mp = pl.Mp;
    int32_t* counter = at<int32_t>(ws, pl.o_work);
    int4* items = at<int4>(ws, pl.o_work + 256);
    void* qprobe = at<void>(ws, pl.o_qprobe);
    DevStatus* status = at<DevStatus>(ws, pl.o_status);
    unsigned long long* visited = at<unsigned long long>(ws, pl.o_work + 8);
    cudaMemsetAsync(counter, 0, 16, st);
    const bool tcore = attention_uses_tc(p);
    count_launch(), build_work_kernel<<<BH, 1024, 0, st>>>(part.q_offsets, part.n_groups, pl.Cq, pl.BM, tcore ? 1 : 0,
                                                           items, counter);
    if (Mp > 0) {
        const int chunks = d * pl.esz / 16;
        if (p.dtype == SPARSEPR_BF16)
            count_launch(), gather_probe_rows_kernel<__nv_bfloat16><<<grid_for((size_t)BH * Mp * chunks, 256), 256, 0, st>>>(
                static_cast<const __nv_bfloat16*>(part.Qp), r.probe_idx, part.pos_q, BH, N, Mp, d,
                static_cast<__nv_bfloat16*>(qprobe));
        else
            count_launch(), gather_probe_rows_kernel<float><<<grid_for((size_t)BH * Mp * chunks, 256), 256, 0, st>>>(
                static_cast<const float*>(part.Qp), r.probe_idx, part.pos_q, BH, N, Mp, d,
                static_cast<float*>(qprobe));
    }
    const int grid = pl.n_probe_items + pl.n_items_max;
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)d);
    if (tcore) {
        const int n_probe2 = Mp > 0 ? BH * ((Mp + 255) / 256) : 0;
        const int grid2 = n_probe2 + pl.n_items_max;
        __half* VH = at<__half>(ws, pl.o_vh);
        unsigned* vmax = at<unsigned>(ws, pl.o_vmax);
        float* vscale = at<float>(ws, pl.o_vscale);
        const size_t per_head = (size_t)N * d;
        const int BHk = BH / pl.G;   // V is per K/V head
        cudaMemsetAsync(vmax, 0, (size_t)BHk * sizeof(unsigned), st);
        const dim3 vgrid((unsigned)std::min<size_t>((per_head / 8 + 255) / 256, 148), BHk);
        count_launch(), vmax_kernel<<<vgrid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(part.Vp), per_head, vmax);
        count_launch(), vconvert_kernel<<<vgrid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(part.Vp), per_head,
                                                              vmax, VH, vscale);
        tc::Maps maps;
        const uint64_t rows = (uint64_t)BH * N, kv_rows = (uint64_t)BHk * N;
        bool ok = true;
        for (int k = 0; k < tc::NBOX; ++k) {
            ok = ok && make_rows_map(&maps.k[k], part.Kp, kv_rows, d, 8 << k, false);
            ok = ok && make_rows_map(&maps.v[k], VH, kv_rows, d, 8 << k, true);
        }
        ok = ok && make_rows_map(&maps.q, part.Qp, rows, d, 128, false);
        if (Mp > 0) ok = ok && make_rows_map(&maps.qp, qprobe, (uint64_t)BH * Mp, d, 128, false);
        else maps.qp = maps.q;
        if (!ok) return SPARSEPR_CUDA_ERROR;
        if (!tc_register_split_ok(d)) return SPARSEPR_UNSUPPORTED;
        if (d == 128) {
            auto k = attention_tc_kernel<128>;
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::Layout<128>::smem);
            count_launch(), k<<<grid2, tc::kThreads, tc::Layout<128>::smem, st>>>(maps, items, counter, n_probe2, N, Mp,
                                                                       pl.Cq, pl.Ck, (int)kv_rows, part.kv_offsets,
                                                                       r.sel_count, r.sel_groups, vscale, O_sp,
                                                                       probe_dense, status, visited, scale_log2,
                                                                       g_stall_polls.load(), pl.G);
        } else {
            auto k = attention_tc_kernel<64>;
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::Layout<64>::smem);
            count_launch(), k<<<grid2, tc::kThreads, tc::Layout<64>::smem, st>>>(maps, items, counter, n_probe2, N, Mp,
                                                                      pl.Cq, pl.Ck, (int)kv_rows, part.kv_offsets,
                                                                      r.sel_count, r.sel_groups, vscale, O_sp,
                                                                      probe_dense, status, visited, scale_log2,
                                                                      g_stall_polls.load(), pl.G);
        }
    } else {
        const int threads = 2 * pl.BM;
#define SPR_SIMT(T, D)                                                                                        \
    count_launch(), attention_simt_kernel<T, D><<<grid, threads, 0, st>>>(                                                    \
        static_cast<const T*>(part.Qp), static_cast<const T*>(part.Kp), static_cast<const T*>(part.Vp),     \
        static_cast<const T*>(qprobe), items, counter, pl.n_probe_items, pl.BM, N, Mp, pl.Cq, pl.Ck,        \
        part.kv_offsets, r.sel_count, r.sel_groups, O_sp, probe_dense, visited, scale_log2, pl.G)
        if (p.dtype == SPARSEPR_BF16) {
            if (d == 128) SPR_SIMT(__nv_bfloat16, 128); else SPR_SIMT(__nv_bfloat16, 64);
        } else {
            if (d == 128) SPR_SIMT(float, 128); else SPR_SIMT(float, 64);
        }
#undef SPR_SIMT
    }
    if (Mp > 0) {
        const int chunks = d * 4 / 16;
        count_launch(), gather_probe_rows_kernel<float><<<grid_for((size_t)BH * Mp * chunks, 256), 256, 0, st>>>(
            O_sp, r.probe_idx, part.pos_q, BH, N, Mp, d, probe_sparse);
    }
    return cuda_status(cudaGetLastError());
}

}  // namespace spr

extern "C" void sparsepr_debug_stall_attention(uint32_t polls) { spr::g_stall_polls.store(polls); }
