// Corrected output on the tensor cores ("Partition the Support, Reconstruct
// the Residual", §4.2): for every permuted query row p of a head,
//   O_out[perm_q[p]] = O^dense of the probe        if p is a probe row,
//                    = O^sp_p + mu_R + Xbar_p B     otherwise,
// with Xbar_p = (O^sp_p - mu_X) / sigma.
//
// Xbar B is a dense (128-row tile) x (d x d) product per head, run as
// tcgen05 kind::tf32 MMAs with a three-term split (Xh Bh + Xh Bl + Xl Bh,
// hi = TF32 rounding, lo = TF32 rounding of the remainder), which keeps it at
// fp32 accuracy.  Persistent blocks walk a contiguous range of 128-row tiles,
// so B is staged (transposed and split, 128-byte swizzled) once per head.
//   warps 0-3: read O^sp 32 columns at a time, standardise, split, store to
//              shared memory in the MMA's K-major swizzled layout (2 buffers)
//   warps 4-7: epilogue, one TMEM lane quadrant each (one row per thread)
//   warp 8:    MMA issuer (accumulators double-buffered in TMEM)
// All waits are bounded; a timeout records SPARSEPR_TIMEOUT.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace spr {
namespace aptc {
constexpr int BM = 128;                 // rows per tile (TMEM lanes)
constexpr int kThreads = 288;
constexpr uint32_t kSpin = 1u << 20;
enum { B_AF = 0, B_AE = 2, B_DF = 4, B_DE = 6, B_BF = 8, B_BE = 9, B_DR = 10, N_BAR = 11 };

template <int D>
struct Layout {
    static constexpr int NCH = D / 32;                  // 32-float (128-byte) K chunks
    static constexpr int CHB = D * 128;                 // one chunk of B^T: D rows x 128 B
    static constexpr int oBh = 0;                       // B^T hi, NCH chunks
    static constexpr int oBl = oBh + NCH * CHB;         // B^T lo
    static constexpr int ACH = BM * 128;                // one chunk of A: 128 rows x 128 B
    static constexpr int oA = oBl + NCH * CHB;          // 2 buffers x (hi, lo)
    static constexpr int oBar = oA + 2 * 2 * ACH;
    static constexpr int oMisc = oBar + N_BAR * 8;
    static constexpr int smem = oMisc + 16 + 1024;      // slack for 1024-byte alignment
    static_assert(oA % 1024 == 0 && oBl % 1024 == 0, "swizzled operands need 1024-byte alignment");
};

// Byte offset of element (row, k) of a [rows x 32] fp32 chunk in the
// 128-byte swizzled K-major layout (16-byte unit index XOR row % 8).
__device__ __forceinline__ uint32_t sw128(int row, int k) {
    return (uint32_t)(row * 128 + ((((k >> 2) ^ row) & 7) << 4) + (k & 3) * 4);
}
}  // namespace aptc

// Tiles are numbered head-major; block b takes tiles [b T / G, (b+1) T / G).
// Nine warps: the SM sub-partitions holding three of them leave 16384 / 96
// registers a lane, so the kernel is capped at 168.
template <int D>
__global__ void __maxnreg__(168) apply_tc_kernel(
    const float* __restrict__ O_sp, const float* __restrict__ Bm, const float* __restrict__ mu_x,
    const float* __restrict__ sigma, const float* __restrict__ mu_r, const int32_t* __restrict__ pslot,
    const float* __restrict__ probe_dense, const int32_t* __restrict__ perm_q, int BH, int N, int Mp,
    float* __restrict__ O_out, DevStatus* status) {
    using namespace aptc;
    using namespace sm100;
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    if (*reinterpret_cast<volatile const int32_t*>(&status->code) != 0) return;
    const int tiles_per_head = (N + BM - 1) / BM;
    const long long total = (long long)BH * tiles_per_head;
    const int w_begin = (int)(total * blockIdx.x / gridDim.x), w_end = (int)(total * (blockIdx.x + 1) / gridDim.x);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t s_base = smem_u32(sm);
    auto bar = [&](int i) -> uint32_t { return s_base + L::oBar + 8 * i; };
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + L::oMisc);   // [0] tmem, [1] abort
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_AF + s), 128);
            mbar_init(bar(B_AE + s), 1);
            mbar_init(bar(B_DF + s), 1);
            mbar_init(bar(B_DE + s), 128);
        }
        mbar_init(bar(B_BF), 128);
        mbar_init(bar(B_BE), 1);
        mbar_init(bar(B_DR), 1);
        fence_barrier_init();
        misc[1] = 0;
    }
    if (warp == 8) {
        tmem_alloc(smem_u32(misc), 2 * D);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp < 4) {
        // ------------------------------------------------ operand producers (128 threads)
        // Steps are (tile, 32-column chunk) pairs.  The raw values of step s + 1
        // are loaded while step s is standardised, split and stored.
        bool ok = true;
        int heads = 0, cur_bh = -1;
        const int steps = (w_end - w_begin) * L::NCH;
        auto load_step = [&](int st, float (&xv)[32]) {
            const int w = w_begin + st / L::NCH, c = st % L::NCH;
            const int bh = w / tiles_per_head, p0 = (w % tiles_per_head) * BM + warp * 32;
            const float* col = O_sp + ((size_t)bh * N + p0) * D + 32 * c + lane;
#pragma unroll
            for (int i = 0; i < 32; ++i) xv[i] = (p0 + i < N) ? col[(size_t)i * D] : 0.f;
        };
        auto store_step = [&](int st, const float (&xv)[32]) -> bool {
            const int w = w_begin + st / L::NCH, c = st % L::NCH, b = st & 1;
            const int bh = w / tiles_per_head, p0 = (w % tiles_per_head) * BM + warp * 32;
            if (bh != cur_bh) {
                // B^T of this head, split: element (n, k) = B[k][n]; the previous
                // head's MMAs must have finished reading the old copy
                if (heads > 0 && !mbar_wait(bar(B_BE), (heads - 1) & 1, abort_flag, kSpin)) return false;
                const float* Bh = Bm + (size_t)bh * D * D;
                for (int e = tid; e < D * D; e += 128) {
                    const int k = e / D, n = e % D;   // coalesced over n
                    const float v = Bh[e];
                    const float hi = tf32_round(v), lo = tf32_round(v - hi);
                    const uint32_t off = (uint32_t)((k >> 5) * L::CHB) + sw128(n, k & 31);
                    *reinterpret_cast<float*>(sm + L::oBh + off) = hi;
                    *reinterpret_cast<float*>(sm + L::oBl + off) = lo;
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(B_BF));
                cur_bh = bh;
                ++heads;
            }
            if (st >= 2 && !mbar_wait(bar(B_AE + b), ((st >> 1) - 1) & 1, abort_flag, kSpin)) return false;
            const int k = 32 * c + lane;   // this lane's column
            const float mx = mu_x[(size_t)bh * D + k], inv_s = 1.f / sigma[(size_t)bh * D + k];
            uint8_t* ah = sm + L::oA + (2 * b) * L::ACH;
            uint8_t* al = ah + L::ACH;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float x = (p0 + i < N) ? (xv[i] - mx) * inv_s : 0.f;
                const float hi = tf32_round(x), lo = tf32_round(x - hi);
                *reinterpret_cast<float*>(ah + sw128(warp * 32 + i, lane)) = hi;
                *reinterpret_cast<float*>(al + sw128(warp * 32 + i, lane)) = lo;
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(B_AF + b));
            return true;
        };
        float xa[32], xb[32];
        if (steps > 0) load_step(0, xa);
        for (int st = 0; st < steps; st += 2) {
            if (st + 1 < steps) load_step(st + 1, xb);
            if (!store_step(st, xa)) { ok = false; break; }
            if (st + 1 >= steps) break;
            if (st + 2 < steps) load_step(st + 2, xa);
            if (!store_step(st + 1, xb)) { ok = false; break; }
        }
        if (!ok) {
            record_status(status, SPARSEPR_TIMEOUT, 70);
            *abort_flag = 1;
        }
    } else if (warp < 8) {
        // ------------------------------------------------ epilogue: one row per thread
        const int quad = warp - 4, m = quad * 32 + lane;
        const uint32_t t_row = tmem + ((uint32_t)(quad * 32) << 16);
        bool ok = true;
        int i = 0;
        for (int w = w_begin; ok && w < w_end; ++w, ++i) {
            const int bh = w / tiles_per_head, p = (w % tiles_per_head) * BM + m;
            const int d = i & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DF + d), (i >> 1) & 1, abort_flag, kSpin));
            if (!ok) break;
            tc_fence_after();
            const bool live = p < N;
            const size_t src = (size_t)bh * N + (live ? p : 0);
            const int slot = live ? pslot[src] : -1;
            float4* dst = reinterpret_cast<float4*>(O_out + ((size_t)bh * N + (live ? perm_q[src] : 0)) * D);
            // columns in halves of 64 (two TMEM loads) to bound the live registers
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh) {
                float acc[2][32];
                tmem_ld32(t_row + d * D + 64 * hh, acc[0]);
                tmem_ld32(t_row + d * D + 64 * hh + 32, acc[1]);
                tmem_wait_ld(acc[0]);
                tmem_wait_ld(acc[1]);
                if (live && slot < 0) {
                    const float4* x = reinterpret_cast<const float4*>(O_sp + src * D) + 16 * hh;
                    const float4* mr = reinterpret_cast<const float4*>(mu_r + (size_t)bh * D) + 16 * hh;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float4 a = x[q], r = mr[q];
                        const float* v = &acc[q / 8][(q % 8) * 4];
                        dst[16 * hh + q] =
                            make_float4(a.x + r.x + v[0], a.y + r.y + v[1], a.z + r.z + v[2], a.w + r.w + v[3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bar(B_DE + d));   // the accumulator is free for tile i + 2
            if (live && slot >= 0) {      // probe rows keep their exact output
                const float4* pd = reinterpret_cast<const float4*>(probe_dense + ((size_t)bh * Mp + slot) * D);
#pragma unroll 8
                for (int q = 0; q < D / 4; ++q) dst[q] = pd[q];
            }
        }
        if (!ok) {
            record_status(status, SPARSEPR_TIMEOUT, 71);
            *abort_flag = 1;
        }
    } else if (lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_f32acc(BM, D, kFmtTF32, false);
        bool ok = true;
        int g = 0, heads = 0, cur_bh = -1, i = 0;
        for (int w = w_begin; ok && w < w_end; ++w, ++i) {
            const int bh = w / tiles_per_head;
            if (bh != cur_bh) {
                if (!mbar_wait(bar(B_BF), heads & 1, abort_flag, kSpin)) { ok = false; break; }
                cur_bh = bh;
                ++heads;
            }
            const int d = i & 1;
            if (i >= 2 && !mbar_wait(bar(B_DE + d), ((i >> 1) - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
            for (int c = 0; c < L::NCH; ++c, ++g) {
                const int b = g & 1;
                if (!mbar_wait(bar(B_AF + b), (g >> 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ah = s_base + L::oA + (2 * b) * L::ACH, al = ah + L::ACH;
                const uint32_t bhi = s_base + L::oBh + c * L::CHB, blo = s_base + L::oBl + c * L::CHB;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {   // K = 8 per instruction, 32-byte steps inside the 128-byte rows
                    const uint64_t a_hi = smem_desc(ah + kk * 32, 16, 1024), a_lo = smem_desc(al + kk * 32, 16, 1024);
                    const uint64_t b_hi = smem_desc(bhi + kk * 32, 16, 1024), b_lo = smem_desc(blo + kk * 32, 16, 1024);
                    const uint32_t dst = tmem + d * D;
                    mma_tf32_ss(dst, a_hi, b_hi, idesc, (c > 0 || kk > 0) ? 1u : 0u);
                    mma_tf32_ss(dst, a_hi, b_lo, idesc, 1u);
                    mma_tf32_ss(dst, a_lo, b_hi, idesc, 1u);
                }
                mma_commit(bar(B_AE + b));
            }
            if (!ok) break;
            mma_commit(bar(B_DF + d));
            // the last tile of a head releases B for the next head's staging
            if (w + 1 == w_end || (w + 1) / tiles_per_head != bh) mma_commit(bar(B_BE));
        }
        if (!ok) {
            record_status(status, SPARSEPR_TIMEOUT, 72);
            *abort_flag = 1;
        }
        // every MMA issued above completes before TMEM is released
        mma_commit(bar(B_DR));
        mbar_wait(bar(B_DR), 0, nullptr, kSpin);
    }
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * D);
    }
}

// ---------------------------------------------------------------- transposed form (d = 128)
// The same output computed as D^T = B'^T Xbar^T with B' = B + diag(sigma), so
//   O_out[perm_q[p]] = (mu_X + mu_R) + (Xbar B')_p
// (Xbar sigma + mu_X gives back O^sp).  B'^T, split into TF32 hi and lo, sits
// in TMEM as the MMA's A operand (lanes = output channels); each 128-row tile
// of O^sp streams in once through a TMA ring of 32-channel chunks, which the
// transform warps standardise and split in place (hi) and beside it (lo); the
// accumulator holds one output channel per lane and one tile row per column,
// so every warp of the epilogue writes a row's 32 channels as one coalesced
// 128-byte store.
//   warp 0: TMA producer; warp 1: MMA issuer; warps 2-5: transform (one tile
//   row each); warps 6-13: epilogue (channels = TMEM lane quadrant, rows =
//   half of the tile) and the per-head staging of B'^T.
// TMEM: B'^T hi [0,128), lo [128,256); accumulators [256,384), [384,512).
namespace aptt {
constexpr int D = 128, BM = 128, NCH = 4, NST = 4;
constexpr int kThreads = 448;
// each SM sub-partition holds 16384 registers and takes every fourth warp of
// the block: ceil(14 / 4) = 4 warps of 32 threads at kRegs registers must fit
constexpr int kRegs = 128;
static_assert((kThreads / 32 + 3) / 4 * 32 * kRegs <= 16384, "registers per sub-partition");
constexpr uint32_t kSpin = 1u << 20;
enum { B_RF = 0, B_XF = NST, B_XE = 2 * NST, B_DF = 3 * NST, B_DE = 3 * NST + 2, B_AF = 3 * NST + 4,
       B_AE = 3 * NST + 5, B_DR = 3 * NST + 6, B_SS = 3 * NST + 7, B_OF = 3 * NST + 9, B_OE = 3 * NST + 11,
       N_BAR = 3 * NST + 13 };
constexpr int CHB = BM * 128;                 // one chunk: 128 rows x 32 fp32
constexpr int oHi = 0;                        // NST chunks: raw O^sp, then Xbar hi in place
constexpr int oLo = oHi + NST * CHB;          // NST chunks: Xbar lo
constexpr int oStat = oLo + NST * CHB;        // 2 x (mu_X, 1 / sigma) of the last two heads (transform warps)
constexpr int oOut = oStat + 2 * 2 * D * 4;    // 2 row halves x 64 rows x 128 fp32: the restored rows
constexpr int oBar = oOut + 2 * 64 * D * 4;
constexpr int oMisc = oBar + N_BAR * 8;
constexpr int kSmem = oMisc + 16 + 1024;
static_assert(oLo % 1024 == 0 && oStat % 16 == 0 && oOut % 16 == 0, "alignment");
static_assert(kSmem <= 232448, "shared memory");
}  // namespace aptt

__global__ void __maxnreg__(aptt::kRegs) apply_t_kernel(
    const __grid_constant__ CUtensorMap osp_map, const float* __restrict__ Bm, const float* __restrict__ mu_x,
    const float* __restrict__ sigma, const float* __restrict__ mu_r, const int32_t* __restrict__ pslot,
    const float* __restrict__ probe_dense, const int32_t* __restrict__ perm_q, int BH, int N, int Mp,
    float* __restrict__ O_out, DevStatus* status) {
    using namespace aptt;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    if (*reinterpret_cast<volatile const int32_t*>(&status->code) != 0) return;
    const int tiles_per_head = (N + BM - 1) / BM;
    const long long total = (long long)BH * tiles_per_head;
    const int w_begin = (int)(total * blockIdx.x / gridDim.x), w_end = (int)(total * (blockIdx.x + 1) / gridDim.x);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t s_base = smem_u32(sm);
    auto bar = [&](int i) -> uint32_t { return s_base + oBar + 8 * i; };
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + oMisc);   // [0] tmem, [1] abort
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(bar(B_RF + s), 1);
            mbar_init(bar(B_XF + s), 128);
            mbar_init(bar(B_XE + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_DF + s), 1);
            mbar_init(bar(B_DE + s), 256);
        }
        mbar_init(bar(B_AF), 256);
        mbar_init(bar(B_AE), 1);
        mbar_init(bar(B_DR), 1);
        mbar_init(bar(B_SS), 128);
        mbar_init(bar(B_SS + 1), 128);
        for (int h = 0; h < 2; ++h) {
            mbar_init(bar(B_OF + h), 4);   // the four channel warps of a row half staged their columns
            mbar_init(bar(B_OE + h), 4);   // ... and wrote their rows out
        }
        fence_barrier_init();
        misc[1] = 0;
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(misc), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer: raw O^sp chunks
            prefetch_tmap(&osp_map);
            bool ok = true;
            int g = 0;
            for (int w = w_begin; ok && w < w_end; ++w) {
                const int bh = w / tiles_per_head, p0 = (w % tiles_per_head) * BM;
                for (int c = 0; c < NCH; ++c, ++g) {
                    const int s = g % NST;
                    if (g >= NST && !mbar_wait(bar(B_XE + s), ((g / NST) - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                    mbar_arrive_expect_tx(bar(B_RF + s), CHB);
                    tma_load_2d(s_base + oHi + s * CHB, &osp_map, bar(B_RF + s), 32 * c, bh * N + p0);
                }
            }
            if (!ok) {
                record_status(status, SPARSEPR_TIMEOUT, 73);
                *abort_flag = 1;
            }
            // every copy issued above lands before the CTA can exit
            for (int t = max(0, g - NST); t < g; ++t) mbar_wait(bar(B_RF + t % NST), (t / NST) & 1, nullptr, kSpin);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = idesc_f32acc(128, BM, kFmtTF32, false);
            const uint64_t dHi = smem_desc(s_base + oHi, 16, 1024), dLo = smem_desc(s_base + oLo, 16, 1024);
            bool ok = true;
            int g = 0, heads = 0, cur_bh = -1, i = 0;
            for (int w = w_begin; ok && w < w_end; ++w, ++i) {
                const int bh = w / tiles_per_head;
                if (bh != cur_bh) {
                    if (!mbar_wait(bar(B_AF), heads & 1, abort_flag, kSpin)) { ok = false; break; }
                    cur_bh = bh;
                    ++heads;
                }
                const int d = i & 1;
                if (i >= 2 && !mbar_wait(bar(B_DE + d), ((i >> 1) - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                const uint32_t acc = tmem + 256 + BM * d;
                for (int c = 0; c < NCH; ++c, ++g) {
                    const int s = g % NST;
                    if (!mbar_wait(bar(B_XF + s), (g / NST) & 1, abort_flag, kSpin)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t bh_d = dHi + (uint64_t)((s * CHB) >> 4), bl_d = dLo + (uint64_t)((s * CHB) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {   // K = 8 per instruction, 32-byte steps inside the 128-byte rows
                        const uint32_t ahi = tmem + 32 * c + 8 * kk, alo = tmem + 128 + 32 * c + 8 * kk;
                        const uint64_t bo = (uint64_t)((kk * 32) >> 4);
                        mma_tf32_ts(acc, ahi, bh_d + bo, idesc, (c > 0 || kk > 0) ? 1u : 0u);
                        mma_tf32_ts(acc, ahi, bl_d + bo, idesc, 1u);
                        mma_tf32_ts(acc, alo, bh_d + bo, idesc, 1u);
                    }
                    mma_commit(bar(B_XE + s));
                }
                if (!ok) break;
                mma_commit(bar(B_DF + d));
                // the last tile of a head releases B'^T for the next head's staging
                if (w + 1 == w_end || (w + 1) / tiles_per_head != bh) mma_commit(bar(B_AE));
            }
            if (!ok) {
                record_status(status, SPARSEPR_TIMEOUT, 74);
                *abort_flag = 1;
            }
            mma_commit(bar(B_DR));
            mbar_wait(bar(B_DR), 0, nullptr, kSpin);
        }
    } else if (warp < 6) {
        // ------------------------------------------------ transform: Xbar = (O^sp - mu_X) / sigma, hi and lo
        const int t = tid - 64;   // tile row
        float* stat = nullptr;
        bool ok = true;
        int g = 0, cur_bh = -1, heads = 0;
        for (int w = w_begin; ok && w < w_end; ++w) {
            const int bh = w / tiles_per_head, p0 = (w % tiles_per_head) * BM;
            if (bh != cur_bh) {
                // the head's mu_X and 1 / sigma, in the buffer of its parity: the
                // other buffer may still be read by a thread on the previous head;
                // this one was last read for head - 2, which every thread left
                // before it passed the previous head's exchange
                const int hp = heads & 1;
                stat = reinterpret_cast<float*>(sm + oStat) + hp * 2 * D;
                stat[t] = mu_x[(size_t)bh * D + t];
                stat[D + t] = 1.f / sigma[(size_t)bh * D + t];
                mbar_arrive(bar(B_SS + hp));
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SS + hp), (heads >> 1) & 1, abort_flag, kSpin));
                if (!ok) break;
                cur_bh = bh;
                ++heads;
            }
            const bool live = p0 + t < N;
            for (int c = 0; c < NCH; ++c, ++g) {
                const int s = g % NST;
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_RF + s), (g / NST) & 1, abort_flag, kSpin));
                if (!ok) break;
                uint8_t* hi = sm + oHi + s * CHB + t * 128;
                uint8_t* lo = sm + oLo + s * CHB + t * 128;
                const float4* m4 = reinterpret_cast<const float4*>(stat) + 8 * c;
                const float4* i4 = reinterpret_cast<const float4*>(stat + D) + 8 * c;
#pragma unroll
                for (int u = 0; u < 8; ++u) {   // 16-byte unit u of the row sits at (u ^ row % 8) (128-byte swizzle)
                    const int pu = (u ^ t) & 7;
                    float4 x = *reinterpret_cast<const float4*>(hi + pu * 16);
                    const float4 m = m4[u], iv = i4[u];
                    x.x = live ? (x.x - m.x) * iv.x : 0.f;
                    x.y = live ? (x.y - m.y) * iv.y : 0.f;
                    x.z = live ? (x.z - m.z) * iv.z : 0.f;
                    x.w = live ? (x.w - m.w) * iv.w : 0.f;
                    const float4 h = make_float4(tf32_round(x.x), tf32_round(x.y), tf32_round(x.z), tf32_round(x.w));
                    *reinterpret_cast<float4*>(hi + pu * 16) = h;
                    *reinterpret_cast<float4*>(lo + pu * 16) =
                        make_float4(tf32_round(x.x - h.x), tf32_round(x.y - h.y), tf32_round(x.z - h.z),
                                    tf32_round(x.w - h.w));
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(B_XF + s));
            }
        }
        if (!ok) {
            record_status(status, SPARSEPR_TIMEOUT, 75);
            *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------ epilogue (and B'^T staging)
        const int q = warp & 3, hrow = (warp - 6) >> 2;   // lane quadrant = output channels, half of the tile rows
        const int n = q * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
        bool ok = true;
        int heads = 0, cur_bh = -1, i = 0;
        float4 bias4 = make_float4(0.f, 0.f, 0.f, 0.f);   // mu_X + mu_R of channels 4 lane .. 4 lane + 3
        // The four channel warps of a row half stage their 32 channels of its 64
        // rows in shared memory; then each writes 16 whole rows (512 bytes, one
        // 16-byte vector per lane) to their restored positions.  Row indices
        // (probe slot, destination) of this warp's 16 rows: lane l holds row
        // 16 q + (l & 15) of the half; loaded one tile ahead.
        float* out_s = reinterpret_cast<float*>(sm + oOut) + hrow * 64 * D;
        auto load_rows = [&](int w, int& sl, int& dq) {
            const int bhw = w / tiles_per_head, r = (w % tiles_per_head) * BM + 64 * hrow + 16 * q + (lane & 15);
            const size_t hb = (size_t)bhw * N;
            sl = r < N ? pslot[hb + r] : -2;
            dq = r < N ? perm_q[hb + r] : 0;
        };
        int nsl = -2, ndq = 0;
        if (w_begin < w_end) load_rows(w_begin, nsl, ndq);
        for (int w = w_begin; ok && w < w_end; ++w, ++i) {
            const int bh = w / tiles_per_head;
            if (bh != cur_bh) {
                // B'^T of this head into TMEM, once the previous head's MMAs are done:
                // lane n, column k holds B[k][n] (+ sigma[n] on the diagonal), hi and lo
                if (heads > 0) {
                    ok = __all_sync(0xffffffffu, mbar_wait(bar(B_AE), (heads - 1) & 1, abort_flag, kSpin));
                    if (!ok) break;
                    tc_fence_after();
                }
                const float* Bh = Bm + (size_t)bh * D * D;
                const float sg = sigma[(size_t)bh * D + n];
                for (int c2 = 0; c2 < 4; ++c2) {   // 32 columns at a time: hi (c2 even), then lo
                    const int k0 = 64 * hrow + 32 * (c2 >> 1);
                    float vb[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int k = k0 + e;
                        const float b = Bh[(size_t)k * D + n] + (k == n ? sg : 0.f);
                        const float h = tf32_round(b);
                        vb[e] = (c2 & 1) ? tf32_round(b - h) : h;
                    }
                    tmem_st32(t_lane + 128 * (c2 & 1) + k0, vb);
                    tmem_wait_st();
                }
                tc_fence_before();
                mbar_arrive(bar(B_AF));
                const float4 mx = reinterpret_cast<const float4*>(mu_x + (size_t)bh * D)[lane];
                const float4 mr = reinterpret_cast<const float4*>(mu_r + (size_t)bh * D)[lane];
                bias4 = make_float4(mx.x + mr.x, mx.y + mr.y, mx.z + mr.z, mx.w + mr.w);
                cur_bh = bh;
                ++heads;
            }
            const int d = i & 1;
            const size_t hb = (size_t)bh * N;
            const int sl = nsl, dq = ndq;
            if (w + 1 < w_end) load_rows(w + 1, nsl, ndq);
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DF + d), (i >> 1) & 1, abort_flag, kSpin));
            if (!ok) break;
            tc_fence_after();
            float v[2][32];
            tmem_ld32(t_lane + 256 + BM * d + 64 * hrow, v[0]);
            tmem_ld32(t_lane + 256 + BM * d + 64 * hrow + 32, v[1]);
            tmem_wait_ld(v[0]);
            tmem_wait_ld(v[1]);
            tc_fence_before();
            mbar_arrive(bar(B_DE + d));   // the accumulator is free for tile i + 2
            // the staging half is free once its rows of the previous tile are written out
            if (i >= 1) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OE + hrow), (i - 1) & 1, abort_flag, kSpin));
                if (!ok) break;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int j = 0; j < 32; ++j) out_s[(32 * h + j) * D + n] = v[h][j];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_OF + hrow));
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OF + hrow), i & 1, abort_flag, kSpin));
            if (!ok) break;
#pragma unroll 4
            for (int r = 0; r < 16; ++r) {
                const int slot = __shfl_sync(0xffffffffu, sl, r);   // uniform: the warp writes one row
                const int dst = __shfl_sync(0xffffffffu, dq, r);
                if (slot == -2) continue;                            // past the head's last row
                float4 x;
                if (slot < 0) {
                    x = reinterpret_cast<const float4*>(out_s + (16 * q + r) * D)[lane];
                    x.x += bias4.x;
                    x.y += bias4.y;
                    x.z += bias4.z;
                    x.w += bias4.w;
                } else {
                    x = reinterpret_cast<const float4*>(probe_dense + ((size_t)bh * Mp + slot) * D)[lane];
                }
                reinterpret_cast<float4*>(O_out + (hb + dst) * D)[lane] = x;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_OE + hrow));
        }
        if (!ok) {
            record_status(status, SPARSEPR_TIMEOUT, 76);
            *abort_flag = 1;
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// O_out[perm_q[p]] = O^sp[p]: the output of a call without probes (one warp per row).
__global__ void unpermute_rows_kernel(const float* __restrict__ O_sp, const int32_t* __restrict__ perm_q, int BH,
                                      int N, int d, float* __restrict__ O_out) {
    const size_t rows = (size_t)BH * N;
    const int lane = threadIdx.x & 31, n4 = d / 4;
    for (size_t r = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5; r < rows;
         r += ((size_t)gridDim.x * blockDim.x) >> 5) {
        const size_t bh = r / N;
        const float4* src = reinterpret_cast<const float4*>(O_sp + r * d);
        float4* dst = reinterpret_cast<float4*>(O_out + (bh * N + perm_q[r]) * d);
        for (int c = lane; c < n4; c += 32) dst[c] = src[c];
    }
}

bool launch_apply_tc(const Plan& pl, const sparsepr_partition_out& part, const float* O_sp, const float* probe_dense,
                     const sparsepr_fit_out& f, const int32_t* pslot, float* O_out, DevStatus* status,
                     cudaStream_t st) {
    const int d = pl.d;
    if (d != 64 && d != 128) return false;
    const long long tiles = (long long)pl.BH * ((pl.N + aptc::BM - 1) / aptc::BM);
    const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
    if (grid == 0) return true;
    if (pl.Mp == 0) {   // no probes, no correction: the sparse output restored to the original order, bit for bit
        const size_t rows = (size_t)pl.BH * pl.N;
        const int g = (int)((rows * 32 + 255) / 256 < (size_t)sm_count() * 16 ? (rows * 32 + 255) / 256
                                                                                 : (size_t)sm_count() * 16);
        count_launch(), unpermute_rows_kernel<<<g, 256, 0, st>>>(O_sp, part.perm_q, pl.BH, pl.N, d, O_out);
        return true;
    }
    if (d == 128) {
        CUtensorMap m;
        if (!encode_rows_map(&m, O_sp, (uint64_t)pl.BH * pl.N, 128, 4, true, 32, aptt::BM)) return false;
        cudaFuncSetAttribute(apply_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, aptt::kSmem);
        count_launch(), apply_t_kernel<<<grid, aptt::kThreads, aptt::kSmem, st>>>(
            m, f.B, f.mu_x, f.sigma, f.mu_r, pslot, probe_dense, part.perm_q, pl.BH, pl.N, pl.Mp, O_out, status);
        return true;
    }
    if (d == 128) {
        auto k = apply_tc_kernel<128>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, aptc::Layout<128>::smem);
        count_launch(), k<<<grid, aptc::kThreads, aptc::Layout<128>::smem, st>>>(
            O_sp, f.B, f.mu_x, f.sigma, f.mu_r, pslot, probe_dense, part.perm_q, pl.BH, pl.N, pl.Mp, O_out, status);
    } else {
        auto k = apply_tc_kernel<64>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, aptc::Layout<64>::smem);
        count_launch(), k<<<grid, aptc::kThreads, aptc::Layout<64>::smem, st>>>(
            O_sp, f.B, f.mu_x, f.sigma, f.mu_r, pslot, probe_dense, part.perm_q, pl.BH, pl.N, pl.Mp, O_out, status);
    }
    return true;
}

}  // namespace spr
