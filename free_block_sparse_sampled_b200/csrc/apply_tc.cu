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

bool launch_apply_tc(const Plan& pl, const sparsepr_partition_out& part, const float* O_sp, const float* probe_dense,
                     const sparsepr_fit_out& f, const int32_t* pslot, float* O_out, DevStatus* status,
                     cudaStream_t st) {
    const int d = pl.d;
    if (d != 64 && d != 128) return false;
    const long long tiles = (long long)pl.BH * ((pl.N + aptc::BM - 1) / aptc::BM);
    const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
    if (grid == 0) return true;
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
