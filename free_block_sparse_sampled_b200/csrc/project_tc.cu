// Coordinates phi = X F on the tensor cores ("Partition the Support,
// Reconstruct the Residual", §4.1 phi_K = K F_K, B.2 phi_Q = RMSNorm(q F_Q)).
//
// X is bf16 [N, d] per head and F fp32 [d, R].  F is split into three bf16
// pieces (F = F0 + F1 + F2, each the bf16 rounding of what is left), so the
// three bf16 x bf16 tcgen05 products, which are exact, accumulate in fp32 to
// the value of an fp32 product.  Persistent blocks walk a contiguous range of
// 128-row tiles; F is staged (transposed, 128-byte swizzled) once per head.
//   warp 0: TMA producer of X tiles (two buffers)
//   warp 1: MMA issuer (accumulators double-buffered in TMEM)
//   warps 2-5: epilogue, one TMEM lane quadrant each (one row per thread):
//              optional RMS normalisation, TF32 rounding, store; they also
//              stage F when the head changes
// All waits are bounded; a timeout records SPARSEPR_TIMEOUT.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace spr {
namespace prtc {
constexpr int BM = 128, D = 128;        // rows per tile, head dimension
constexpr int kThreads = 192;
constexpr uint32_t kSpin = 1u << 20;
enum { B_AF = 0, B_AE = 2, B_DF = 4, B_DE = 6, B_FF = 8, B_FE = 9, B_DR = 10, N_BAR = 11 };

template <int R>
struct Layout {
    static constexpr int AB = BM * D * 2;               // one X tile: 2 chunks of 128 rows x 128 B
    static constexpr int FB = R * D * 2;                // one F piece (transposed): 2 chunks of R rows x 128 B
    static constexpr int oA = 0;                        // 2 buffers
    static constexpr int oF = oA + 2 * AB;              // 3 pieces
    static constexpr int oBar = oF + 3 * FB;
    static constexpr int oMisc = oBar + N_BAR * 8;
    static constexpr int smem = oMisc + 16 + 1024;
    static_assert(oF % 1024 == 0 && FB % 1024 == 0, "swizzled operands need 1024-byte alignment");
};

// Byte offset of bf16 element (row, k), k < 64, of a [rows x 64] chunk in the
// 128-byte swizzled K-major layout (16-byte unit index XOR row % 8).
__device__ __forceinline__ uint32_t sw128_h(int row, int k) {
    return (uint32_t)(row * 128 + ((((k >> 3) ^ row) & 7) << 4) + (k & 7) * 2);
}
}  // namespace prtc

template <int R, bool RMS>
__global__ void __launch_bounds__(prtc::kThreads, 1) project_tc_kernel(
    const __grid_constant__ CUtensorMap xmap, const float* __restrict__ F, int BH, int N,
    const int32_t* __restrict__ r_eff, float eps, float* __restrict__ phi, DevStatus* status) {
    using namespace prtc;
    using namespace sm100;
    using L = Layout<R>;
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
    constexpr uint32_t kCols = R <= 16 ? 32 : (R <= 32 ? 64 : 128);   // 2 accumulators, power of two >= 32

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_AF + s), 1);
            mbar_init(bar(B_AE + s), 1);
            mbar_init(bar(B_DF + s), 1);
            mbar_init(bar(B_DE + s), 128);
        }
        mbar_init(bar(B_FF), 128);
        mbar_init(bar(B_FE), 1);
        mbar_init(bar(B_DR), 1);
        fence_barrier_init();
        misc[1] = 0;
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(misc), kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp == 0) {
        if (lane == 0) {   // ------------------------------------------------ TMA producer
            prefetch_tmap(&xmap);
            bool ok = true;
            int i = 0;
            for (int w = w_begin; w < w_end; ++w, ++i) {
                const int b = i & 1;
                if (i >= 2 && !mbar_wait(bar(B_AE + b), ((i >> 1) - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                const int bh = w / tiles_per_head, p0 = (w % tiles_per_head) * BM;
                mbar_arrive_expect_tx(bar(B_AF + b), L::AB);
                for (int hh = 0; hh < 2; ++hh)
                    tma_load_2d(s_base + L::oA + b * L::AB + hh * BM * 128, &xmap, bar(B_AF + b), hh * 64,
                                bh * N + p0);
            }
            if (!ok) {
                record_status(status, SPARSEPR_TIMEOUT, 80);
                *abort_flag = 1;
            }
            // every copy issued lands before the block can exit
            for (int t = max(0, i - 2); t < i; ++t) mbar_wait(bar(B_AF + (t & 1)), (t >> 1) & 1, nullptr, kSpin);
        }
    } else if (warp == 1) {
        if (lane == 0) {   // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = idesc_f32acc(BM, R, kFmtBF16, false);
            bool ok = true;
            int heads = 0, cur_bh = -1, i = 0;
            for (int w = w_begin; ok && w < w_end; ++w, ++i) {
                const int bh = w / tiles_per_head;
                if (bh != cur_bh) {
                    if (!mbar_wait(bar(B_FF), heads & 1, abort_flag, kSpin)) { ok = false; break; }
                    cur_bh = bh;
                    ++heads;
                }
                const int b = i & 1, d = i & 1;
                if (!mbar_wait(bar(B_AF + b), (i >> 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                if (i >= 2 && !mbar_wait(bar(B_DE + d), ((i >> 1) - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                tc_fence_after();
                const uint32_t dst = tmem + d * (kCols / 2);
                int n = 0;
                for (int pc = 0; pc < 3; ++pc)
                    for (int kk = 0; kk < D / 16; ++kk, ++n) {
                        const uint64_t a =
                            smem_desc(s_base + L::oA + b * L::AB + (kk / 4) * BM * 128 + (kk % 4) * 32, 16, 1024);
                        const uint64_t f =
                            smem_desc(s_base + L::oF + pc * L::FB + (kk / 4) * R * 128 + (kk % 4) * 32, 16, 1024);
                        mma_f16_ss(dst, a, f, idesc, n > 0 ? 1u : 0u);
                    }
                mma_commit(bar(B_AE + b));
                mma_commit(bar(B_DF + d));
                // the last tile of a head releases F for the next head's staging
                if (w + 1 == w_end || (w + 1) / tiles_per_head != bh) mma_commit(bar(B_FE));
            }
            if (!ok) {
                record_status(status, SPARSEPR_TIMEOUT, 81);
                *abort_flag = 1;
            }
            mma_commit(bar(B_DR));
            mbar_wait(bar(B_DR), 0, nullptr, kSpin);
        }
    } else {
        // ------------------------------------------------ epilogue (and F staging), 128 threads
        const int et = tid - 64, quad = warp & 3, m = quad * 32 + lane;
        const uint32_t t_row = tmem + ((uint32_t)(quad * 32) << 16);
        bool ok = true;
        int heads = 0, cur_bh = -1, i = 0;
        for (int w = w_begin; ok && w < w_end; ++w, ++i) {
            const int bh = w / tiles_per_head, p = (w % tiles_per_head) * BM + m;
            if (bh != cur_bh) {
                // F^T pieces of this head: element (c, t) = F[t][c]; the previous
                // head's MMAs must have finished reading the old copy
                if (heads > 0 && !mbar_wait(bar(B_FE), (heads - 1) & 1, abort_flag, kSpin)) { ok = false; break; }
                const float* Fh = F + (size_t)bh * D * R;
                for (int e = et; e < D * R; e += 128) {
                    const int t = e / R, c = e % R;
                    const float f = Fh[e];
                    const __nv_bfloat16 f0 = __float2bfloat16_rn(f);
                    const float r1 = f - __bfloat162float(f0);
                    const __nv_bfloat16 f1 = __float2bfloat16_rn(r1);
                    const __nv_bfloat16 f2 = __float2bfloat16_rn(r1 - __bfloat162float(f1));
                    const uint32_t off = (uint32_t)((t >> 6) * R * 128) + sw128_h(c, t & 63);
                    *reinterpret_cast<__nv_bfloat16*>(sm + L::oF + off) = f0;
                    *reinterpret_cast<__nv_bfloat16*>(sm + L::oF + L::FB + off) = f1;
                    *reinterpret_cast<__nv_bfloat16*>(sm + L::oF + 2 * L::FB + off) = f2;
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(B_FF));
                cur_bh = bh;
                ++heads;
            }
            const int d = i & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DF + d), (i >> 1) & 1, abort_flag, kSpin));
            if (!ok) break;
            tc_fence_after();
            float acc[R];
#pragma unroll
            for (int c = 0; c < R; c += 16) {
                float v[16];
                tmem_ld16(t_row + d * (kCols / 2) + c, v);
                tmem_wait_ld(v);
#pragma unroll
                for (int u = 0; u < 16; ++u) acc[c + u] = v[u];
            }
            tc_fence_before();
            mbar_arrive(bar(B_DE + d));
            if (p < N) {
                if (RMS) {
                    float ss = 0.f;
#pragma unroll
                    for (int c = 0; c < R; ++c) ss = fmaf(acc[c], acc[c], ss);
                    const float den = fmaxf(sqrtf(ss / (float)r_eff[bh]), eps);
#pragma unroll
                    for (int c = 0; c < R; ++c) acc[c] = acc[c] / den;
                }
                // k-means runs on TF32 coordinates (exact products on the tensor cores)
                float4* out = reinterpret_cast<float4*>(phi + ((size_t)bh * N + p) * R);
#pragma unroll
                for (int c = 0; c < R; c += 4)
                    out[c / 4] = make_float4(tf32_round(acc[c]), tf32_round(acc[c + 1]), tf32_round(acc[c + 2]),
                                             tf32_round(acc[c + 3]));
            }
        }
        if (!ok) {
            record_status(status, SPARSEPR_TIMEOUT, 82);
            *abort_flag = 1;
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kCols);
    }
}

bool launch_project_tc(const void* X, const float* F, int BH, int N, int d, int R, bool rms, const int32_t* r_eff,
                       float eps, float* phi, DevStatus* status, cudaStream_t st) {
    if (d != prtc::D || (R != 16 && R != 32 && R != 48 && R != 64)) return false;
    CUtensorMap xmap;
    if (!encode_rows_map(&xmap, X, (uint64_t)BH * N, (uint64_t)d, 2, false, 64, prtc::BM)) return false;
    const long long tiles = (long long)BH * ((N + prtc::BM - 1) / prtc::BM);
    const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
    if (grid == 0) return true;
#define SPR_PTC(RR, MM)                                                                                          \
    {                                                                                                            \
        auto k = project_tc_kernel<RR, MM>;                                                                      \
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, prtc::Layout<RR>::smem);            \
        count_launch(), k<<<grid, prtc::kThreads, prtc::Layout<RR>::smem, st>>>(xmap, F, BH, N, r_eff, eps, phi, \
                                                                               status);                         \
    }
    if (rms) {
        switch (R) {
            case 16: SPR_PTC(16, true) break;
            case 32: SPR_PTC(32, true) break;
            case 48: SPR_PTC(48, true) break;
            default: SPR_PTC(64, true) break;
        }
    } else {
        switch (R) {
            case 16: SPR_PTC(16, false) break;
            case 32: SPR_PTC(32, false) break;
            case 48: SPR_PTC(48, false) break;
            default: SPR_PTC(64, false) break;
        }
    }
#undef SPR_PTC
    return true;
}

}  // namespace spr
