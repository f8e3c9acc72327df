// Stage entry points shared by the C ABI (api.cu) and the stage files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace spr {

// Warm start (paper C.1): where the previous call's state lives.  `valid`
// (or nullptr) points at a word that must equal kWarmMagic for it to be used.
// Under GQA the K/V-side state of K/V head h is read at head h * fk_stride
// (F_K) and h * G (k_centroid and n_groups, which are per query head).
struct WarmSource {
    const float* F_K;
    const float* F_Q;
    const float* k_centroid;
    const float* q_centroid;
    const int32_t* n_groups;
    const int32_t* valid;
    int fk_stride;
};
sparsepr_status run_partition(const sparsepr_params& p, const Plan& pl, const void* Q, const void* K,
                              const void* V, const sparsepr_partition_out& out, void* ws, cudaStream_t st,
                              const WarmSource* warm = nullptr);
// Initial centres of a warm k-means: previous centroids `cbar` ([BH,C,d]) of
// the first ng_prev[bh*2+which] groups projected by F ([BH,d,R]).
struct WarmInit {
    const float* cbar;
    const int32_t* ng_prev;
    int which;
    int prev_stride;   // head of the previous state = this head * prev_stride
    const float* F;
    int d;
    bool rms;
    const int32_t* r_eff;
    float eps;
    const int32_t* valid;
};
void launch_warm_init(const WarmInit& w, int R, const float* phi, int BH, int N, int C, uint64_t seed, int stage,
                      float* cen, float* hn, cudaStream_t st);
// Leading r eigenpairs of BH symmetric d x d fp32 matrices: F[:, c] = u_c
// sqrt(max(lambda_c, 0)) for c < r, zero up to Rp (parallel cyclic Jacobi).
void launch_jacobi_factor(const float* A, float* F, int Rp, int r, int BH, int d, cudaStream_t st);
// *word = value, in stream order (one thread).
void launch_set_word(int32_t* word, int32_t value, cudaStream_t st);
// Warm metric factor; heads it cannot factor get cold[bh] = 1 (else 0).
void launch_warm_factor(const float* M, const float* Fprev, int ld_prev, int prev_stride, int r_req, const int32_t* ng,
                        float scale, float* F, int Rp, int32_t* r_out, int32_t* cold, const int32_t* valid, int BH,
                        int d, cudaStream_t st);
sparsepr_status run_route(const sparsepr_params& p, const Plan& pl, const sparsepr_partition_out& part,
                          const sparsepr_route_out& r, void* ws, cudaStream_t st);
bool attention_uses_tc(const sparsepr_params& p);
bool route_uses_tc(const sparsepr_params& p);
// Tensor-core routing-score segment sums; false if its tensor maps could not be built.
bool launch_route_tc(const Plan& pl, const sparsepr_partition_out& part, void* ws, float* t1, float* t2, float* ml,
                     cudaStream_t st);
// Tensor-core k-means assignment; false if its tensor maps could not be built.
// hs: scratch of BH * C * 8 floats for the split half-norms of the centres.
bool launch_kmeans_assign_tc(const float* phi, const float* cen, const float* hn, float* hs, int BH, int N, int C,
                             int R, int32_t* labels, int32_t* ctl, int first, float* dbg_scores, int32_t* dbg_hist,
                             int max_iter, DevStatus* status, cudaStream_t st);
// 2-D tensor map over [rows, cols] row-major elements (4-byte fp32, or 2-byte
// fp16 / bf16 chosen by is_float), boxes of box_cols x box_rows, 128-byte swizzle.
bool encode_rows_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, int elem_bytes, bool is_float,
                     uint32_t box_cols, uint32_t box_rows);
// Tensor-core projection phi = X F (bf16 X, R in {16,32,48,64}, optional RMS
// normalisation); false if it cannot run (its tensor map could not be built).
bool launch_project_tc(const void* X, const float* F, int BH, int N, int d, int R, bool rms, const int32_t* r_eff,
                       float eps, float* phi, DevStatus* status, cudaStream_t st);
// Tensor-core corrected output (d = 64 or 128); false if d is not supported.
bool launch_apply_tc(const Plan& pl, const sparsepr_partition_out& part, const float* O_sp, const float* probe_dense,
                     const sparsepr_fit_out& f, const int32_t* pslot, float* O_out, DevStatus* status,
                     cudaStream_t st);
sparsepr_status run_attention(const sparsepr_params& p, const Plan& pl, const sparsepr_partition_out& part,
                              const sparsepr_route_out& r, float* O_sp, float* probe_dense,
                              float* probe_sparse, void* ws, cudaStream_t st);
sparsepr_status run_fit(const sparsepr_params& p, const Plan& pl, const sparsepr_partition_out& part,
                        const sparsepr_route_out& r, const float* probe_sparse, const float* probe_dense,
                        const sparsepr_fit_out& f, void* ws, cudaStream_t st);
sparsepr_status run_apply(const sparsepr_params& p, const Plan& pl, const sparsepr_partition_out& part,
                          const sparsepr_route_out& r, const float* O_sp, const float* probe_dense, const sparsepr_fit_out& f, float* O_out,
                          void* ws, cudaStream_t st);

}  // namespace spr
