// C ABI of the SparsePR call: validation, workspace plan, stage entry points
// and the fused call.  See include/sparsepr.h for the contract.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace spr {

namespace {
size_t bump(size_t& cur, size_t bytes) {
    const size_t off = cur;
    cur += (bytes + 255) / 256 * 256;
    return off;
}
}  // namespace

bool make_plan(const sparsepr_params& p, Plan& pl) {
    if (sparsepr_validate(&p) != SPARSEPR_OK) return false;
    const size_t BH = (size_t)p.B * p.H, N = p.N, d = p.d;
    pl.BH = (int)BH;
    pl.G = p.Hkv > 0 ? p.H / p.Hkv : 1;
    pl.N = p.N;
    pl.d = p.d;
    pl.Cq = p.Cq;
    pl.Ck = p.Ck;
    pl.Cmax = p.Cq > p.Ck ? p.Cq : p.Ck;
    pl.Ms_eff = p.Ms < p.N ? p.Ms : p.N;
    int rk = p.rK < p.d ? p.rK : p.d;
    rk = rk < pl.Ms_eff ? rk : pl.Ms_eff;
    pl.rK_eff = rk;
    // coordinate rows: a multiple of 16 floats and at least one 128-byte TMA
    // chunk; the raw rows (d floats) for a semantic side
    pl.RKp = round_up(rk, 16) < 32 ? 32 : round_up(rk, 16);
    pl.RQp = round_up(p.rQ < p.d ? p.rQ : p.d, 16) < 32 ? 32 : round_up(p.rQ < p.d ? p.rQ : p.d, 16);
    if (p.flags & SPARSEPR_FLAG_SEMANTIC_KEYS) pl.RKp = p.d;
    if (p.flags & SPARSEPR_FLAG_SEMANTIC_QUERIES) pl.RQp = p.d;
    pl.Mp = p.M < p.N ? p.M : p.N;
    pl.esz = p.dtype == SPARSEPR_BF16 ? 2 : 4;
    pl.n_sort_tiles = (p.N + kSortTile - 1) / kSortTile;
    pl.BM = p.block;
    pl.n_items_max = (int)(BH * ((N + p.block - 1) / p.block + (size_t)p.Cq));
    pl.n_probe_items = pl.Mp > 0 ? (int)(BH * ((pl.Mp + p.block - 1) / p.block)) : 0;
    // key budget: beta = (rho - M/N) N clamped to [0, N]; "reaches beta" on
    // integer counts means >= ceil(beta), with beta within 1e-6 of an integer
    // taken as that integer.
    double beta = (p.density - (double)pl.Mp / (double)p.N) * (double)p.N;
    beta = beta < 0.0 ? 0.0 : (beta > (double)p.N ? (double)p.N : beta);
    pl.beta = (int64_t)ceil(beta - 1e-6);
    pl.stop_changed = (int)floor(p.kmeans_tol * (double)p.N);

    const size_t Cq = p.Cq, Ck = p.Ck, Cm = pl.Cmax, Mp = pl.Mp, es = pl.esz;
    size_t c = 0;
    pl.o_status = bump(c, 256);
    pl.o_ctl = bump(c, BH * kCtlStride * 4);
    pl.o_mat = bump(c, BH * d * d * 4);
    pl.o_FK = bump(c, BH * d * pl.RKp * 4);
    pl.o_FQ = bump(c, BH * d * pl.RQp * 4);
    pl.o_rq = bump(c, BH * 4);
    pl.o_phiK = bump(c, BH * N * pl.RKp * 4);
    pl.o_phiQ = bump(c, BH * N * pl.RQp * 4);
    pl.o_cenK = bump(c, BH * Ck * pl.RKp * 4);
    pl.o_hnK = bump(c, BH * Ck * 4);
    pl.o_cenQ = bump(c, BH * Cq * pl.RQp * 4);
    pl.o_hnQ = bump(c, BH * Cq * 4);
    pl.o_hs = bump(c, BH * Cm * 8 * 4);
    pl.o_raw = bump(c, BH * N * 4);
    pl.o_hist = bump(c, BH * pl.n_sort_tiles * Cm * 4);
    pl.o_sorted = bump(c, BH * N * 4);
    pl.o_offs = bump(c, BH * (Cm + 1) * 4);
    pl.o_newid = bump(c, BH * Cm * 4);
    pl.o_muK = bump(c, BH * d * 4);
    pl.o_t1 = bump(c, BH * Cq * Ck * 4);
    pl.o_t2 = bump(c, BH * Cq * Ck * 4);
    pl.o_mloc = bump(c, BH * Cq * Ck * 4);
    pl.o_pslot = bump(c, BH * N * 4);
    pl.o_palloc = bump(c, BH * Cq * 4);
    pl.o_poff = bump(c, BH * Cq * 4);
    pl.o_psum = bump(c, BH * 4);
    pl.o_qprobe = bump(c, BH * (Mp > 0 ? Mp : 1) * d * es);
    pl.o_work = bump(c, 256 + (size_t)pl.n_items_max * 16);
    pl.o_fstat = bump(c, BH * 3 * d * 8);
    pl.o_G = bump(c, BH * d * d * 8);
    pl.o_rhs = bump(c, BH * d * d * 8);
    const size_t BHk = BH / pl.G;   // K/V heads: the permuted K/V and their fp16 copy are per K/V head
    pl.o_vh = bump(c, p.dtype == SPARSEPR_BF16 ? BHk * N * d * 2 : 256);
    pl.o_vmax = bump(c, BH * 4);
    pl.o_vscale = bump(c, BH * 4);
    pl.o_qsplit = bump(c, BH * 3 * (size_t)round_up(p.Cq, 128) * d * 2);
    pl.o_uw = bump(c, BH * N * 8);
    pl.o_lbar = bump(c, BH * Cq * Ck * 4);
    pl.o_vv = bump(c, BH * Ck * 4);
    pl.o_warm = bump(c, (1 + 2 * BH) * 4);
    pl.o_pbits = bump(c, BH * ((N + 31) / 32) * 4);
    pl.o_S = bump(c, p.residual_rank > 0 ? BH * d * d * 8 : 256);
    pl.o_rawkv = bump(c, pl.G > 1 ? BH / pl.G * N * 4 : 256);
    {
        const size_t Rmax = pl.RKp > pl.RQp ? pl.RKp : pl.RQp;
        pl.o_csum = bump(c, BH * Cm * Rmax * 8);
        pl.o_ccnt = bump(c, BH * Cm * 4);
        pl.o_prev = bump(c, BH * N * 4);
        pl.o_cscale = bump(c, BH * 4);
    }
    // outputs owned by the workspace (fused call)
    pl.o_Qp = bump(c, BH * N * d * es);
    pl.o_Kp = bump(c, BHk * N * d * es);
    pl.o_Vp = bump(c, BHk * N * d * es);
    pl.o_qlab = bump(c, BH * N * 4);
    pl.o_kvlab = bump(c, BH * N * 4);
    pl.o_permq = bump(c, BH * N * 4);
    pl.o_permk = bump(c, BH * N * 4);
    pl.o_posq = bump(c, BH * N * 4);
    pl.o_qoff = bump(c, BH * (Cq + 1) * 4);
    pl.o_kvoff = bump(c, BH * (Ck + 1) * 4);
    pl.o_ng = bump(c, BH * 2 * 4);
    pl.o_its = bump(c, BH * 2 * 4);
    pl.o_qcen = bump(c, BH * Cq * d * 4);
    pl.o_kcen = bump(c, BH * Ck * d * 4);
    pl.o_vcen = bump(c, BH * Ck * d * 4);
    pl.o_qdist = bump(c, BH * N * 4);
    pl.o_score = bump(c, BH * Cq * Ck * 4);
    pl.o_mask = bump(c, BH * Cq * Ck);
    pl.o_selc = bump(c, BH * Cq * 4);
    pl.o_selg = bump(c, BH * Cq * Ck * 4);
    pl.o_pairs = bump(c, BH * 2 * 8);
    pl.o_pidx = bump(c, BH * (Mp > 0 ? Mp : 1) * 4);
    pl.o_pgrp = bump(c, BH * (Mp > 0 ? Mp : 1) * 4);
    pl.o_pw = bump(c, BH * (Mp > 0 ? Mp : 1) * 4);
    pl.o_Osp = bump(c, BH * N * d * 4);
    pl.o_pdense = bump(c, BH * (Mp > 0 ? Mp : 1) * d * 4);
    pl.o_psparse = bump(c, BH * (Mp > 0 ? Mp : 1) * d * 4);
    pl.o_fB = bump(c, BH * d * d * 4);
    pl.o_fmux = bump(c, BH * d * 4);
    pl.o_fsig = bump(c, BH * d * 4);
    pl.o_fmur = bump(c, BH * d * 4);
    pl.total = c;
    return true;
}

namespace {

sparsepr_status check_ws(const sparsepr_params* p, Plan& pl, void* ws, size_t bytes) {
    if (p == nullptr) return SPARSEPR_INVALID_ARG;
    const sparsepr_status v = sparsepr_validate(p);
    if (v != SPARSEPR_OK) return v;
    if (!make_plan(*p, pl)) return SPARSEPR_INVALID_ARG;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SPARSEPR_INVALID_ARG;
    if (bytes < pl.total) return SPARSEPR_WORKSPACE_TOO_SMALL;
    return SPARSEPR_OK;
}

bool partition_ok(const sparsepr_partition_out* o) {
    return o && o->Qp && o->Kp && o->Vp && o->q_label && o->kv_label && o->perm_q && o->perm_kv && o->pos_q &&
           o->q_offsets && o->kv_offsets && o->n_groups && o->kmeans_iters_run && o->q_centroid &&
           o->k_centroid && o->v_centroid && o->q_dist;
}
bool route_ok(const sparsepr_route_out* r, int Mp) {
    return r && r->score && r->mask && r->sel_count && r->sel_groups && r->pairs && r->probe_alloc &&
           (Mp == 0 || (r->probe_idx && r->probe_group && r->probe_weight));
}
bool fit_ok(const sparsepr_fit_out* f) { return f && f->B && f->mu_x && f->sigma && f->mu_r; }

sparsepr_partition_out owned_partition(const Plan& pl, void* ws) {
    sparsepr_partition_out o = {};
    o.Qp = at<void>(ws, pl.o_Qp);
    o.Kp = at<void>(ws, pl.o_Kp);
    o.Vp = at<void>(ws, pl.o_Vp);
    o.q_label = at<int32_t>(ws, pl.o_qlab);
    o.kv_label = at<int32_t>(ws, pl.o_kvlab);
    o.perm_q = at<int32_t>(ws, pl.o_permq);
    o.perm_kv = at<int32_t>(ws, pl.o_permk);
    o.pos_q = at<int32_t>(ws, pl.o_posq);
    o.q_offsets = at<int32_t>(ws, pl.o_qoff);
    o.kv_offsets = at<int32_t>(ws, pl.o_kvoff);
    o.n_groups = at<int32_t>(ws, pl.o_ng);
    o.kmeans_iters_run = at<int32_t>(ws, pl.o_its);
    o.q_centroid = at<float>(ws, pl.o_qcen);
    o.k_centroid = at<float>(ws, pl.o_kcen);
    o.v_centroid = at<float>(ws, pl.o_vcen);
    o.q_dist = at<float>(ws, pl.o_qdist);
    return o;
}
sparsepr_route_out owned_route(const Plan& pl, void* ws) {
    sparsepr_route_out r = {};
    r.score = at<float>(ws, pl.o_score);
    r.mask = at<uint8_t>(ws, pl.o_mask);
    r.sel_count = at<int32_t>(ws, pl.o_selc);
    r.sel_groups = at<int32_t>(ws, pl.o_selg);
    r.pairs = at<int64_t>(ws, pl.o_pairs);
    r.probe_idx = at<int32_t>(ws, pl.o_pidx);
    r.probe_group = at<int32_t>(ws, pl.o_pgrp);
    r.probe_weight = at<float>(ws, pl.o_pw);
    r.probe_alloc = at<int32_t>(ws, pl.o_palloc);
    return r;
}
sparsepr_fit_out owned_fit(const Plan& pl, void* ws) {
    sparsepr_fit_out f = {};
    f.B = at<float>(ws, pl.o_fB);
    f.mu_x = at<float>(ws, pl.o_fmux);
    f.sigma = at<float>(ws, pl.o_fsig);
    f.mu_r = at<float>(ws, pl.o_fmur);
    return f;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace
}  // namespace spr

using namespace spr;

extern "C" {

const char* sparsepr_status_string(int32_t s) {
    switch (s) {
        case SPARSEPR_OK: return "ok";
        case SPARSEPR_INVALID_ARG: return "invalid argument";
        case SPARSEPR_UNSUPPORTED: return "unsupported configuration";
        case SPARSEPR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case SPARSEPR_CUDA_ERROR: return "CUDA error";
        case SPARSEPR_TIMEOUT: return "device wait timed out";
        case SPARSEPR_NUMERIC: return "ridge Gram matrix not positive definite";
        default: return "unknown status";
    }
}

sparsepr_status sparsepr_validate(const sparsepr_params* p) {
    if (p == nullptr) return SPARSEPR_INVALID_ARG;
    if (p->B < 1 || p->H < 1 || p->N < 1 || p->d < 1) return SPARSEPR_INVALID_ARG;
    if ((long long)p->T * p->Y * p->X != (long long)p->N || p->T < 1 || p->Y < 1 || p->X < 1)
        return SPARSEPR_INVALID_ARG;
    if (p->dtype != SPARSEPR_BF16 && p->dtype != SPARSEPR_F32) return SPARSEPR_INVALID_ARG;
    if (!(p->density > 0.0) || !isfinite(p->density)) return SPARSEPR_INVALID_ARG;
    if (p->M < 0 || p->Ms < 1) return SPARSEPR_INVALID_ARG;
    if (!(p->lambda > 0.0) || !isfinite(p->lambda)) return SPARSEPR_INVALID_ARG;
    if (p->Cq < 1 || p->Ck < 1 || p->rK < 1 || p->rQ < 1) return SPARSEPR_INVALID_ARG;
    if (p->kmeans_iters < 1 || p->kmeans_iters > 1000 || !(p->kmeans_tol >= 0.0)) return SPARSEPR_INVALID_ARG;
    if (!(p->eps_rms > 0.f) || !(p->eps_std >= 0.f)) return SPARSEPR_INVALID_ARG;
    if (p->block != 64 && p->block != 128) return SPARSEPR_INVALID_ARG;
    if (p->probe_select < 0 || p->probe_select > 2 || p->correction < 0 || p->correction > 3) return SPARSEPR_INVALID_ARG;
    if (p->residual_rank < 0 || p->residual_rank > p->d) return SPARSEPR_INVALID_ARG;
    if (p->Hkv < 0 || (p->Hkv > 0 && p->H % p->Hkv != 0)) return SPARSEPR_INVALID_ARG;
    if (p->d != 64 && p->d != 128) return SPARSEPR_UNSUPPORTED;
    if (p->Cq > kMaxGroups || p->Ck > kMaxGroups) return SPARSEPR_UNSUPPORTED;
    if (p->rK > kMaxRank || p->rQ > kMaxRank) return SPARSEPR_UNSUPPORTED;
    if (p->N > kMaxN) return SPARSEPR_UNSUPPORTED;
    if ((long long)p->B * p->H * p->N > (1LL << 31) - 1) return SPARSEPR_UNSUPPORTED;
    return SPARSEPR_OK;
}

size_t sparsepr_workspace_size(const sparsepr_params* p) {
    if (p == nullptr) return 0;
    Plan pl;
    if (!make_plan(*p, pl)) return 0;
    return pl.total;
}

sparsepr_status sparsepr_partition(const sparsepr_params* p, const void* Q, const void* K, const void* V,
                                   const sparsepr_partition_out* part, void* ws, size_t bytes, void* stream) {
    Plan pl;
    sparsepr_status s = check_ws(p, pl, ws, bytes);
    if (s != SPARSEPR_OK) return s;
    if (!Q || !K || !V || !partition_ok(part)) return SPARSEPR_INVALID_ARG;
    if ((p->flags & SPARSEPR_FLAG_DEBUG_EXPORT) &&
        !(part->debug_kv_scores && part->debug_q_scores && part->debug_kv_hist && part->debug_q_hist))
        return SPARSEPR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (cudaMemsetAsync(at<void>(ws, pl.o_status), 0, 256, st) != cudaSuccess) return SPARSEPR_CUDA_ERROR;
    // the workspace no longer holds a complete fused-call state
    if (cudaMemsetAsync(at<void>(ws, pl.o_warm), 0, 4, st) != cudaSuccess) return SPARSEPR_CUDA_ERROR;
    return run_partition(*p, pl, Q, K, V, *part, ws, st);
}

sparsepr_status sparsepr_partition_warm(const sparsepr_params* p, const void* Q, const void* K, const void* V,
                                        const sparsepr_warm_state* prev, const sparsepr_partition_out* part,
                                        void* ws, size_t bytes, void* stream) {
    Plan pl;
    sparsepr_status s = check_ws(p, pl, ws, bytes);
    if (s != SPARSEPR_OK) return s;
    if (!Q || !K || !V || !partition_ok(part)) return SPARSEPR_INVALID_ARG;
    if (!prev || !prev->F_K || !prev->F_Q || !prev->k_centroid || !prev->q_centroid || !prev->n_groups)
        return SPARSEPR_INVALID_ARG;
    if ((p->flags & SPARSEPR_FLAG_DEBUG_EXPORT) &&
        !(part->debug_kv_scores && part->debug_q_scores && part->debug_kv_hist && part->debug_q_hist))
        return SPARSEPR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (cudaMemsetAsync(at<void>(ws, pl.o_status), 0, 256, st) != cudaSuccess) return SPARSEPR_CUDA_ERROR;
    if (cudaMemsetAsync(at<void>(ws, pl.o_warm), 0, 4, st) != cudaSuccess) return SPARSEPR_CUDA_ERROR;
    // F_K is per query head in the caller's outputs: K/V head h reads query head h * G
    const WarmSource src{prev->F_K, prev->F_Q, prev->k_centroid, prev->q_centroid, prev->n_groups, nullptr, pl.G};
    return run_partition(*p, pl, Q, K, V, *part, ws, st, &src);
}

sparsepr_status sparsepr_route(const sparsepr_params* p, const sparsepr_partition_out* part,
                               const sparsepr_route_out* route, void* ws, size_t bytes, void* stream) {
    Plan pl;
    sparsepr_status s = check_ws(p, pl, ws, bytes);
    if (s != SPARSEPR_OK) return s;
    if (!partition_ok(part) || !route_ok(route, pl.Mp)) return SPARSEPR_INVALID_ARG;
    return run_route(*p, pl, *part, *route, ws, as_stream(stream));
}

sparsepr_status sparsepr_attention(const sparsepr_params* p, const sparsepr_partition_out* part,
                                   const sparsepr_route_out* route, float* O_sp, float* probe_dense,
                                   float* probe_sparse, void* ws, size_t bytes, void* stream) {
    Plan pl;
    sparsepr_status s = check_ws(p, pl, ws, bytes);
    if (s != SPARSEPR_OK) return s;
    if (!partition_ok(part) || !route_ok(route, pl.Mp) || !O_sp) return SPARSEPR_INVALID_ARG;
    if (pl.Mp > 0 && (!probe_dense || !probe_sparse)) return SPARSEPR_INVALID_ARG;
    return run_attention(*p, pl, *part, *route, O_sp, probe_dense, probe_sparse, ws, as_stream(stream));
}

sparsepr_status sparsepr_probe_fit(const sparsepr_params* p, const sparsepr_partition_out* part,
                                   const sparsepr_route_out* route, const float* probe_sparse,
                                   const float* probe_dense, const sparsepr_fit_out* fit, void* ws, size_t bytes,
                                   void* stream) {
    Plan pl;
    sparsepr_status s = check_ws(p, pl, ws, bytes);
    if (s != SPARSEPR_OK) return s;
    if (!partition_ok(part) || !route_ok(route, pl.Mp) || !fit_ok(fit)) return SPARSEPR_INVALID_ARG;
    if (pl.Mp > 0 && (!probe_dense || !probe_sparse)) return SPARSEPR_INVALID_ARG;
    return run_fit(*p, pl, *part, *route, probe_sparse, probe_dense, *fit, ws, as_stream(stream));
}

sparsepr_status sparsepr_apply(const sparsepr_params* p, const sparsepr_partition_out* part,
                               const sparsepr_route_out* route, const float* O_sp, const float* probe_dense,
                               const sparsepr_fit_out* fit, float* O_out, void* ws, size_t bytes, void* stream) {
    Plan pl;
    sparsepr_status s = check_ws(p, pl, ws, bytes);
    if (s != SPARSEPR_OK) return s;
    if (!partition_ok(part) || !route_ok(route, pl.Mp) || !fit_ok(fit) || !O_sp || !O_out) return SPARSEPR_INVALID_ARG;
    if (pl.Mp > 0 && !probe_dense) return SPARSEPR_INVALID_ARG;
    return run_apply(*p, pl, *part, *route, O_sp, probe_dense, *fit, O_out, ws, as_stream(stream));
}

sparsepr_status sparsepr_call(const sparsepr_params* p, const void* Q, const void* K, const void* V, float* O_out,
                              sparsepr_stats* stats, void* ws, size_t bytes, void* stream) {
    Plan pl;
    sparsepr_status s = check_ws(p, pl, ws, bytes);
    if (s != SPARSEPR_OK) return s;
    if (!Q || !K || !V || !O_out) return SPARSEPR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    const sparsepr_partition_out part = owned_partition(pl, ws);
    const sparsepr_route_out route = owned_route(pl, ws);
    const sparsepr_fit_out fit = owned_fit(pl, ws);
    float* O_sp = at<float>(ws, pl.o_Osp);
    float* pdense = at<float>(ws, pl.o_pdense);
    float* psparse = at<float>(ws, pl.o_psparse);
    cudaEvent_t ev[6] = {};
    if (stats) {
        for (int i = 0; i < 6; ++i)
            if (cudaEventCreate(&ev[i]) != cudaSuccess) return SPARSEPR_CUDA_ERROR;
        cudaEventRecord(ev[0], st);
    }
    if (cudaMemsetAsync(at<void>(ws, pl.o_status), 0, 256, st) != cudaSuccess) return SPARSEPR_CUDA_ERROR;
    const long long launches0 = launch_counter();
    sparsepr_params q = *p;
    q.flags &= ~SPARSEPR_FLAG_DEBUG_EXPORT;
    int32_t* warm_word = at<int32_t>(ws, pl.o_warm);
    // the workspace keeps F_K per K/V head (stride 1); centroids and counts are per query head
    const WarmSource src{at<float>(ws, pl.o_FK), at<float>(ws, pl.o_FQ), part.k_centroid, part.q_centroid,
                         part.n_groups, warm_word, 1};
    const bool warm = (p->flags & SPARSEPR_FLAG_WARM_START) != 0;
    if ((s = run_partition(q, pl, Q, K, V, part, ws, st, warm ? &src : nullptr)) != SPARSEPR_OK) return s;
    launch_set_word(warm_word, kWarmMagic, st);
    if (stats) cudaEventRecord(ev[1], st);
    if ((s = run_route(q, pl, part, route, ws, st)) != SPARSEPR_OK) return s;
    if (stats) cudaEventRecord(ev[2], st);
    if ((s = run_attention(q, pl, part, route, O_sp, pdense, psparse, ws, st)) != SPARSEPR_OK) return s;
    if (stats) cudaEventRecord(ev[3], st);
    if ((s = run_fit(q, pl, part, route, psparse, pdense, fit, ws, st)) != SPARSEPR_OK) return s;
    if (stats) cudaEventRecord(ev[4], st);
    if ((s = run_apply(q, pl, part, route, O_sp, pdense, fit, O_out, ws, st)) != SPARSEPR_OK) return s;
    if (stats) {
        cudaEventRecord(ev[5], st);
        if (cuda_status(cudaEventSynchronize(ev[5])) != SPARSEPR_OK) return SPARSEPR_CUDA_ERROR;
        float ms[5];
        for (int i = 0; i < 5; ++i) cudaEventElapsedTime(&ms[i], ev[i], ev[i + 1]);
        stats->ms_partition = ms[0];
        stats->ms_route = ms[1];
        stats->ms_attention = ms[2];
        stats->ms_fit = ms[3];
        stats->ms_apply = ms[4];
        cudaEventElapsedTime(&stats->ms_total, ev[0], ev[5]);
        for (int i = 0; i < 6; ++i) cudaEventDestroy(ev[i]);
        int64_t pairs_h[2] = {0, 0};
        int64_t route_sum = 0, exec_sum = 0;
        for (int bh = 0; bh < pl.BH; ++bh) {
            if (cudaMemcpy(pairs_h, route.pairs + 2 * bh, 16, cudaMemcpyDeviceToHost) != cudaSuccess)
                return SPARSEPR_CUDA_ERROR;
            route_sum += pairs_h[0];
            exec_sum += pairs_h[1];
        }
        int64_t visited = 0;
        if (cudaMemcpy(&visited, at<int64_t>(ws, pl.o_work + 8), 8, cudaMemcpyDeviceToHost) != cudaSuccess)
            return SPARSEPR_CUDA_ERROR;
        stats->pairs_route = route_sum;
        stats->pairs_exec = exec_sum;
        stats->pairs_visited = visited;
        stats->rho_exec = (double)exec_sum / ((double)pl.BH * (double)pl.N * (double)pl.N);
        stats->launches = launch_counter() - launches0;
    }
    return cuda_status(cudaGetLastError());
}

const char* sparsepr_last_error_string(void) { return last_error_buffer(); }

sparsepr_status sparsepr_get_device_status(void* ws, void* stream, int32_t* out) {
    if (ws == nullptr || out == nullptr) return SPARSEPR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    int32_t v = 0;
    sparsepr_status s = cuda_status(cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, st));
    if (s == SPARSEPR_OK) s = cuda_status(cudaStreamSynchronize(st));
    if (s == SPARSEPR_OK) s = cuda_status(cudaMemsetAsync(ws, 0, 256, st));
    if (s != SPARSEPR_OK) return s;
    *out = v;
    return SPARSEPR_OK;
}

}  // extern "C"
