/*
 * sparsepr.h -- C ABI of the B200 (sm_100a) SparsePR attention call.
 *
 * The operation is one attention call of "Partition the Support, Reconstruct
 * the Residual: Training-Free Sparse Attention for Video Generation and World
 * Models" (Taghavi, Langari, Pandey; arXiv 2608.18484v2), written "paper"
 * below with the section or formula that defines each step:
 *
 *   partition  response-coupled partitioning           paper §4.1, B.1, B.2, C.1
 *              (cold, or warm-started from a previous  paper C.1 "Warm start",
 *              call of the same problem shape)         Table C.1
 *   route      value-error score + prefix budget rule   paper §4.3, B.3, A.2
 *   attention  renormalised block-sparse attention       paper §3 Eq. (2), §4.3
 *              and exact attention on the probe rows
 *   probe_fit  weighted ridge on probe residuals         paper §4.2, A.3, D.3
 *   apply      corrected output, original query order    paper §4.2 (O-hat)
 *   call       all of the above, fused on one stream
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are caller-owned DEVICE pointers (e.g. from torch).  The library
 *   allocates no device memory: every intermediate lives in one caller-owned
 *   device workspace of sparsepr_workspace_size() bytes, 256-byte aligned.
 * - Q, K, V are [B, H, N, d] row-major, contiguous, in p->dtype (bf16 or
 *   fp32); K and V are [B, Hkv, N, d] under GQA (p->Hkv, see below).  All float outputs are fp32.  Index outputs are int32 unless noted.
 *   "BH" below is B*H; per-head slices are contiguous.
 * - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *   NULL = legacy default stream) unless documented otherwise.  Group counts
 *   and list lengths stay on the device; no entry point synchronises except
 *   sparsepr_call with a non-NULL stats pointer and
 *   sparsepr_get_device_status.
 * - Arguments are validated on the host before anything is launched; a
 *   failed check returns SPARSEPR_INVALID_ARG / UNSUPPORTED /
 *   WORKSPACE_TOO_SMALL and launches nothing.  A failed launch returns
 *   SPARSEPR_CUDA_ERROR.  Failures found on the device (a bounded wait that
 *   ran out, a non-positive Cholesky pivot) are recorded in a status word in
 *   the workspace, read by sparsepr_get_device_status(); no kernel traps.
 * - Outputs sized with C_q or C_k are sized for the REQUESTED counts; only the
 *   first C_q' / C_k' (nonempty groups, reported in n_groups) entries are
 *   meaningful.
 */
#ifndef SPARSEPR_H
#define SPARSEPR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPARSEPR_OK = 0,
    SPARSEPR_INVALID_ARG = 1,          /* bad shape, null pointer, value out of range */
    SPARSEPR_UNSUPPORTED = 2,          /* valid but not built (e.g. d not in {64,128}) */
    SPARSEPR_WORKSPACE_TOO_SMALL = 3,
    SPARSEPR_CUDA_ERROR = 4,           /* a CUDA runtime call or launch failed */
    SPARSEPR_TIMEOUT = 5,              /* device: a bounded wait gave up */
    SPARSEPR_NUMERIC = 6               /* device: ridge Gram matrix not positive definite */
} sparsepr_status;

typedef enum { SPARSEPR_BF16 = 0, SPARSEPR_F32 = 1 } sparsepr_dtype;

/* Probe selection (paper A.2; Table 4's variants).  With M >= N every
 * variant takes all rows as probes. */
typedef enum {
    SPARSEPR_PROBES_STRATIFIED = 0, /* largest-remainder m_a per query group, the m_a members
                                       nearest the group mean (A.2) */
    SPARSEPR_PROBES_RANDOM = 1,     /* M distinct rows uniformly at random: Floyd's algorithm on
                                       a SplitMix64 stream seeded by
                                       mix(seed ^ mix((bh+1)*0x9E3779B97F4A7C15 ^ 0x50524F4245));
                                       draw s (s = 0..M-1, the (s+1)-th output) with top 32 bits u
                                       gives t = (u*(j+1)) >> 32 for j = N-M+s, and the sample
                                       gains t, or j if t is already in it */
    SPARSEPR_PROBES_UNIFORM = 2     /* rows floor((2j+1)N / 2M), j < M: evenly spaced over the
                                       row-major (t,y,x) grid */
} sparsepr_probe_select;

/* Correction family (paper D.4); every family keeps the weighted
 * standardisation, centring and coverage weights of A.3. */
typedef enum {
    SPARSEPR_CORRECTION_FULL = 0,     /* unrestricted B (weighted ridge, §4.2) */
    SPARSEPR_CORRECTION_DIAGONAL = 1, /* B = diag(b), b_j = (X^T W R)_jj / ((X^T W X)_jj + lambda) */
    SPARSEPR_CORRECTION_SCALAR = 2,   /* B = a I, a = tr(X^T W R) / (tr(X^T W X) + lambda d) */
    SPARSEPR_CORRECTION_MEAN = 3      /* B = 0: the weighted mean residual only */
} sparsepr_correction;

/* flags */
#define SPARSEPR_FLAG_DEBUG_EXPORT 1   /* fill the debug_* outputs of partition */
#define SPARSEPR_FLAG_SIMT_ATTENTION 2 /* bf16: use the CUDA-core attention kernel */
#define SPARSEPR_FLAG_WARM_START 4     /* sparsepr_call: warm-start the partition from the state the
                                          previous sparsepr_call with the same *p left in this
                                          workspace (see sparsepr_partition_warm); without such a
                                          state the call is cold */
#define SPARSEPR_FLAG_SEMANTIC_KEYS 8  /* K/V groups by k-means on the raw key rows instead of the
                                          key-response coordinates (paper §3 reference partition,
                                          Table 2 baseline); F_K is then the d x d identity and
                                          RKp = d */
#define SPARSEPR_FLAG_SEMANTIC_QUERIES 16 /* query groups by k-means on the raw query rows (no
                                          RMSNorm); d_i is the raw-space distance to the group
                                          mean, F_Q the identity and RQp = d.  With
                                          SEMANTIC_KEYS: the semantic partition; alone: Table 2's
                                          key-response K/V variant */

/* Problem statement (paper §3 / §4 notation).  All fields are read on the host. */
typedef struct {
    int32_t B, H, N, d;        /* batch, heads, tokens, head dim (d in {64,128}) */
    int32_t T, Y, X;           /* token grid; N must equal T*Y*X (row-major t,y,x) */
    int32_t dtype;             /* sparsepr_dtype of Q, K, V */
    double density;            /* target executed-pair density incl. probes (§4.3) */
    int32_t M;                 /* exact probe rows per head (§4.2); min(M,N) used */
    int32_t Ms;                /* sampled queries for M_K (§4.1, C.2) */
    double lambda;             /* ridge coefficient (§4.2), > 0 */
    int32_t Cq, Ck;            /* requested query / K-V group counts, 1..2048 */
    int32_t rK, rQ;            /* response ranks (§4.1, B.2), 1..64 */
    int32_t kmeans_iters;      /* maximum k-means assignments, >= 1 (Table C.1) */
    double kmeans_tol;         /* stop when changed labels <= floor(tol*N) */
    uint64_t seed;             /* k-means initial-centre stream seed (C.1) */
    int32_t block;             /* attention query tile rows: 64 or 128 */
    float eps_rms;             /* RMSNorm floor in phi_Q (B.2) */
    float eps_std;             /* variance floor in the standardisation (D.3) */
    int32_t flags;             /* SPARSEPR_FLAG_* */
    int32_t probe_select;      /* sparsepr_probe_select (0 = stratified, the paper's method) */
    int32_t correction;        /* sparsepr_correction (0 = full ridge, the paper's method) */
    int32_t residual_rank;     /* 0: no truncation (the paper's method); r in 1..d: B V_r V_r^T with
                                  V_r the leading r right singular vectors of W^1/2 Rbar (D.3) */
    int32_t Hkv;               /* K/V heads: 0 or H (one per query head), else a divisor of H:
                                  grouped-query attention with G = H/Hkv query heads per K/V head,
                                  query head h using K/V head h/G.  The G heads share the key
                                  metric (G*Ms evenly spaced rows of their stacked queries), F_K
                                  and the K/V groups (§4.3 "Routing and GQA", C.1); query groups,
                                  routing, probes and fit stay per query head.  K and V are then
                                  [B,Hkv,N,d]; every output stays per query head (K/V-side
                                  outputs repeated G times; the debug K/V arrays are indexed by
                                  K/V head). */
} sparsepr_params;

/* Outputs of sparsepr_partition (paper §4.1).  Required unless marked
 * optional (NULL = not written).  Sizes: BH*N int32 for per-row arrays. */
typedef struct {
    void* Qp;             /* [BH,N,d] p->dtype: rows in group-major order, stable by original index (§4.3) */
    void* Kp; void* Vp;   /* [B*Hkv,N,d] p->dtype: the same for the keys (V keeps its key's row), one per
                             K/V head: under GQA the G query heads of a K/V head share its groups, so
                             its rows are stored once (without GQA, Hkv = H) */
    int32_t* q_label;     /* [BH,N] query group of each ORIGINAL row (0..C_q'-1) */
    int32_t* kv_label;    /* [BH,N] K/V group of each original key row */
    int32_t* perm_q;      /* [BH,N] permuted row -> original row */
    int32_t* perm_kv;     /* [BH,N] */
    int32_t* pos_q;       /* [BH,N] original row -> permuted row */
    int32_t* q_offsets;   /* [BH,Cq+1] first permuted row of each query group */
    int32_t* kv_offsets;  /* [BH,Ck+1] */
    int32_t* n_groups;    /* [BH,2] (C_q', C_k') nonempty group counts */
    int32_t* kmeans_iters_run; /* [BH,2] assignments run (K/V, query) */
    float* q_centroid;    /* [BH,Cq,d] qbar_a: mean of raw query rows (B.3) */
    float* k_centroid;    /* [BH,Ck,d] kbar_b */
    float* v_centroid;    /* [BH,Ck,d] vbar_b */
    float* q_dist;        /* [BH,N] d_i = |phi_Q(q_i) - c_a| by original row (A.2) */
    /* optional */
    float* F_K;           /* [BH,d,RKp] key factor (columns beyond r_K' zero); RKp = d with
                             SPARSEPR_FLAG_SEMANTIC_KEYS, likewise RQp with SEMANTIC_QUERIES */
    float* F_Q;           /* [BH,d,RQp] query factor, RQp = min(rQ,d) rounded up to 16
                             (at least 32; columns beyond r_Q' zero) */
    float* phi_K;         /* [BH,N,RKp] key coordinates, RKp = r_K' rounded up to 16 (at least 32) */
    float* phi_Q;         /* [BH,N,RQp] query coordinates (after RMSNorm) */
    float* kv_centres;    /* [BH,Ck,RKp] k-means centres used by the last assignment */
    float* q_centres;     /* [BH,Cq,RQp] */
    /* optional, only with SPARSEPR_FLAG_DEBUG_EXPORT (small problems) */
    float* debug_kv_scores;   /* [BH,N,Ck] fp32 scores of the last K/V assignment */
    float* debug_q_scores;    /* [BH,N,Cq] */
    int32_t* debug_kv_hist;   /* [BH,kmeans_iters,N] raw labels after each assignment */
    int32_t* debug_q_hist;    /* [BH,kmeans_iters,N] */
} sparsepr_partition_out;

/* Outputs of sparsepr_route (paper §4.3, B.3, A.2). */
typedef struct {
    float* score;         /* [BH,Cq,Ck] s_ab (B.3), rows a<C_q', cols b<C_k' */
    uint8_t* mask;        /* [BH,Cq,Ck] z_ab */
    int32_t* sel_count;   /* [BH,Cq] number of selected K/V groups of group a */
    int32_t* sel_groups;  /* [BH,Cq,Ck] selected K/V groups of a, ascending, first sel_count */
    int64_t* pairs;       /* [BH,2] (P_route, P_exec = P_route + min(M,N)*N) */
    int32_t* probe_idx;   /* [BH,M'] probe rows (original index), M' = min(M,N); ordered by
                             group, then by (d_i, i) (stratified, or M >= N) or by index */
    int32_t* probe_group; /* [BH,M'] query group of each probe */
    float* probe_weight;  /* [BH,M'] w~_p (unit mean, A.3) */
    int32_t* probe_alloc; /* [BH,Cq] m_a probes per query group (for random and uniform
                             probes: the number that fall in the group) */
} sparsepr_route_out;

/* Outputs of sparsepr_probe_fit (paper §4.2, A.3). */
typedef struct {
    float* B;             /* [BH,d,d] B_lambda (row i, column j) */
    float* mu_x;          /* [BH,d] */
    float* sigma;         /* [BH,d] sqrt(weighted var + eps_std) */
    float* mu_r;          /* [BH,d] */
} sparsepr_fit_out;

/* Optional statistics of sparsepr_call. */
typedef struct {
    float ms_partition, ms_route, ms_attention, ms_fit, ms_apply, ms_total;
    int64_t pairs_route;    /* summed over heads */
    int64_t pairs_exec;     /* pairs_route + BH * min(M,N) * N */
    int64_t pairs_visited;  /* query-key pairs the attention tiles computed (incl. masked) */
    double rho_exec;        /* pairs_exec / (BH * N * N) */
    int64_t launches;       /* kernels this call launched (memsets and copies not counted) */
} sparsepr_stats;

/* Status text for a sparsepr_status value (static string). */
const char* sparsepr_status_string(int32_t status);

/* Host-side validation of *p; returns SPARSEPR_OK or the first failed check. */
sparsepr_status sparsepr_validate(const sparsepr_params* p);

/* Bytes of device workspace every entry point below needs for *p (0 if *p is
 * invalid).  The same workspace may be reused by successive calls on one
 * stream; calls on different streams need different workspaces. */
size_t sparsepr_workspace_size(const sparsepr_params* p);

/* §4.1: sampled-query key metric M_K, FP32 eigen-factor F_K, K/V k-means in
 * phi_K; centroids, M_Q, F_Q, phi_Q = RMSNorm(q F_Q), query k-means;
 * compaction to nonempty groups, group-major permutation and gather of
 * Q, K, V, q-bar/k-bar/v-bar and d_i.  Q, K, V: [BH,N,d] device, p->dtype. */
sparsepr_status sparsepr_partition(const sparsepr_params* p, const void* Q, const void* K,
                                   const void* V, const sparsepr_partition_out* part,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* State a warm-started partition starts from (paper C.1 "Warm start"): the
 * outputs of an earlier partition of the same *p (e.g. the previous denoising
 * step of the same layer).  DEVICE pointers, caller-owned, read only. */
typedef struct {
    const float* F_K;         /* [BH,d,RKp] that call's part->F_K */
    const float* F_Q;         /* [BH,d,RQp] that call's part->F_Q */
    const float* k_centroid;  /* [BH,Ck,d] that call's kbar_b */
    const float* q_centroid;  /* [BH,Cq,d] that call's qbar_a */
    const int32_t* n_groups;  /* [BH,2] that call's (C_q', C_k') */
} sparsepr_warm_state;

/* sparsepr_partition started from a previous call's state (paper C.1):
 *  - metric factors: two subspace iterations from the previous factor
 *    (Y = M Q, Q = Y L^-T with L L^T = Y^T Y), then F = Q C with
 *    C C^T = Q^T M Q (times 1/sqrt(d) for F_K), in place of the
 *    eigendecomposition.  A head whose Cholesky pivot vanishes (square not
 *    above 1e-12 x the largest diagonal entry), or whose previous F_Q has
 *    fewer nonzero columns than this call's r_Q', takes the cold factor.
 *  - k-means: initial centre b < C_k'(prev) of the K/V groups is kbar_b F_K,
 *    initial centre a < C_q'(prev) of the query groups is RMSNorm(qbar_a F_Q)
 *    (both TF32-rounded); later centres are the cold start's sampled rows.
 *    p->kmeans_iters is the limit of this call (Table C.1 uses 2 after the
 *    first call).
 * Every other step, output and error is that of sparsepr_partition.  `prev`
 * may point into `part` of the previous call: each previous value is read
 * before this call overwrites it.  Under GQA (p->Hkv) the state is per query
 * head, as the outputs are; K/V head h starts from query head h*G's F_K,
 * k_centroid and C_k'. */
sparsepr_status sparsepr_partition_warm(const sparsepr_params* p, const void* Q, const void* K,
                                        const void* V, const sparsepr_warm_state* prev,
                                        const sparsepr_partition_out* part, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* §4.3, B.3, A.2: routing scores, per-query-group prefix selection at the key
 * budget beta = (density - M/N) N, executed-pair counts, stratified probe
 * selection and coverage weights.  Reads the partition outputs. */
sparsepr_status sparsepr_route(const sparsepr_params* p, const sparsepr_partition_out* part,
                               const sparsepr_route_out* route, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Eq. (2) over the selected cells for every permuted query row, plus exact
 * dense attention for the probe rows.
 *   O_sp:         [BH,N,d] fp32, PERMUTED query order (row r = part->perm_q[r])
 *   probe_dense:  [BH,M',d] fp32, O^dense of each probe (route->probe_idx order)
 *   probe_sparse: [BH,M',d] fp32, O^sp of each probe */
sparsepr_status sparsepr_attention(const sparsepr_params* p, const sparsepr_partition_out* part,
                                   const sparsepr_route_out* route, float* O_sp,
                                   float* probe_dense, float* probe_sparse, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* §4.2 / A.3: coverage weights w_p = |G_a|/m_a (group sizes from
 * part->q_offsets, m_a from route->probe_alloc), weighted standardisation,
 * centring and the ridge solve B = (Xbar^T W Xbar + lambda I)^-1 Xbar^T W Rbar
 * on R = probe_dense - probe_sparse (Cholesky, fp64 internally).  A
 * non-positive pivot records SPARSEPR_NUMERIC in the device status word and
 * leaves B = 0.  p->correction selects a restricted family instead (D.4),
 * and p->residual_rank > 0 projects B onto the leading right singular
 * vectors of W^1/2 Rbar (fp32 Jacobi eigenvectors of Rbar^T W Rbar; D.3). */
sparsepr_status sparsepr_probe_fit(const sparsepr_params* p, const sparsepr_partition_out* part,
                                   const sparsepr_route_out* route, const float* probe_sparse,
                                   const float* probe_dense, const sparsepr_fit_out* fit,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Size in bytes of the static scratch array behind sparsepr_probe_fit_static
 * (8 MiB).  A call needs
 *   256 + r(4 BH) + r(24 BH d) + 2 r(8 BH d^2) bytes,  r(x) = x rounded up to 256,
 * which allows up to 31 heads (B*H) at d = 128 and 125 heads at d = 64. */
#define SPARSEPR_FIT_STATIC_SCRATCH_BYTES ((size_t)8 << 20)

/* sparsepr_probe_fit without a workspace (p->residual_rank must be 0:
 * the truncation needs workspace scratch; otherwise SPARSEPR_UNSUPPORTED).  The paper has no counterpart: it
 * exists for callers that hold the partition and routing results but cannot
 * allocate device memory where they run the fit -- a host framework whose
 * caching allocator has taken all free HBM, or a loop that must not take the
 * device-wide synchronisation of cudaMalloc/cudaFree.
 *
 * Same kernels, arguments and outputs as sparsepr_probe_fit, except that the
 * fit's scratch (fp64 weighted statistics, Gram matrices and right-hand
 * sides) lives in one static device array of SPARSEPR_FIT_STATIC_SCRATCH_BYTES
 * that every GPU loading the library holds until the process exits.  The
 * function allocates nothing and calls no allocating routine.
 *   device_status: optional caller-owned DEVICE int32 that receives
 *                  SPARSEPR_OK, or SPARSEPR_NUMERIC after a non-positive
 *                  Cholesky pivot (B is then 0), in stream order.
 * Errors: a call whose scratch exceeds the array returns SPARSEPR_UNSUPPORTED
 * before anything is launched; sparsepr_last_error_string() then gives the
 * bytes needed and the limit.  Other checks as sparsepr_probe_fit.
 * The first call on a device looks up the array's device address (which can
 * load the module); make that first call before any stream capture.  The
 * address is kept per device index for the life of the process and belongs
 * to the device context that was current at that first call: after
 * cudaDeviceReset, or anything else that destroys and re-creates the
 * device's primary context, the module may load at another address, so a
 * process that resets a device must not call this entry point on that
 * device again.
 * Every call on a device shares the array and finds the previous call's
 * contents there; each call clears the status word it needs zeroed, and the
 * rest is fully rewritten before it is read.  Calls whose work overlaps on
 * the GPU (different streams, or host threads without ordering) race on the
 * array and give undefined results. */
sparsepr_status sparsepr_probe_fit_static(const sparsepr_params* p, const sparsepr_partition_out* part,
                                          const sparsepr_route_out* route, const float* probe_sparse,
                                          const float* probe_dense, const sparsepr_fit_out* fit,
                                          int32_t* device_status, void* stream);

/* §4.2: O_out[b,h,i] = O^dense for probe rows, O^sp + mu_R + ((O^sp - mu_X)/sigma) B
 * otherwise, written in ORIGINAL query order.  O_out: [BH,N,d] fp32. */
sparsepr_status sparsepr_apply(const sparsepr_params* p, const sparsepr_partition_out* part,
                               const sparsepr_route_out* route, const float* O_sp,
                               const float* probe_dense, const sparsepr_fit_out* fit,
                               float* O_out, void* workspace, size_t workspace_bytes,
                               void* stream);

/* The whole call on one stream: partition -> route -> attention -> fit ->
 * apply.  O_out: [BH,N,d] fp32 original order.  With stats != NULL the call
 * records per-stage CUDA events, synchronises the stream and fills *stats. */
sparsepr_status sparsepr_call(const sparsepr_params* p, const void* Q, const void* K,
                              const void* V, float* O_out, sparsepr_stats* stats,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Name and message of the last CUDA error any entry point met on this host
 * thread ("no error" if none); valid until the next failing call. */
const char* sparsepr_last_error_string(void);

/* Reads (synchronously on `stream`) and clears the device status word of
 * `workspace`: *out = SPARSEPR_OK or the first device-side failure. */
sparsepr_status sparsepr_get_device_status(void* workspace, void* stream, int32_t* out);

/* Testing hook for the device-timeout path (no counterpart in the paper).
 * While polls > 0, every block of the tensor-core attention kernel launched
 * afterwards (by sparsepr_attention or sparsepr_call, from any host thread)
 * first waits at most `polls` polls on an mbarrier that nothing signals.  The
 * wait runs out like any bounded wait that gives up: the kernel records
 * SPARSEPR_TIMEOUT in the workspace status word, stops its other warps, lets
 * the copies and MMAs it issued finish, frees its tensor memory and returns,
 * and the blocks that start later return at once.  O_sp and the probe rows of
 * such a call are undefined.  polls = 0 (the default) turns the hook off.
 * Nothing else uses it; it exists so that tests can check that a timed-out
 * kernel leaves the context usable and the status readable. */
void sparsepr_debug_stall_attention(uint32_t polls);

#ifdef __cplusplus
}
#endif

#endif /* SPARSEPR_H */
