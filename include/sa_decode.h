/*
 * sa_decode.h -- C ABI of libsa_b200.so: sparse single-token decode attention
 * over a long GQA KV cache, with the unread tail added back by a residual
 * estimator.  Built for NVIDIA B200 (sm_100a).
 *
 * One decode step of one unit u = (sequence b, KV head g) reads exactly
 *   I = attention sink [0, sink) + local window [L-local, L) + the k_blocks
 *       best 16-token blocks, ranked by sum_{h in group} q_h . kbar_c
 *       (kbar_c = mean key of block c),
 * and estimates the rest T (|T| = n_T) with one of
 *   SA_DROP    no estimate (plain sparse attention);
 *   SA_RESA    the RESA rank-1 prior: O_Est and the normaliser Z computed once
 *              at prefill end, bias (q - mu_Q) . mu_K / sqrt(d), merged in
 *              O(|I|) by removing the prior terms at I and adding the exact ones
 *              ("RESA: Bringing Back What Sparse Attention Ignores with Residual
 *              Estimation", Method, key designs 1 and 2);
 *   SA_PROXY   one virtual token: key = tail-mean K, value = tail-mean V,
 *              logit + ln n_T, tail sums = prefill totals minus the selected
 *              rows ("OpenAttention: One Percent Is Enough with Tail Proxies",
 *              abstract and method stage 04);
 *   SA_SAMPLE  b tail positions drawn uniformly with replacement, weighted
 *              n_T / b ("vAttention: Verified Sparse Attention via Sampling",
 *              Method, key design 1, paper eq. 3), b fixed or from the CLT
 *              budget of key designs 2-3.
 * With n_T = 0 every mode is exact dense attention.
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers to caller-owned memory (PyTorch tensors),
 *     16-byte aligned, dense row-major in the layouts stated below.  The
 *     library never allocates or frees device memory; scratch comes in `ws`.
 *   - `stream` is a cudaStream_t passed as void*; NULL = the legacy default
 *     stream.  Every call only enqueues work: no host synchronisation.
 *   - Argument errors return SA_ERR_INVALID_ARG / SA_ERR_UNSUPPORTED /
 *     SA_ERR_WORKSPACE before anything is launched; a failed launch returns
 *     SA_ERR_CUDA.  Nothing aborts or traps.
 *   - Workspace: size it with sa_workspace_size(); it must be ZERO-FILLED
 *     once when first allocated.  Each call leaves its completion counters at
 *     zero again, so the same buffer can be reused by later calls on the same
 *     stream.  Calls that share a workspace must not overlap on the GPU.
 *   - Outputs are fp32.  Results are deterministic: no floating-point
 *     atomics; partial results are combined in a fixed order.
 *
 * Layouts (dtype = shape.dtype for the cache and all queries)
 *   k, v        [B, Hkv, ld, d]      KV cache; tokens [0, L) are valid
 *   q_ctx       [B, Hq, L, d]        context queries (prefill only)
 *   q           [B, Hq, d]           decode queries of this step
 *   query head h belongs to KV head h / (Hq / Hkv).
 *   ld (shape.ld, 0 = L) is the cache's capacity in tokens per unit; the
 *   per-block arrays of sa_stats have ld / 16 rows per unit.  sa_append
 *   grows L by one token inside that capacity.
 */
#ifndef SA_DECODE_H
#define SA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SA_API __attribute__((visibility("default")))
#else
#define SA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer   */
    SA_ERR_UNSUPPORTED = 2,  /* a valid request this library does not handle */
    SA_ERR_WORKSPACE = 3,    /* ws NULL or smaller than sa_workspace_size()  */
    SA_ERR_CUDA = 4          /* a kernel launch failed                      */
} sa_status;

typedef enum { SA_F32 = 0, SA_BF16 = 1 } sa_dtype;

typedef enum { SA_DROP = 0, SA_RESA = 1, SA_PROXY = 2, SA_SAMPLE = 3 } sa_mode;

/* How sa_select ranks the candidate blocks of a KV head (all three on the
 * exact score rounded once, ties to the lower block index):
 *   SA_SCORE_MEAN_SUM  sum_{h in group} q_h . kbar_c (the group's summed
 *                      query against the block mean; the default)
 *   SA_SCORE_MEAN_MAX  max_{h in group} q_h . kbar_c (the group's strongest
 *                      head decides: the per-head alternative to one score
 *                      per KV head)
 *   SA_SCORE_QUEST     sum_h sum_e max(q_he min_ce, q_he max_ce) over the
 *                      block's elementwise key minimum and maximum (the
 *                      page-level upper-bound selector the RESA page's
 *                      related work wraps; needs blk_min / blk_max)
 * The two alternatives support up to 16384 candidate blocks per unit. */
typedef enum { SA_SCORE_MEAN_SUM = 0, SA_SCORE_MEAN_MAX = 1, SA_SCORE_QUEST = 2 } sa_score;

/* How the sampling budget b is set from the base sample when clt_base > 0
 * ("vAttention: Verified Sparse Attention via Sampling", Method, key designs
 * 2 and 3; the lemma b >= (Phi^-1(1 - delta_i/2) n_T sqrt(spread) / tau)^2
 * with tau = eps1 ||N_hat|| for the numerator, eps2 D_hat for the
 * denominator, and Lemma 4.2's 2 (eps1 + eps2) = eps, delta1 + delta2 =
 * delta):
 *   SA_BUDGET_CLT         even split: eps1 = eps2 = eps/4, delta1 = delta2 =
 *                         delta/2 (the default)
 *   SA_BUDGET_CLT_SEARCH  the split searched (Theorem 4.3's minimisation, its
 *                         formula not printed; read as): eps1 = f eps/2,
 *                         delta1 = g delta, f and g on {1/20, ..., 19/20}
 *                         (eps2 < 0.5), the smallest max over heads and
 *                         bounds, ties to the first (f, g) in order
 *   SA_BUDGET_HOEFFDING   the conservative bound (the page's appendix
 *                         remark), even split: b_D = n_T^2 ln(2/delta2) R_D^2
 *                         / (2 tau_D^2), b_N = d n_T^2 ln(2d/delta1) max_e
 *                         R_e^2 / (2 tau_N^2), R the base sample's ranges of
 *                         the weights e and of each coordinate of e V        */
typedef enum { SA_BUDGET_CLT = 0, SA_BUDGET_CLT_SEARCH = 1, SA_BUDGET_HOEFFDING = 2 } sa_budget;

typedef enum {
    SA_OP_PREFILL = 0,   /* sa_prefill_stats */
    SA_OP_SELECT = 1,    /* sa_select        */
    SA_OP_DECODE = 2,    /* sa_decode        */
    SA_OP_DENSE = 3,     /* sa_dense_decode  */
    SA_OP_STEP = 4,      /* sa_step          */
    SA_OP_MULTI = 5,     /* sa_multi_step    */
    SA_OP_CLUSTER = 6    /* sa_cluster_build */
} sa_op;

/* Supported: d in {64, 128}; Hq % Hkv == 0 with G = Hq/Hkv in {1,2,4,8};
 * L >= 16 (a multiple of 16 for sa_prefill_stats, whose statistics cover
 * whole blocks); ld = 0 (meaning ld = L) or a multiple of 16 with
 * L <= ld < 2^31 / d; B, Hkv >= 1.  A length L that is not a multiple of 16
 * needs ld given.  Only the complete blocks [0, L/16) are candidates for
 * selection, and a partial last block lies in the local window when
 * local >= 16. */
typedef struct {
    int B, Hq, Hkv, d, L;
    sa_dtype dtype;
    int ld;
} sa_shape;

/* Prefill-end statistics, written by sa_prefill_stats, read by sa_select and
 * sa_decode.  All caller-allocated (RESA page, key design 1: "computed once at
 * prefill end").
 *   mu_q        [B, Hq, d]   f32  typical query: mean of the L context queries
 *   o_est       [B, Hq, d]   f32  sum_j softmax_j(s mu_q . K_j) V_j
 *   log_z0      [B, Hq]      f32  ln sum_j exp(s mu_q . K_j)  (no bias)
 *   mu_k        [B, Hkv, d]  f32  typical key: mean of the L cached keys
 *   sum_k       [B, Hkv, d]  f32  sum of the L cached keys
 *   sum_v       [B, Hkv, d]  f32  sum of the L cached values
 *   blk_mean    [B, Hkv, ld/16, d] in dtype: 16-token block means, summed in
 *               fp64 and rounded once (nearest, ties to even)
 *   kbar_absmax [B, Hkv]     f32  max |blk_mean| (reported; not needed by
 *               sa_select)
 *   blk_code    [B, Hkv, ld/16, d] int8 and
 *   blk_meta    [B, Hkv, ld/16, 4] f32: the scan sketch of blk_mean relative
 *               to mu_k, written with it.  Per block row kbar, t = kbar - mu_k
 *               (fp64), s = fl32(max_e |t_e| / 127), code_e = clamp(rint(t_e /
 *               s), -127, 127) (0 when s = 0), meta = {s, rn, kn, 0} with
 *               rn >= ||t - s code||_2 and kn >= ||s code||_2 (f32 upper
 *               bounds).  Centring shifts every block's score by one constant,
 *               so the ranking is unchanged.  sa_select ranks the blocks on the
 *               sketch with these bounds and certifies the top-k exactly from
 *               blk_mean, so the selection equals the one on blk_mean alone; a
 *               sketch not built from this blk_mean and mu_k (rebuild it with
 *               sa_block_sketch when either changes) makes it wrong.  The
 *               selector's own data structure: the pages have no counterpart.
 *   blk_min, blk_max [B, Hkv, ld/16, d] in dtype, or both NULL: the
 *               elementwise minimum and maximum of each block's keys (the
 *               summaries of SA_SCORE_QUEST); written by sa_prefill_stats,
 *               sa_block_minmax and sa_append when not NULL. */
typedef struct {
    float* mu_q;
    float* o_est;
    float* log_z0;
    float* mu_k;
    float* sum_k;
    float* sum_v;
    void* blk_mean;
    float* kbar_absmax;
    int8_t* blk_code;
    float* blk_meta;
    void* blk_min;
    void* blk_max;
} sa_stats;

/* The OpenAttention multi-proxy state of a cache ("OpenAttention: One
 * Percent Is Enough with Tail Proxies", method overview stages 01-04), per
 * unit (sequence b, KV head g), caller-allocated:
 *   n_clusters  C, 1..64 (the page's C = 64)
 *   basis       [B, Hkv, 32, d] f32: rows = the eigenvectors of the second
 *               moment of the unit's context queries, decreasing eigenvalue
 *               (the QGS basis, r = 32; its first 16 rows the clustering
 *               basis); written by sa_cluster_build or by the caller
 *   assign      [B, Hkv, ld] uint8: each token's cluster (k-means of the keys
 *               projected on the first 16 rows); sa_cluster_build or caller
 *   order       [B, Hkv, ld] int32: the token positions grouped by cluster
 *               (cluster 0's members in ascending position, then cluster
 *               1's, ...); written by sa_cluster_prep
 *   start       [B, Hkv, C + 1] int32: cluster c's members are
 *               order[start[c] .. start[c + 1]); written by sa_cluster_prep
 *   codes       [B, Hkv, ld, 32] int8 and scales [B, Hkv, ld] f32: the QGS
 *               codes of each key, z = basis . K_j (exact sums rounded once),
 *               sigma = fl32(max |z| / 127), code = clamp(rint(z / sigma),
 *               +-127), stored in the order of `order` (row i holds token
 *               order[i], so that a cluster's codes are contiguous); written
 *               by sa_cluster_prep
 *   count       [B, Hkv, C] int32 and sum_k, sum_v, sum_k2 [B, Hkv, C, d] f32:
 *               per cluster the member count and the sums of keys, values and
 *               squared keys (the cached mean and diagonal variance);
 *               written by sa_cluster_prep
 * Pointers non-null and 16-byte aligned. */
typedef struct {
    int n_clusters;
    float* basis;
    uint8_t* assign;
    int8_t* codes;
    float* scales;
    int32_t* count;
    float* sum_k;
    float* sum_v;
    float* sum_k2;
    int32_t* order;
    int32_t* start;
} sa_clusters;

/* Which tokens one step reads exactly, and how the tail is sampled.
 *   sink, local   >= 0: first / last tokens always read (vAttention page,
 *                 overall framework: sink + local window + top-k)
 *   k_blocks      >= 0: blocks chosen per unit among those disjoint from the
 *                 sink and the window (fewer if fewer candidates exist)
 *   sample_b      draws per unit for SA_SAMPLE when clt_base == 0
 *   clt_base      > 0: choose b per unit by the CLT budget (vAttention, key
 *                 designs 2-3) from the first clt_base draws, target (eps,
 *                 delta) on the output split evenly between numerator and
 *                 denominator (Lemma 4.2), b clamped to [clt_base, min(n_T,
 *                 sample_cap)]; requires 2 <= clt_base <= min(256,
 *                 sample_cap), eps > 0, 0 < delta < 1 and k, v in sa_select;
 *                 0: fixed sample_b
 *   sample_cap    capacity per unit of sa_selection.samp_idx (>= sample_b)
 *   seed, step    SplitMix64 stream of unit (b, g) at this step:
 *                 key = out(out(out(out(seed)^b)^g)^step), draw i =
 *                 out(key + i*0x9E3779B97F4A7C15), out(x) = SplitMix64 mixer
 *                 of x + 0x9E3779B97F4A7C15; rank = ((draw>>32)*n_T)>>32
 *   score         block score, an sa_score (0 = SA_SCORE_MEAN_SUM)
 *   budget        rule for b when clt_base > 0, an sa_budget (0 = the even
 *                 CLT split)
 *   per_head      0: one draw stream and one budget per KV head, shared by
 *                 its query heads; 1: one per query head (the vAttention
 *                 page samples and budgets per head): query head hq of
 *                 sequence b draws from the stream of (seed, b, hq, step),
 *                 its budget from its own base sample, and the decode
 *                 weights each head's draws by n_T / b_hq for that head
 *                 alone; sa_selection's samp_idx / samp_count then have
 *                 B * Hq rows                                                 */
typedef struct {
    int sink, local, k_blocks;
    int sample_b, clt_base, sample_cap;
    float eps, delta;
    uint64_t seed;
    int step;
    int score;
    int budget;
    int per_head;
} sa_select_params;

/* Output of sa_select, input of sa_decode (caller-allocated).
 *   blk_idx     [B, Hkv, k_blocks] int32: chosen block indices, ascending;
 *               min(k_blocks, n_cand) valid entries per unit, rest = -1
 *   samp_idx    [B, Hkv, sample_cap] int32 ([B, Hq, sample_cap] with
 *               per_head): drawn token positions (draw order)
 *   samp_count  [B, Hkv] int32 ([B, Hq] with per_head): draws per stream
 *               (0 unless sampling)
 *   n_rescored  [B, Hkv] int32 or NULL: candidates whose sketch interval
 *               reached the k-th best lower bound and were rescored exactly
 *               (0 when the sketch alone decided; diagnostic)                */
typedef struct {
    int32_t* blk_idx;
    int32_t* samp_idx;
    int32_t* samp_count;
    int32_t* n_rescored;
} sa_selection;

/* mode; lambda = prior weight of SA_RESA in [0,1] (1 = the RESA page's
 * merge, 0 = plain sparse attention); scale = softmax scale (0 = 1/sqrt(d)). */
typedef struct {
    sa_mode mode;
    float lambda;
    float scale;
} sa_decode_params;

/* Bytes of zero-initialised scratch the op needs for this shape (params may
 * be NULL for SA_OP_PREFILL and SA_OP_DENSE).  0 on invalid arguments. */
SA_API size_t sa_workspace_size(const sa_shape* shape, const sa_select_params* params, int op);

/* Prefill-end statistics (RESA page, key design 1: mu_Q, mu_K, O_Est and Z
 * as one extra query at prefill end; OpenAttention stage 04: totals for the
 * tail means; block means for the selector).  Reads q_ctx once and k, v once.
 * scale = softmax scale (0 = 1/sqrt(d)). */
SA_API sa_status sa_prefill_stats(const sa_shape* shape, const void* q_ctx, const void* k,
                           const void* v, const sa_stats* out, float scale,
                           void* ws, size_t ws_bytes, void* stream);

/* Block means of blocks [blk_begin, blk_end) of every unit into blk_mean
 * ([B, Hkv, ld/16, d], dtype; blk_end <= L/16), their sketch relative to
 * mu_k ([B, Hkv, d] f32,
 * read only) into blk_code / blk_meta (layouts of sa_stats), and raises
 * kbar_absmax [B, Hkv] to cover them (for a cache that grew by whole blocks;
 * keep mu_k as it was when the other rows were sketched).  No workspace. */
SA_API sa_status sa_block_summaries(const sa_shape* shape, const void* k, int blk_begin, int blk_end,
                                    void* blk_mean, float* kbar_absmax, const float* mu_k, int8_t* blk_code,
                                    float* blk_meta, void* stream);

/* Appends one token per unit at position L = shape->L of a cache with room
 * for it (L < ld): k[b, g, L, :] = k_new[b, g, :] and v likewise (k_new,
 * v_new [B, Hkv, d] in dtype), and refreshes the statistics so that they
 * describe the L + 1 tokens:
 *   sum_k += k_new, sum_v += v_new (the totals behind the tail means of
 *   SA_PROXY, OpenAttention stage 04);
 *   per query head h of the unit, with p = s mu_q,h . k_new (fp32):
 *     log_z0' = ln(exp(log_z0) + exp(p)),
 *     o_est'  = exp(log_z0 - log_z0') o_est + exp(p - log_z0') v_new,
 *   so that O_Est and Z stay the typical query's attention over the whole
 *   cache (RESA, key design 1), which SA_RESA's tail estimate subtracts the
 *   read set from;
 *   when the token completes block c = (L + 1)/16 - 1: blk_mean[c], its
 *   sketch row and kbar_absmax, as sa_block_summaries for that block, and
 *   blk_min[c] / blk_max[c] when the stats carry them.
 * mu_q and mu_k stay as computed at prefill end (the RESA page fixes the
 * typical query and key there; mu_k is also the sketch's centre, which must
 * not move while rows sketched against it remain).  After the call the
 * cache holds L + 1 tokens: later calls pass L + 1.  scale = softmax scale
 * (0 = 1/sqrt(d)).  No workspace; one kernel. */
SA_API sa_status sa_append(const sa_shape* shape, const void* k_new, const void* v_new, void* k, void* v,
                           const sa_stats* stats, float scale, void* stream);

/* Elementwise key minimum and maximum of blocks [blk_begin, blk_end) of every
 * unit (blk_end <= L/16) into blk_min / blk_max ([B, Hkv, ld/16, d], dtype):
 * the per-block key bounds of SA_SCORE_QUEST (Quest's page summaries, which
 * the RESA page's related work names).  sa_prefill_stats writes them for
 * every block when the stats carry the two pointers; this call covers blocks
 * written later.  No workspace. */
SA_API sa_status sa_block_minmax(const sa_shape* shape, const void* k, int blk_begin, int blk_end, void* blk_min,
                                 void* blk_max, void* stream);

/* Rebuilds the sketch (blk_code, blk_meta) of blocks [blk_begin, blk_end) of
 * every unit from blk_mean relative to mu_k, for callers that write blk_mean
 * or mu_k themselves (sa_prefill_stats and sa_block_summaries already write
 * the sketch).  No workspace.  The pages have no counterpart (see blk_code in
 * sa_stats). */
SA_API sa_status sa_block_sketch(const sa_shape* shape, const void* blk_mean, const float* mu_k, int blk_begin,
                                 int blk_end, int8_t* blk_code, float* blk_meta, void* stream);

/* Selection of one decode step for every unit: block scores, exact top-k by
 * (score desc, block index asc) on the exact score rounded once to fp64, and
 * the tail draws for sampling.  With SA_SCORE_MEAN_SUM the scan reads the
 * int8 sketch (integer dot products with an int8 copy of the group query)
 * and bounds each score's error; every candidate whose interval reaches the
 * k-th best lower bound is rescored exactly from blk_mean.  The other scores
 * scan blk_mean (or blk_min and blk_max) in fp32 with the same certified
 * intervals and exact rescoring of the band.  k and v are read only for the CLT base sample (may be NULL
 * when clt_base == 0). */
SA_API sa_status sa_select(const sa_shape* shape, const sa_select_params* params, const void* q,
                    const sa_stats* stats, const void* k, const void* v,
                    const sa_selection* out, float scale, void* ws, size_t ws_bytes,
                    void* stream);

/* sa_select without a workspace, for callers that cannot allocate device
 * memory (for example code that runs inside an allocator's hooks or in a
 * plug-in restricted to the buffers it is given).  The paper has no
 * counterpart: this is a deployment convenience.  Same inputs, outputs and
 * results as sa_select; the scratch is a fixed 8 MiB array inside the
 * library (present on every device that loads it), so shapes whose
 * selection workspace exceeds 8 MiB return SA_ERR_WORKSPACE.  The arguments
 * are checked first, exactly as sa_select checks them; a rejected call
 * enqueues nothing.  The array is shared by all calls on a device: an
 * accepted call clears its completion counters with cudaMemsetAsync on
 * `stream` first, and calls that overlap on the GPU race and must not be
 * issued.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  Allocates nothing. */
SA_API sa_status sa_select_noalloc(const sa_shape* shape, const sa_select_params* params, const void* q,
                                   const sa_stats* stats, const void* k, const void* v,
                                   const sa_selection* out, float scale, void* stream);

/* Sparse decode: gathers I (and the draws), one fp32 online softmax over the
 * G query heads of each unit, folds in the mode's residual, writes
 * out [B, Hq, d] f32. */
SA_API sa_status sa_decode(const sa_shape* shape, const sa_decode_params* dparams,
                    const sa_select_params* sparams, const void* q, const void* k,
                    const void* v, const sa_stats* stats, const sa_selection* sel,
                    float* out, void* ws, size_t ws_bytes, void* stream);

/* One whole decode step: sa_select then sa_decode on the same stream, the
 * decode launched as a programmatic dependent of the selection, so that its
 * CTAs stream the sink and window rows (which do not depend on the selection)
 * while the selection finishes, and wait for it (griddepcontrol.wait) before
 * reading the chosen blocks and draws.  Same arguments, layouts and results
 * as the two calls in sequence; scale = dparams->scale; the workspace is
 * sa_workspace_size(..., SA_OP_STEP) bytes (selection part first). */
SA_API sa_status sa_step(const sa_shape* shape, const sa_decode_params* dparams,
                         const sa_select_params* sparams, const void* q, const void* k, const void* v,
                         const sa_stats* stats, const sa_selection* sel, float* out, void* ws,
                         size_t ws_bytes, void* stream);

/* Query-geometry clustering of the cache at prefill end (OpenAttention,
 * method stage 01, QGC), for every unit: unless basis_given, the second
 * moment M = (1/(G L)) sum q q^T of the unit's context queries q_ctx
 * [B, Hq, L, d] and its 32 leading eigenvectors into cl->basis (subspace
 * iteration with CholeskyQR2 in fp64, ordered by Rayleigh quotient); then
 * k-means of the keys projected on the first 16 basis rows into cl->assign
 * (centroid c starts at the projection of token floor(c L / C); 10 rounds of
 * nearest centroid, lowest index on ties, and member means, an empty
 * cluster's centroid kept; a last assignment); then sa_cluster_prep.
 * basis_given = 1 keeps the caller's basis (q_ctx unused, may be NULL).
 * Workspace: sa_workspace_size(.., SA_OP_CLUSTER), zero-filled once. */
SA_API sa_status sa_cluster_build(const sa_shape* shape, const void* q_ctx, const void* k, const void* v,
                                  const sa_clusters* cl, int basis_given, void* ws, size_t ws_bytes, void* stream);

/* The per-cluster state that follows from basis and assign over tokens
 * [0, L): the cluster order and starts, the QGS codes and scales, the counts
 * and the sums (layouts of sa_clusters).  Prefill-time; no workspace. */
SA_API sa_status sa_cluster_prep(const sa_shape* shape, const void* k, const void* v, const sa_clusters* cl,
                                 void* stream);

/* One decode step of the multi-proxy pipeline (OpenAttention, method
 * stages 02-04) for every unit:
 *   ErrorGate: per cluster and query head of the group the member-logit mean
 *   mu = s q_h . Kbar and variance s^2 sum_e q_he^2 var_e (diagonal); the
 *   proxy's weight error n e^mu (e^(var/2) - 1) over the head's estimated
 *   mass sum n e^(mu + var/2), summed over the heads, made integers
 *   w = rint(2^30 err / max err); the budget E = min(budget, L) split as
 *   q_c = min(n_c, floor(E w_c / W)) and the rest one token at a time by
 *   largest remainder (E w_c mod W), lower cluster first, round after round;
 *   QGS: every token's score fl32(sigma_j (qq . code_j)), qq = the group's
 *   projected query p = basis . sum_h q_h coded to 16 bits (sq = max|p| /
 *   32767, qq = rint(p / sq)); each cluster reads its q_c best tokens by
 *   (score desc, position asc);
 *   stage 04: one softmax over the read tokens' exact logits and, per cluster
 *   with n' = n_c - q_c > 0 unread members, one proxy of logit s q . Kbar' +
 *   ln n' and value Vbar' (means over the unread members: the cluster's sums
 *   minus the read rows').
 * read [B, Hkv, budget] int32 gets the read positions grouped by cluster
 * (cluster order, ascending positions; -1 after the last), read_count
 * [B, Hkv, C] int32 the q_c, out [B, Hq, d] f32 the output.  scale = softmax
 * scale (0 = 1/sqrt(d)).  Workspace: sa_workspace_size(.., SA_OP_MULTI). */
SA_API sa_status sa_multi_step(const sa_shape* shape, const void* q, const void* k, const void* v,
                               const sa_clusters* cl, int budget, float scale, int32_t* read, int32_t* read_count,
                               float* out, void* ws, size_t ws_bytes, void* stream);

/* Dense flash-decode over all L tokens (the in-build speed reference, not
 * part of the method): out [B, Hq, d] f32 = softmax(s q K^T) V. */
SA_API sa_status sa_dense_decode(const sa_shape* shape, const void* q, const void* k, const void* v,
                          float* out, float scale, void* ws, size_t ws_bytes, void* stream);

/* Bounded waits.  The selection kernel streams the block summaries into
   shared memory with bulk copies and waits on each one for at most about two
   seconds; a CTA whose wait runs out marks its unit's selection invalid
   (blk_idx row all -1, samp_count 0, n_rescored -1) and returns.  *count gets
   the number of such CTAs on the current device since the library was loaded
   (cumulative; compare two readings).  Synchronous with respect to the device
   (it reads a device counter).  The method has no counterpart: this is the
   library's guard against a copy that never lands. */
SA_API sa_status sa_wait_timeouts(unsigned* count);

/* Static string for a status code. */
SA_API const char* sa_status_string(sa_status status);

#ifdef __cplusplus
}
#endif
#endif /* SA_DECODE_H */
