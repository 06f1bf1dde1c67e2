/*
 * svgear.h -- C ABI of the B200 clustered sparse attention library
 * (SVG-EAR's error-aware routing and centroid compensation on top of SVG2's
 * semantic-aware permutation).
 *
 * The layer, for every batch b and head h independently:
 *   1. k-means over the query tokens and, independently, over the key tokens
 *      (k-means++ seeding on a cold call, the caller's cached centroids on a
 *      warm call), returning labels, the permutation that makes every cluster
 *      contiguous, the segment offsets and the centroids;
 *   2. the permuted values and one mean value vector per key cluster;
 *   3. a per-(query cluster, key cluster) compensation-error probe and a
 *      greedy error-to-cost selection of blocks under a density budget;
 *   4. one attention pass that computes the selected blocks exactly and adds
 *      every skipped key cluster as its centroid weighted by its size, inside
 *      the same online softmax, writing O back in the original token order.
 *
 * Sources (page title, section):
 *   [TASK]   "SVG-EAR" task page (sotabase FrontierCS-2): the three routines
 *            -- one averages each cluster, one picks which cluster pairs to
 *            compute, one computes them and estimates the rest; the agent's
 *            steps 1-3 (k-means returning the sorted order, skipped clusters
 *            as one key at the centroid with its score raised by log n).
 *   [BLOG]   "SVG-EAR measured error" (frontier-cs.org blog): worked toy
 *            example, weight n*e^{s_bar}, the probe error sum, error per pair.
 *   [REVIEW] "SVG-EAR: Parameter-Free Linear Compensation for Sparse Video
 *            Generation via Error-aware Routing" (pith.science review): greedy
 *            error-to-cost routing under a density budget, O(Cq*Nk*d) probe.
 *   [SVG2]   "Sparse VideoGen2: Accelerate Video Generation with Sparse
 *            Attention via Semantic-Aware Permutation" (paper-graph summary),
 *            section 3.4: independent k-means on Q and K, permutation
 *            validity O = pi_q^T Attn(pi_q Q, pi_k K, pi_k V), k-means++ and
 *            the centroid cache, the dynamic block-size kernel.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers unless stated; the caller allocates every
 *     buffer (outputs and workspace) and keeps ownership.  The library never
 *     allocates device memory and keeps no state between calls, with two
 *     exceptions: the per-device tensor-memory guard (svgear_device_status)
 *     and the fixed scratch of svgear_label_sort_noalloc.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream) and is asynchronous: a return of SVGEAR_OK
 *     means the arguments were valid and the kernels launched.
 *   - Tensors are dense row-major with the head dimension d innermost:
 *     tokens X[B][H][N][d]; per-token ints [B][H][N]; centroids
 *     float[B][H][C][d]; segment offsets int32[B][H][C+1] holding positions
 *     0..N within the head.
 *   - dtype SVGEAR_F32 (float) or SVGEAR_BF16 (bfloat16) for token tensors;
 *     centroids and errors are always float.  d must be 64 or 128.
 *   - Errors: a negative svgear_status.  SVGEAR_ERR_INVALID_ARG for a null
 *     required pointer or sizes out of range, SVGEAR_ERR_UNSUPPORTED for a
 *     dtype / d / cluster count outside what the kernels implement,
 *     SVGEAR_ERR_WORKSPACE when ws_bytes is below svgear_workspace_bytes(),
 *     SVGEAR_ERR_CUDA when a launch fails (the CUDA error stays readable with
 *     cudaGetLastError).  Nothing is launched when validation fails.
 */
#ifndef SVGEAR_H
#define SVGEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SVGEAR_OK = 0,
    SVGEAR_ERR_INVALID_ARG = -1,
    SVGEAR_ERR_UNSUPPORTED = -2,
    SVGEAR_ERR_CUDA = -3,
    SVGEAR_ERR_TIMEOUT = -4,
    SVGEAR_ERR_WORKSPACE = -5,
    SVGEAR_ERR_SCRATCH_LIMIT = -6,
    SVGEAR_ERR_TMEM_LOST = -7
} svgear_status;

typedef enum { SVGEAR_F32 = 0, SVGEAR_BF16 = 1 } svgear_dtype;

/* Shape of one token tensor X[B][H][N][d]. */
typedef struct {
    int32_t B, H, N, d;
    int32_t dtype; /* svgear_dtype */
} svgear_dims;

/* Operation selector for svgear_workspace_bytes. */
typedef enum {
    SVGEAR_OP_CLUSTER = 0,
    SVGEAR_OP_KMEANSPP = 1,
    SVGEAR_OP_LABEL_SORT = 2,
    SVGEAR_OP_KMEANS_UPDATE = 3,
    SVGEAR_OP_ROUTE = 4,
    SVGEAR_OP_ATTEND = 5,
    SVGEAR_OP_KMEANS_ASSIGN = 6,
    SVGEAR_OP_ROUTE_TOPP = 7,
    SVGEAR_OP_CENTROIDS = 8
} svgear_op;

/* Largest cluster count any call accepts (shared-memory tables). */
#define SVGEAR_MAX_CLUSTERS 4096

/* --------------------------------------------------------------------------
 * svgear_cluster -- k-means over the tokens of every (b, h) and the
 * semantic-aware permutation ([SVG2] "The clustering operation", "The
 * permutation operation", "Fast k-means with centroid cache"; [TASK] step 1).
 *
 *   X               [B][H][N][d] tokens (dtype).
 *   C               clusters per head, 1 <= C <= min(N, SVGEAR_MAX_CLUSTERS).
 *   iters           rounds of (assign, update), >= 1.  The last round's
 *                   labels are final and its update gives the returned
 *                   centroids, so every non-empty centroid is exactly the
 *                   mean of its final members.
 *   warm_centroids  float[B][H][C][d] starting centroids (the previous
 *                   step's), or NULL for a cold start with k-means++ seeding
 *                   driven by Philox4x64-10 draws under `seed` (stream word =
 *                   b*H + h; see svgear_kmeanspp_init).
 *   labels          out int32[B][H][N]: argmin_c |x - c|^2, lowest c on ties.
 *   perm            out int32[B][H][N]: perm[p] = original token index at
 *                   permuted position p; stable in the original index.
 *   offsets         out int32[B][H][C+1]: cluster c occupies permuted
 *                   positions offsets[c] .. offsets[c+1]-1.
 *   centroids       out float[B][H][C][d]; an empty cluster keeps its
 *                   previous centroid.  May alias warm_centroids.
 *   Xp              out [B][H][N][d] (dtype) permuted copy X[perm], or NULL.
 *   ws, ws_bytes    workspace of svgear_workspace_bytes(SVGEAR_OP_CLUSTER); it
 *                   starts with the device status words of the bf16
 *                   assignment kernel (svgear_device_status).
 * ------------------------------------------------------------------------ */
int svgear_cluster(const void* X, svgear_dims dims, int32_t C, int32_t iters,
                   const float* warm_centroids, uint64_t seed, int32_t* labels,
                   int32_t* perm, int32_t* offsets, float* centroids, void* Xp,
                   void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * Sub-steps of svgear_cluster, exposed for stage-wise use and checking.
 * ------------------------------------------------------------------------ */

/* k-means++ seeding ([SVG2] "Fast k-means with centroid cache": k-means++
 * initialisation).  Draw j of head s = b*H + h is u_j = top 53 bits of the
 * first word of Philox4x64-10(counter = {j, s, 0, 0}, key = {seed, 0}) times
 * 2^-53.  Seed 0 is token floor(u_0 * N); seed j >= 1 is the smallest token
 * whose running sum of D^2 (squared distance to the nearest earlier seed,
 * fp32, summed in fp64) exceeds u_j * sum(D^2); if every D^2 is zero it is the
 * lowest token not chosen yet.  centroids[c] = X[seed_index[c]] as float.
 *   seed_index  out int32[B][H][C], or NULL.
 *   ws          svgear_workspace_bytes(SVGEAR_OP_KMEANSPP). */
int svgear_kmeanspp_init(const void* X, svgear_dims dims, int32_t C, uint64_t seed,
                         float* centroids, int32_t* seed_index, void* ws,
                         size_t ws_bytes, void* stream);

/* k-means assignment: labels[t] = argmin_c |x_t - c|^2, lowest c on exact
 * ties, evaluated with fp32-grade dot products: f32 tokens as |c|^2 - 2 x.c
 * by fp32 FMAs; bf16 tokens on the tensor cores as the argmax of
 * x.c - |c|^2/2, the fp32 centroid split into two bf16 planes (hi, lo) whose
 * products with the bf16 token are exact and accumulate in fp32 (what the
 * planes leave out is at most 2^-17 |c_k| per element: the worst-case
 * rounding of an fp32 dot product of length 128), and -|c|^2/2 added in the
 * same accumulation as three bf16 parts (held to 2^-24).
 *   ws  svgear_workspace_bytes(SVGEAR_OP_KMEANS_ASSIGN): the device status
 *       words (svgear_device_status), then the centroids re-laid for the
 *       kernel (planes and the norm parts). */
int svgear_kmeans_assign(const void* X, svgear_dims dims, const float* centroids,
                         int32_t C, int32_t* labels, void* ws, size_t ws_bytes,
                         void* stream);

/* Stable counting sort of labels ([TASK] step 1: the sorted order).
 *   labels   int32[B][H][N] in 0..C-1.
 *   perm     out int32[B][H][N]; offsets out int32[B][H][C+1].
 *   ws       svgear_workspace_bytes(SVGEAR_OP_LABEL_SORT) (dims.d and
 *            dims.dtype are ignored). */
int svgear_label_sort(const int32_t* labels, svgear_dims dims, int32_t C,
                      int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes,
                      void* stream);

/* k-means update: centroids[c] = mean of the tokens labelled c (fp32 sums in
 * a fixed order, so the result is deterministic); an empty cluster keeps the
 * value already in `centroids` (in/out).
 *   ws  svgear_workspace_bytes(SVGEAR_OP_KMEANS_UPDATE). */
int svgear_kmeans_update(const void* X, svgear_dims dims, const int32_t* labels,
                         int32_t C, float* centroids, void* ws, size_t ws_bytes,
                         void* stream);

/* --------------------------------------------------------------------------
 * svgear_permute -- Xp[p] = X[perm[p]] within every (b, h): the values share
 * the keys' permutation ([SVG2] "K and V share the same permutation").
 * ------------------------------------------------------------------------ */
int svgear_permute(const void* X, const int32_t* perm, svgear_dims dims, void* Xp,
                   void* stream);

/* --------------------------------------------------------------------------
 * svgear_centroids -- per-cluster mean of a permuted tensor in one pass
 * ([TASK] "one averages each cluster"; step 1: a small kernel averages each
 * cluster's values in one pass).
 *   Xp        [B][H][N][d] permuted tokens (dtype).
 *   offsets   int32[B][H][C+1] segments.
 *   centroids out float[B][H][C][d]; an empty segment gives zeros.
 *   ws        svgear_workspace_bytes(SVGEAR_OP_CENTROIDS, dims, C, 0): the
 *             partial sums of segments longer than one 512-position chunk.
 * The work is split by position (every CTA reads the same 512 rows,
 * whatever the cluster sizes); each segment is summed in fp32 in an order
 * fixed by the positions alone (rows of a chunk by lane group, groups in
 * order, chunks in order), so the result is the same from run to run.
 * ------------------------------------------------------------------------ */
int svgear_centroids(const void* Xp, const int32_t* offsets, int32_t C,
                     svgear_dims dims, float* centroids, void* ws, size_t ws_bytes,
                     void* stream);

/* --------------------------------------------------------------------------
 * svgear_probe -- compensation-error probe ([BLOG] probe paragraph; [REVIEW]
 * O(Cq*Nk*d) probe).  With s_it = scale * qbar_i . k_t, sbar_ic = scale *
 * qbar_i . kbar_c and m_i = max_t s_it over every key of the head:
 *   E[i][c] = sum_{t in K_c} | e^{sbar_ic - m_i} vbar_c - e^{s_it - m_i} v_t |^2
 * (fp32).  The shift m_i keeps the exponentials finite and leaves every
 * ranking within a row unchanged.  E is 0 for an empty key cluster.  Each
 * term is evaluated expanded around the key's residual w_t = v_t - vbar_c,
 * (a-b)^2 |vbar_c|^2 - 2 (a-b) b vbar_c.w_t + b^2 |w_t|^2 with a = e^{sbar-m},
 * b = e^{s-m} (the same quantity), summed in a fixed order.  One pass over
 * the keys: each cluster's sum is first taken with its own maximum score
 * m_ic as the shift, and then multiplied by e^{2 (m_ic - m_i)} with
 * m_i = max_c m_ic (every term is quadratic in e^{-m}).
 *   qbar      float[B][H][Cq][d] query centroids (the probes).
 *   Kp, Vp    [B][H][Nk][d] permuted keys and values (kdims.dtype).
 *   kbar,vbar float[B][H][Ck][d] key and value centroids.
 *   k_off     int32[B][H][Ck+1] key segments.
 *   kdims     shape of Kp (N = Nk).
 *   E         out float[B][H][Cq][Ck].
 *   ws        svgear_workspace_bytes(SVGEAR_OP_ROUTE, kdims, Cq, Ck) (holds the
 *             per-cluster maxima m_ic and the probes transposed in blocks of
 *             128).
 * ------------------------------------------------------------------------ */
int svgear_probe(const float* qbar, int32_t Cq, const void* Kp, const void* Vp,
                 const float* kbar, const float* vbar, const int32_t* k_off,
                 int32_t Ck, svgear_dims kdims, float scale, float* E, void* ws,
                 size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * svgear_route_select -- greedy error-to-cost selection ([REVIEW] greedy
 * routing under a density budget; [BLOG] error divided by the block's token
 * pairs, budget spent per query cluster).  For every non-empty query cluster
 * i: the key r_c = E[i][c] / n_c (one fp32 IEEE division; |Q_i| is constant
 * within the row) over the non-empty key clusters, ordered by r descending,
 * ties to the lower c, NaN last; c is taken if the keys taken so far plus n_c
 * stay within floor(density * Nk), else skipped, and the scan continues.
 *   pair_off  out int32[B][H][Cq+1]: row i's clusters are
 *             pair_kc[pair_off[i] .. pair_off[i+1]-1] (relative to the
 *             head's base B*H-index * Cq*Ck), ascending c.
 *   pair_kc   out int32[B][H][Cq*Ck].
 *   density   in (0, 1].
 *   ws        svgear_workspace_bytes(SVGEAR_OP_ROUTE, ...) suffices.
 * ------------------------------------------------------------------------ */
int svgear_route_select(const float* E, const int32_t* q_off, int32_t Cq,
                        const int32_t* k_off, int32_t Ck, int32_t B, int32_t H,
                        int32_t Nk, float density, int32_t* pair_off,
                        int32_t* pair_kc, void* ws, size_t ws_bytes, void* stream);

/* svgear_route -- probe + select in one call ([TASK] "one picks which cluster
 * pairs to compute").  E_out (float[B][H][Cq][Ck]) may be NULL, in which case
 * the errors live in the workspace (svgear_workspace_bytes(SVGEAR_OP_ROUTE)). */
int svgear_route(const float* qbar, const int32_t* q_off, int32_t Cq,
                 const float* kbar, const float* vbar, const int32_t* k_off,
                 int32_t Ck, const void* Kp, const void* Vp, svgear_dims kdims,
                 float density, float scale, int32_t* pair_off, int32_t* pair_kc,
                 float* E_out, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * svgear_topp_budget -- the per-query-cluster budget that holds p of the
 * estimated attention weight ([SVG2] section 3.4, "From pre-softmax scores to
 * attention probability estimates" and "Top-p selection for dynamic budget
 * allocation"; [BLOG] budget paragraph: the token pairs of the blocks that
 * hold 90% of the estimated weight).  For every non-empty query cluster i:
 *   S_ij  = scale * qbar_i . kbar_j
 *   P'_ij = n_j e^{S_ij} / sum_l n_l e^{S_il}        (n_j = |K_j|)
 * the non-empty key clusters in descending P' (ties: lower j), taken until
 * the running sum of P' reaches p (at least p); budget[i] = the keys of the
 * taken clusters (|Q_i| * budget[i] token pairs).  fp64 throughout, summed in
 * the sorted order; NaN scores take no part; an empty query cluster gets 0.
 *   qbar, kbar  float[B][H][Cq][d], float[B][H][Ck][d] centroids.
 *   q_off, k_off int32 segments ([B][H][Cq+1], [B][H][Ck+1]); Nk = keys.
 *   p           in (0, 1].
 *   budget      out int32[B][H][Cq].
 * No workspace; asynchronous on `stream`.
 * ------------------------------------------------------------------------ */
int svgear_topp_budget(const float* qbar, const int32_t* q_off, int32_t Cq,
                       const float* kbar, const int32_t* k_off, int32_t Ck, int32_t B,
                       int32_t H, int32_t d, int32_t Nk, float p, float scale,
                       int32_t* budget, void* stream);

/* svgear_route_select with a budget per query cluster: budget int32[B][H][Cq]
 * keys (e.g. from svgear_topp_budget) in place of floor(density * Nk); the
 * greedy, ordering and outputs are those of svgear_route_select.  ws as for
 * svgear_route_select. */
int svgear_route_select_budget(const float* E, const int32_t* q_off, int32_t Cq,
                               const int32_t* k_off, int32_t Ck, int32_t B, int32_t H,
                               int32_t Nk, const int32_t* budget, int32_t* pair_off,
                               int32_t* pair_kc, void* ws, size_t ws_bytes, void* stream);

/* svgear_route_topp -- probe + top-p budget + select in one call: SVG-EAR
 * spends the pairs of the blocks that hold p of the estimated weight on the
 * blocks with the most error per pair ([BLOG] budget paragraph).  E_out and
 * budget_out (int32[B][H][Cq]) may be NULL (then they live in the workspace,
 * svgear_workspace_bytes(SVGEAR_OP_ROUTE_TOPP, kdims, Cq, Ck)). */
int svgear_route_topp(const float* qbar, const int32_t* q_off, int32_t Cq,
                      const float* kbar, const float* vbar, const int32_t* k_off,
                      int32_t Ck, const void* Kp, const void* Vp, svgear_dims kdims,
                      float p, float scale, int32_t* pair_off, int32_t* pair_kc,
                      float* E_out, int32_t* budget_out, void* ws, size_t ws_bytes,
                      void* stream);

/* --------------------------------------------------------------------------
 * svgear_attend -- exact selected blocks plus centroid compensation in one
 * online softmax ([TASK] "one computes them and estimates the rest"; [BLOG]
 * weight n*e^{s_bar} and average value of a skipped cluster; [SVG2]
 * O = pi_q^T Attn(pi_q Q, pi_k K, pi_k V)).  For permuted query row p of
 * query cluster i and q = Qp[p]:
 *   num = sum_{c in S_i} sum_{u in K_c} e^{scale q.k_u} v_u
 *       + sum_{c not in S_i, n_c > 0} n_c e^{scale q.kbar_c} vbar_c
 *   den = the same sums with 1 in place of the value vectors
 *   O[q_perm[p]] = num / den          (O in the original token order).
 *   Qp        [B][H][Nq][d]; Kp, Vp [B][H][Nk][d] (all qdims.dtype).
 *   q_off     int32[B][H][Cq+1]; k_off int32[B][H][Ck+1].
 *   pair_off, pair_kc   from svgear_route / svgear_route_select.
 *   kbar,vbar float[B][H][Ck][d].
 *   q_perm    int32[B][H][Nq] (svgear_cluster's perm for the queries).
 *   O         out [B][H][Nq][d] (qdims.dtype).
 *   ws        svgear_workspace_bytes(SVGEAR_OP_ATTEND, qdims, Cq, Ck); holds
 *             bf16 centroid copies, the per-query-cluster key lists, the tile
 *             table and a device status word (svgear_attend_status).
 * bf16 runs on the tcgen05 tensor-core kernel; f32 on an fp32 SIMT kernel.
 * ------------------------------------------------------------------------ */
int svgear_attend(const void* Qp, const void* Kp, const void* Vp, svgear_dims qdims,
                  int32_t Nk, const int32_t* q_off, int32_t Cq, const int32_t* k_off,
                  int32_t Ck, const int32_t* pair_off, const int32_t* pair_kc,
                  const float* kbar, const float* vbar, const int32_t* q_perm,
                  float scale, void* O, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * svgear_key_variance -- per-coordinate variance of every key cluster ([BLOG]
 * variance paragraph: one variance per key coordinate, the coordinates'
 * co-movement ignored): kvar[c][k] = (1/n_c) sum_{t in K_c} (k_tk - mean_ck)^2
 * over the contiguous segment c of Kp (population variance, fp32, mean taken
 * first); an empty cluster gets 0.
 *   Kp     [B][H][Nk][d] permuted keys (kdims.dtype); k_off int32[B][H][Ck+1].
 *   kvar   out float[B][H][Ck][d].
 * No workspace; asynchronous on `stream`.
 * ------------------------------------------------------------------------ */
int svgear_key_variance(const void* Kp, const int32_t* k_off, int32_t Ck, svgear_dims kdims,
                        float* kvar, void* stream);

/* --------------------------------------------------------------------------
 * svgear_attend_var -- svgear_attend with variance-corrected compensation
 * ([BLOG] variance paragraph: the mean of e^{s_j} over a cluster is about
 * e^{sbar + sigma^2/2}; sigma^2 ~ scale^2 sum_k q_k^2 Var(k_k)).  Every
 * skipped cluster's log-weight gains
 *     lambda * scale^2 / 2 * sum_k q_k^2 kvar[c][k]
 * for each query row q (its own query, as the plain compensation uses);
 * lambda = 0 (or kvar = NULL) is exactly svgear_attend.
 *   kvar    float[B][H][Ck][d] (svgear_key_variance), nullable.
 *   lambda  finite strength of the term (the blog's runs use 0 to 1.5).
 * Other arguments, layouts, workspace and status word as svgear_attend.  On
 * the bf16 tensor-core path the term is one more MMA per compensation tile
 * with bf16 q^2 and bf16 lambda*scale/2*Var operands, and compensation tiles
 * then take 64 clusters each.
 * ------------------------------------------------------------------------ */
int svgear_attend_var(const void* Qp, const void* Kp, const void* Vp, svgear_dims qdims,
                      int32_t Nk, const int32_t* q_off, int32_t Cq, const int32_t* k_off,
                      int32_t Ck, const int32_t* pair_off, const int32_t* pair_kc,
                      const float* kbar, const float* vbar, const float* kvar, float lambda,
                      const int32_t* q_perm, float scale, void* O, void* ws, size_t ws_bytes,
                      void* stream);

/* --------------------------------------------------------------------------
 * svgear_probe_value_free -- the probe error without the values ([REVIEW]
 * minor comment 1 names a value-free error beside the value-aware one; its
 * formula is not printed there).  Reading:
 *   Ehat[i][c] = sum_{t in K_c} ( e^{sbar_ic - m_i} - e^{s_it - m_i} )^2
 * (the svgear_probe error when every value is the same unit vector; fp32).
 * Arguments, layouts and workspace as svgear_probe minus the values; the
 * result feeds svgear_route_select / svgear_route_select_budget like E.
 * ------------------------------------------------------------------------ */
int svgear_probe_value_free(const float* qbar, int32_t Cq, const void* Kp, const float* kbar,
                            const int32_t* k_off, int32_t Ck, svgear_dims kdims, float scale,
                            float* E, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * svgear_diagnostics -- how close a layer call came to dense attention, on
 * sampled query rows ([SVG2] section 3.1, attention recall under the oracle
 * policy; [REVIEW] Fig. 6a, attention MSE against full attention).  For each
 * sampled row p (a permuted position) of query cluster i:
 *   recall[r] = sum over the keys of i's selected clusters of e^{s_pu}
 *               / sum over every key of e^{s_pu}
 *   err2[r]   = | O[q_perm[p]] - O_dense(p) |^2,  ref2[r] = | O_dense(p) |^2
 * with O_dense(p) the dense softmax output (fp32, every key).
 *   Qp, Kp, Vp, q_off, k_off, pair_off, pair_kc, q_perm: as for svgear_attend.
 *   O      [B][H][Nq][d] the layer's output (qdims.dtype), original order.
 *   rows   int32[B][H][R] permuted row positions; R >= 0.
 *   recall, err2, ref2  out float[B][H][R] (NaN for a row out of range).
 * No workspace; asynchronous on `stream`.  A measurement, not part of the
 * layer: its cost is R * Nk * d multiply-adds per head.
 * ------------------------------------------------------------------------ */
int svgear_diagnostics(const void* Qp, const void* Kp, const void* Vp, svgear_dims qdims,
                       int32_t Nk, const int32_t* q_off, int32_t Cq, const int32_t* k_off,
                       int32_t Ck, const int32_t* pair_off, const int32_t* pair_kc, const void* O,
                       const int32_t* q_perm, float scale, const int32_t* rows, int32_t R,
                       float* recall, float* err2, float* ref2, void* stream);

/* Device status of the last svgear_cluster, svgear_kmeans_assign,
 * svgear_attend or svgear_selftest_wait that used `ws`: writes 4 int32 to
 * status[0..3] (host memory) and synchronises `stream`.  status[0] is 0 when
 * every wait in the tensor-core kernels completed, SVGEAR_ERR_TIMEOUT when a
 * bounded wait gave up (the kernel drained what it had issued and returned;
 * its outputs are not valid), SVGEAR_ERR_TMEM_LOST when a kernel refused to
 * start (below); status[1] and status[2] then say which wait
 * (site * 65536 + index; site 61 for the refusal) and which CTA
 * (blockIdx.y * 65536 + blockIdx.x).  These words sit at the start of the
 * workspace and each of those calls clears them first.
 * status[3] is 1 when the device's tensor memory is lost: a kernel gave up
 * while an MMA it had issued might still be running, so it could not free its
 * tensor memory, and on that SM no later tensor-core kernel could allocate
 * any.  Every tensor-core kernel checks a device word for this before it
 * allocates and returns SVGEAR_ERR_TMEM_LOST at once; once this call has seen
 * the word set, svgear_cluster and svgear_kmeans_assign on bf16 tokens and
 * svgear_attend(_var) on bf16 return SVGEAR_ERR_TMEM_LOST without launching.
 * The state lasts as long as the CUDA context (the process, or until a
 * device reset); nothing clears it.  The library's own extension, with no
 * counterpart in the method. */
int svgear_device_status(const void* ws, size_t ws_bytes, int32_t* status, void* stream);

/* The same as svgear_device_status (kept for svgear_attend callers). */
int svgear_attend_status(const void* ws, size_t ws_bytes, int32_t* status, void* stream);

/* svgear_selftest_wait -- the bounded device wait that every tensor-core
 * kernel uses, run on its own so that its give-up path can be checked
 * without disturbing a real kernel: one thread waits on a shared-memory
 * mbarrier that expects one arrival.  With arrive = 1 the thread makes that
 * arrival first and the wait completes; with arrive = 0 nothing arrives and
 * the wait gives up after timeout_us microseconds, recording
 * SVGEAR_ERR_TIMEOUT, site 60 and CTA 0 in the status words.  The kernel
 * allocates no tensor memory and issues no MMA or copy.  With mark_lost = 1 a
 * wait that gives up also sets the device's tensor-memory-lost word, as a
 * tensor-core kernel does when its final drain expires; every later
 * tensor-core call in this CUDA context then refuses to run (see
 * svgear_device_status), so use it only in a process of its own.
 *   ws          >= 16 bytes of device memory: the status words that
 *               svgear_device_status reads (cleared first).
 *   arrive, mark_lost   0 or 1.  timeout_us  1 .. 10,000,000.
 * A diagnostic with no counterpart in the method. */
int svgear_selftest_wait(void* ws, size_t ws_bytes, int32_t arrive, int32_t timeout_us,
                         int32_t mark_lost, void* stream);

/* --------------------------------------------------------------------------
 * svgear_label_sort_noalloc -- svgear_label_sort for callers that cannot give
 * the library any scratch memory: a framework whose memory planner owns all
 * device memory and forbids side allocations, a real-time loop in which
 * cudaMalloc (slow and synchronising) is off limits once running, or a plugin
 * interface that hands an operator only its inputs and outputs.  The paper
 * has no counterpart; this is an interface convenience.
 *
 * Same arguments and results as svgear_label_sort, minus the workspace: the
 * block histograms live in a fixed device array of
 * SVGEAR_NOALLOC_SORT_SCRATCH_INTS int32 (8 MiB) that every GPU which loads the
 * library keeps until the process exits.  B*H*ceil(N/1024)*C must not exceed
 * that count (the Wan 720p key sort, 40*74*500, fits); larger sizes return
 * SVGEAR_ERR_SCRATCH_LIMIT without launching.  No call allocates or frees
 * device memory.
 *   - The first call in each CUDA context -- on each device, and again after
 *     a device reset, which destroys the context and the array with it --
 *     looks up the array's device address (cudaGetSymbolAddress, with that
 *     device current); make that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (every entry a call reads is rewritten by that call first), so
 *     calls that overlap on the GPU -- on different streams, or from several
 *     threads -- race and corrupt each other's result; serialise them.
 * ------------------------------------------------------------------------ */
#define SVGEAR_NOALLOC_SORT_SCRATCH_INTS (2u * 1024u * 1024u)
int svgear_label_sort_noalloc(const int32_t* labels, svgear_dims dims, int32_t C,
                              int32_t* perm, int32_t* offsets, void* stream);

/* --------------------------------------------------------------------------
 * svgear_layer -- one whole layer call ([TASK] the layer and its three
 * routines, agent steps 1-3; [SVG2] section 3.4): svgear_cluster on Q (seed
 * 2*seed) and on K (seed 2*seed+1), svgear_permute of V by the key
 * permutation and svgear_centroids of the result, the probe and greedy
 * routing (svgear_route, or svgear_route_topp when topp > 0), the key
 * variance when var_lambda != 0, and svgear_attend(_var), which writes O in
 * the original token order.  Each stage's result is the one its own entry
 * point gives; every intermediate lives in the workspace.
 * ------------------------------------------------------------------------ */
typedef struct {
    int32_t Cq, Ck;     /* query / key clusters per head */
    int32_t iters;      /* Lloyd rounds of each clustering, >= 1 */
    float density;      /* floor(density * N) keys per query cluster, in (0, 1]
                           (unused when topp > 0) */
    float topp;         /* 0: fixed density; in (0, 1]: the budget of the key
                           clusters holding topp of the estimated weight */
    float scale;        /* softmax scale, finite (1/sqrt(d) for the method) */
    float var_lambda;   /* variance-corrected compensation strength; 0: plain */
    uint64_t seed;      /* k-means++ draws of a cold call */
} svgear_layer_params;

/* Workspace bytes of svgear_layer (host_buffers = 0) or svgear_layer_host
 * (host_buffers = 1); 0 for arguments the call would reject. */
size_t svgear_layer_workspace_bytes(svgear_dims dims, const svgear_layer_params* params,
                                    int32_t host_buffers);

/* The layer on device buffers.
 *   Q, K, V         [B][H][N][d] (dims.dtype), the same shape (self-attention).
 *   warm_q, warm_k  float [B][H][Cq][d] / [B][H][Ck][d] cached centroids of
 *                   the previous step, or NULL for a cold start (k-means++).
 *   O               out [B][H][N][d] (dims.dtype), original token order.
 *   cent_q, cent_k  out final centroids (the cache of the next step), or NULL;
 *                   each may alias its warm_ buffer.
 *   ws, ws_bytes    svgear_layer_workspace_bytes(dims, params, 0).
 *   stage_events    NULL, or 6 cudaEvent_t (NULL entries skipped) recorded on
 *                   `stream` before clustering Q, after clustering Q, after
 *                   clustering K, after the value centroids, after routing
 *                   and after attention: per-stage timing.
 * Status, validation and asynchrony as for the stage entry points; a stage's
 * error status ends the call with that status. */
int svgear_layer(const void* Q, const void* K, const void* V, svgear_dims dims,
                 const svgear_layer_params* params, const float* warm_q, const float* warm_k,
                 void* O, float* cent_q, float* cent_k, void* ws, size_t ws_bytes,
                 void* const* stage_events, void* stream);

/* The layer on HOST buffers: Q_host, K_host, V_host and O_host are host
 * memory of the shapes above (page-locked, for the copies to run
 * asynchronously and overlap the stages).  The call copies Q, K and V to the
 * workspace on a stream of its own, which first waits for all work already
 * on `stream`; each stage waits only for the input it reads, so clustering Q
 * runs while K and V are still arriving.  O is copied back into O_host on
 * `stream` after attention: O_host is complete once `stream` has passed this
 * call.  warm_q, warm_k, cent_q, cent_k are device pointers as for
 * svgear_layer; ws is svgear_layer_workspace_bytes(dims, params, 1). */
int svgear_layer_host(const void* Q_host, const void* K_host, const void* V_host,
                      svgear_dims dims, const svgear_layer_params* params, const float* warm_q,
                      const float* warm_k, void* O_host, float* cent_q, float* cent_k, void* ws,
                      size_t ws_bytes, void* stream);

/* Workspace bytes for `op` at shape `dims` (N = tokens of the clustered
 * tensor; for SVGEAR_OP_ROUTE and SVGEAR_OP_ATTEND, dims.N = Nq and C2 = Ck),
 * with C1 = C (or Cq).  Returns 0 for arguments the op would reject. */
size_t svgear_workspace_bytes(int32_t op, svgear_dims dims, int32_t C1, int32_t C2);

/* Static description of a status code. */
const char* svgear_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int32_t svgear_version(void);

/* Number of kernels this library has launched since it was loaded, over all
 * devices and threads (a host-side counter; no device synchronisation). */
uint64_t svgear_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* SVGEAR_H */
