/*
 * ear.h - C ABI of libear, the B200 (sm_100a) SVG-EAR attention hot path.
 *
 * The method is SVG-EAR ("SVG-EAR: Parameter-Free Linear Compensation for
 * Sparse Video Generation via Error-aware Routing", arXiv 2603.08982); the
 * section cited beside each entry point defines what it computes.
 *
 * One attention layer runs five calls, in this order, for all (batch, head)
 * slices at once ("BH" slices):
 *   ear_kmeans(Q), ear_kmeans(K)       cluster queries and keys
 *   ear_permute(Q), (K)                make each cluster contiguous
 *   ear_permute_apply(V, K's perm)     V in K's order, also producing v̄
 *   ear_probe                          per-block compensation-error estimate
 *   ear_route                          greedy error-to-cost block selection
 *   ear_attention                      block-sparse exact attention plus
 *                                      centroid compensation, one softmax
 * or, with no permuted copy of Q, K or V (the gathered layer):
 *   ear_kmeans(Q), ear_kmeans(K); ear_permute(Q), (K) without X (perm and
 *   offsets only); ear_permute_apply(V, K's perm) with X_perm = NULL (v̄
 *   only); ear_probe_gather; ear_route; ear_attention_gather.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every array pointer is a DEVICE pointer owned by the caller, contiguous,
 *    16-byte aligned, row-major.  The library keeps no pointer after a call
 *    returns and allocates no device or host memory.
 *  - Token matrices are [BH][N][d]; d is 64 or 128.  Element type is given by
 *    an ear_dtype: EAR_F32 (float) or EAR_BF16 (bfloat16 bits, uint16).
 *  - Scratch memory is passed as (ws, ws_bytes); its required size comes from
 *    ear_workspace_bytes().  Contents need not be initialised and are
 *    clobbered.  Two calls that run concurrently need separate workspaces.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *    void*; NULL = the legacy default stream).  Outputs are valid once the
 *    stream reaches the call.
 *  - Host-side validation runs first.  On any error other than EAR_OK the
 *    call launches nothing and writes no output.  EAR_ERR_CUDA means a CUDA
 *    runtime call failed; work enqueued before it by the same call may have
 *    run.
 *  - Device-side faults that validation cannot see (a label out of range, an
 *    offset table that is not monotone, a bounded wait that ran out) do not
 *    trap: the kernel skips the bad item and latches an error code in a
 *    per-device status word, read and cleared by ear_get_device_status().
 *  - N < 2^31 and every cluster count C <= 65536.
 *  - The library is thread-compatible: calls on different streams may run
 *    from different host threads.
 */
#ifndef EAR_H_
#define EAR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EAR_API __attribute__((visibility("default")))
#else
#define EAR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  EAR_OK = 0,
  EAR_ERR_ARG = 1,          /* null pointer, bad size or value; nothing launched     */
  EAR_ERR_UNSUPPORTED = 2,  /* well-formed but outside what is built (d, dtype, C)   */
  EAR_ERR_WORKSPACE = 3,    /* ws_bytes smaller than ear_workspace_bytes() says      */
  EAR_ERR_CUDA = 4,         /* a CUDA runtime call failed                            */
  EAR_ERR_TIMEOUT = 5,      /* device status: a bounded device-side wait ran out     */
  EAR_ERR_DEVICE = 6        /* device status: an input index/offset was out of range */
} ear_status;

typedef enum { EAR_F32 = 0, EAR_BF16 = 1 } ear_dtype;

typedef enum {
  EAR_OP_KMEANS = 0,
  EAR_OP_PERMUTE = 1,
  EAR_OP_PROBE = 2,
  EAR_OP_ROUTE = 3,
  EAR_OP_ATTENTION = 4,
  EAR_OP_ROUTE_ROWS = 5
} ear_op;

/* ear_attention flags */
#define EAR_COMPENSATE 1 /* fold skipped blocks in through their centroids (SVG-EAR §4.3);
                            without it skipped blocks are dropped (the §3.1 baseline)    */

/* Static string naming a status code. */
EAR_API const char* ear_status_string(ear_status s);

/*
 * Scratch bytes an entry point needs for the given sizes.
 *   op = EAR_OP_KMEANS:  rows N = n_q, clusters C = c_q   (n_k, c_k ignored)
 *   op = EAR_OP_PERMUTE: rows N = n_q, clusters C = c_q   (n_k, c_k ignored)
 *   op = EAR_OP_PROBE / ROUTE / ATTENTION: all sizes as in those calls.
 *   op = EAR_OP_ROUTE_ROWS: bh and c_q (the rest ignored).
 * Returns EAR_ERR_ARG for negative sizes or a null `bytes`.
 */
EAR_API ear_status ear_workspace_bytes(ear_op op, int64_t bh, int64_t n_q, int64_t n_k, int32_t d,
                               int32_t c_q, int32_t c_k, size_t* bytes);

/*
 * Lloyd k-means of every slice's N rows into C clusters (SVG-EAR §4.1: Q and K
 * are clustered with "flash k-means"; q̄_i / k̄_j is the mean token of the
 * cluster holding i / j).
 *   X          [BH][N][d] dtype       rows to cluster
 *   init       [BH][C][d] float       initial centroids (e.g. C seeded rows of X)
 *   centroids  [BH][C][d] float  out  means of the final members; an empty
 *                                     cluster keeps its previous centroid
 *   labels     [BH][N] int32     out  cluster of each row from the LAST assignment
 *   counts     [BH][C] int32     out  members per cluster under `labels`
 * Each of `iters` (>= 1) iterations assigns every row to the nearest centroid
 * (squared Euclidean distance; ties go to the lowest index) and then moves
 * every centroid to the mean of its members.  Assignments are exact: a row
 * whose fast distance gap is within its rounding bound is re-decided in fp64.
 * Requires 1 <= C <= min(N, 65536).
 */
EAR_API ear_status ear_kmeans(const void* X, ear_dtype dtype, int64_t bh, int64_t n, int32_t d,
                      int32_t c, int32_t iters, const float* init, float* centroids,
                      int32_t* labels, int32_t* counts, void* ws, size_t ws_bytes,
                      void* stream);

/*
 * Cluster-contiguous permutation (SVG-EAR §3.1: tokens are permuted so that
 * each cluster is contiguous and the attention map splits into blocks).
 *   labels   [BH][N] int32        cluster of each token, in [0, C)
 *   perm     [BH][N] int32   out  perm[r] = original index of permuted row r;
 *                                 a stable sort by label (ties by index)
 *   offsets  [BH][C+1] int32 out  first permuted row of each cluster; offsets[C] = N
 *   X        [BH][N][d] dtype     optional (NULL: only perm/offsets are produced)
 *   X_perm   [BH][N][d] dtype out X_perm[r] = X[perm[r]]            (needs X)
 *   seg_mean [BH][C][d] float out optional per-cluster mean of X's rows
 *                                 (SVG-EAR §4.3: v̄ = mean of V over a key
 *                                 cluster); zero rows for empty clusters (needs X)
 * A label outside [0, C) latches EAR_ERR_DEVICE and that token is dropped.
 */
EAR_API ear_status ear_permute(const int32_t* labels, int64_t bh, int64_t n, int32_t c,
                       int32_t* perm, int32_t* offsets, const void* X, void* X_perm,
                       ear_dtype dtype, int32_t d, float* seg_mean, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * Applies a permutation made by ear_permute to another token matrix (SVG-EAR
 * §4.3: V follows the key clustering, so V is laid out with K's permutation
 * and v̄_b is the mean of V over key cluster b).  No labels are recounted.
 *   perm     [BH][N] int32          from ear_permute (a bijection of [0, N))
 *   offsets  [BH][C+1] int32        from the same call
 *   X        [BH][N][d] dtype       rows in original order
 *   X_perm   [BH][N][d] dtype  out  X_perm[r] = X[perm[r]]; may be NULL when
 *                                   seg_mean is given (the means alone: the
 *                                   gathered layer keeps V in original order)
 *   seg_mean [BH][C][d] float  out  optional mean of X's rows of each cluster
 *                                   (rows offsets[c] .. offsets[c+1]-1 of
 *                                   X_perm); zero rows for empty clusters
 * Takes no workspace.  A perm entry outside [0, N) latches EAR_ERR_DEVICE and
 * that row is not written.  With seg_mean, rows are gathered cluster by
 * cluster, so the offsets must partition [0, N) (offsets[0] = 0,
 * offsets[C] = N, non-decreasing, as ear_permute writes them); a table that
 * does not latches EAR_ERR_DEVICE.
 */
EAR_API ear_status ear_permute_apply(const int32_t* perm, const int32_t* offsets, int64_t bh,
                                     int64_t n, int32_t c, const void* X, void* X_perm,
                                     ear_dtype dtype, int32_t d, float* seg_mean, void* stream);

/*
 * ear_permute_static - ear_permute for callers that cannot allocate device
 * memory (the paper has no counterpart: this is a deployment variant).
 *
 * Some callers have no way to allocate scratch: a plugin whose host
 * application owns every device buffer and passes in only inputs and
 * outputs, or an embedded runtime with a fixed memory plan.  This entry point
 * takes no workspace; its scratch is one fixed array of
 * EAR_PERMUTE_STATIC_MAX_BYTES compiled into the library, which every GPU
 * that loads the library keeps for the life of the process.
 *   - Arguments, outputs and results are exactly those of ear_permute.
 *   - The scratch needed is the one ear_workspace_bytes(EAR_OP_PERMUTE, ...)
 *     reports; a problem needing more than EAR_PERMUTE_STATIC_MAX_BYTES is
 *     rejected with EAR_ERR_WORKSPACE before anything runs.  (8 MiB holds,
 *     e.g., 40 slices of 75,600 tokens in 500 clusters.)
 *   - Every call looks up the array's device address on the current device
 *     (so a device reset between calls is safe); the first call on a device
 *     also loads the library's GPU code there, so make it before any stream
 *     capture begins.
 *   - No call allocates or frees memory (no cudaMalloc / cudaFree).
 *   - Every call reuses the same array and leaves its contents behind; each
 *     call clears what it needs zeroed.  Calls whose work overlaps on the
 *     GPU (two streams, or two host threads, on one device) race on the
 *     array: serialize them.
 */
#define EAR_PERMUTE_STATIC_MAX_BYTES (8u << 20)
EAR_API ear_status ear_permute_static(const int32_t* labels, int64_t bh, int64_t n, int32_t c,
                                      int32_t* perm, int32_t* offsets, const void* X,
                                      void* X_perm, ear_dtype dtype, int32_t d, float* seg_mean,
                                      void* stream);

/* ear_probe modes */
#define EAR_PROBE_LOGIT 0  /* logit-space gaps (§4.2 "Error estimation")             */
#define EAR_PROBE_WEIGHTS 1 /* gaps of the unnormalized attention weights (§4.2 relaxed) */
#define EAR_PROBE_VALUE 2  /* value-aware gaps of weight x value (§4.3)                 */

/*
 * Compensation-error probe (SVG-EAR §4.2 "Error estimation"; §1: query
 * centroids stand in for individual queries, O(C_q N_k d) work).
 *   q_centroids [BH][C_q][d] float     q̄_a
 *   q_counts    [BH][C_q] int32        |a|; rows with |a| = 0 get E = 0
 *   k_centroids [BH][C_k][d] float     k̄_b
 *   K_perm      [BH][N_k][d] dtype     keys in cluster-contiguous order
 *   k_offsets   [BH][C_k+1] int32      cluster b = rows [k_offsets[b], k_offsets[b+1])
 *   mode        EAR_PROBE_LOGIT / _WEIGHTS / _VALUE (the last two: bf16 keys only)
 *   V_perm      [BH][N_k][d] dtype     values in the keys' order (EAR_PROBE_VALUE; else NULL)
 *   v_centroids [BH][C_k][d] float     v̄_b (EAR_PROBE_VALUE; else NULL)
 *   E           [BH][C_q][C_k] float out, with z_j = scale q̄_a·k_j, z̄_b = scale q̄_a·k̄_b:
 *     LOGIT:   E[a][b] = sum_{j in b} (z_j - z̄_b)^2
 *     WEIGHTS: E[a][b] = sum_{j in b} (w_j - w̄_b)^2,   w = e^{z - m_a}
 *     VALUE:   E[a][b] = sum_{j in b} |w_j v_j - w̄_b v̄_b|^2
 *   where m_a is the largest z_j over all keys of the slice (the running
 *   maximum of §4.4 at the end of the stream).  scale is 1/sqrt(d) for the
 *   paper's logits.  Empty key or query clusters get 0.  fp32 keys support
 *   EAR_PROBE_LOGIT only (EAR_ERR_UNSUPPORTED otherwise).
 */
EAR_API ear_status ear_probe(const float* q_centroids, const int32_t* q_counts,
                     const float* k_centroids, const void* K_perm, ear_dtype dtype,
                     const int32_t* k_offsets, int64_t bh, int64_t n_k, int32_t d,
                     int32_t c_q, int32_t c_k, float scale, int32_t mode, const void* V_perm,
                     const float* v_centroids, float* E, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * ear_probe on keys (and values) left in their ORIGINAL token order (SVG-EAR
 * §3.1's cluster-contiguous layout folded into the loads, no permuted copy):
 *   K        [BH][N_k][d] dtype   keys in original order
 *   k_perm   [BH][N_k] int32      from ear_permute of K's labels: permuted
 *                                 key r is K[k_perm[r]]
 *   V        [BH][N_k][d] dtype   values in original order (EAR_PROBE_VALUE; else NULL)
 * Every other argument, the workspace (EAR_OP_PROBE) and E are as in
 * ear_probe, whose result this reproduces bit for bit on K_perm = K[k_perm].
 * A k_perm entry outside [0, N_k) latches EAR_ERR_DEVICE and row 0 is read
 * in its place.
 */
EAR_API ear_status ear_probe_gather(const float* q_centroids, const int32_t* q_counts,
                                    const float* k_centroids, const void* K,
                                    const int32_t* k_perm, ear_dtype dtype,
                                    const int32_t* k_offsets, int64_t bh, int64_t n_k, int32_t d,
                                    int32_t c_q, int32_t c_k, float scale, int32_t mode,
                                    const void* V, const float* v_centroids, float* E, void* ws,
                                    size_t ws_bytes, void* stream);

/*
 * Greedy error-to-cost routing under a density budget (SVG-EAR §4.2 "Error
 * estimation": blocks with the highest error-to-size ratio are computed
 * exactly until the budget is spent; §4.1: nnz(M) <= rho N_q N_k).
 *   E          [BH][C_q][C_k] float    probe output
 *   q_counts   [BH][C_q] int32, k_counts [BH][C_k] int32   cluster sizes
 *   density    rho in [0, 1]; budget B = floor(rho * (N_q*N_k)) pairs per slice
 *   ratio_mode 0: E[a][b] / |b|  (the pages' ratio: the block sum of the
 *                 per-entry estimates, |a| E[a][b], over |a||b|)
 *              1: E[a][b] / (|a| |b|)
 *   exact       [BH][C_q][C_k] uint8 out  1 = computed exactly
 *   blk_offsets [BH][C_q+1] int32    out  CSR row starts into blk_list (per slice)
 *   blk_list    [BH][C_q*C_k] int32  out  exact key clusters of each query
 *                                         cluster, ascending
 *   exact_pairs [BH] int64           out  (query, key) pairs computed exactly
 * Order: ratio descending (computed in fp64), ties to the lower a*C_k+b.
 * Blocks with |a||b| = 0 are never exact.  The walk adds |a||b| while the
 * total stays <= B and stops at the first block that does not fit.
 */
EAR_API ear_status ear_route(const float* E, const int32_t* q_counts, const int32_t* k_counts,
                     int64_t bh, int64_t n_q, int64_t n_k, int32_t c_q, int32_t c_k,
                     double density, int32_t ratio_mode, uint8_t* exact,
                     int32_t* blk_offsets, int32_t* blk_list, int64_t* exact_pairs,
                     void* ws, size_t ws_bytes, void* stream);

/*
 * Greedy error-to-cost routing inside each query cluster, under that
 * cluster's own budget (SVG-EAR §5 "Implementation": SVG2 assigns an adaptive
 * budget to each query cluster and SVG-EAR routes at that granularity).
 *   E, q_counts, k_counts   as in ear_route
 *   row_budget [BH][C_q] int64     pairs query cluster a may compute exactly
 *   exact, blk_offsets, blk_list, exact_pairs   out, as in ear_route
 * For query cluster a: its blocks with |a||b| > 0 in decreasing E[a][b] / |b|
 * (fp64; within one query cluster the same order as E / (|a||b|)), ties to
 * the lower b; |a||b| is added while the total stays <= row_budget[a], and
 * the walk stops at the first block that does not fit.  C_k <= 8192.
 */
EAR_API ear_status ear_route_rows(const float* E, const int32_t* q_counts,
                                  const int32_t* k_counts, int64_t bh, int32_t c_q, int32_t c_k,
                                  const int64_t* row_budget, uint8_t* exact,
                                  int32_t* blk_offsets, int32_t* blk_list, int64_t* exact_pairs,
                                  void* ws, size_t ws_bytes, void* stream);

/*
 * SVG2-style adaptive budget of each query cluster from its centroid
 * attention (the score-based top-p selection of SVG-EAR §3.1 / Fig. 2(c)).
 *   q_centroids [BH][C_q][d], q_counts [BH][C_q], k_centroids [BH][C_k][d],
 *   k_counts [BH][C_k]; scale = 1/sqrt(d) for the paper's logits; p in [0, 1]
 *   row_budget [BH][C_q] int64 out
 * The mass of key cluster b for query cluster a is |b| e^{scale q̄_a·k̄_b}
 * (computed in fp64) over non-empty b; sorted by decreasing mass (ties to the
 * lower b), the smallest prefix whose mass reaches p of the total is the
 * top-p set, and row_budget[a] = |a| x its key count (0 if |a| = 0).  With
 * E = that mass x |b|, ear_route_rows under these budgets selects exactly the
 * top-p sets.  C_k <= 8192.  Takes no workspace.
 */
EAR_API ear_status ear_topp_budget(const float* q_centroids, const int32_t* q_counts,
                                   const float* k_centroids, const int32_t* k_counts, int64_t bh,
                                   int32_t d, int32_t c_q, int32_t c_k, float scale, double p,
                                   int64_t* row_budget, void* stream);

/*
 * Each query cluster's share of a global density budget:
 * row_budget[a] = floor(density * (|a| * N_k)) (the product exact in int64,
 * then one double product).  Takes no workspace.
 */
EAR_API ear_status ear_uniform_budget(const int32_t* q_counts, int64_t bh, int32_t c_q,
                                      int64_t n_k, double density, int64_t* row_budget,
                                      void* stream);

/*
 * Block-sparse attention with linear compensation (SVG-EAR §4.1 routing mask,
 * §4.3 Linear Compensation).  For query i of cluster a one softmax runs over
 *   - exact logits scale q_i·k_j, value v_j, for every key j of every key
 *     cluster b listed in blk_list for a, and
 *   - (with EAR_COMPENSATE) for every other non-empty key cluster b, the
 *     logit scale q_i·k̄_b with weight |b| and value v̄_b.
 *   Q_perm, K_perm, V_perm [BH][N][d] dtype   cluster-contiguous rows
 *   q_offsets [BH][C_q+1], k_offsets [BH][C_k+1] int32
 *   q_perm    [BH][N_q] int32        original index of each permuted query
 *   k_centroids, v_centroids [BH][C_k][d] float   k̄_b, v̄_b
 *   exact     [BH][C_q][C_k] uint8, blk_offsets, blk_list   from ear_route
 *   O   [BH][N_q][d] dtype out  written at ORIGINAL query order
 *   lse [BH][N_q] float    out  optional natural-log normalizer per query
 * fp32 inputs are computed in fp32; bf16 inputs on the tensor cores with fp32
 * accumulation.  A query with no term at all gets O = 0 and lse = -inf.
 */
EAR_API ear_status ear_attention(const void* Q_perm, const void* K_perm, const void* V_perm,
                         ear_dtype dtype, const int32_t* q_offsets, const int32_t* k_offsets,
                         const int32_t* q_perm, const float* k_centroids,
                         const float* v_centroids, const uint8_t* exact,
                         const int32_t* blk_offsets, const int32_t* blk_list, int64_t bh,
                         int64_t n_q, int64_t n_k, int32_t d, int32_t c_q, int32_t c_k,
                         float scale, int32_t flags, void* O, float* lse, void* ws,
                         size_t ws_bytes, void* stream);

/*
 * ear_attention on Q, K and V left in their ORIGINAL token order (SVG-EAR
 * §3.1's cluster-contiguous layout folded into the loads: bf16 rows are
 * fetched four at a time with TMA tile::gather4, so no permuted copy of Q,
 * K or V is ever written).
 *   Q        [BH][N_q][d] dtype   queries in original order
 *   K, V     [BH][N_k][d] dtype   keys and values in original order
 *   q_perm   [BH][N_q] int32      permuted query r is Q[q_perm[r]] (and its
 *                                 output row is O[q_perm[r]], as in ear_attention)
 *   k_perm   [BH][N_k] int32      permuted key r is K[k_perm[r]], V[k_perm[r]]
 * Every other argument, the workspace (EAR_OP_ATTENTION), O and lse are as in
 * ear_attention, whose result this reproduces bit for bit on
 * Q_perm = Q[q_perm], K_perm = K[k_perm], V_perm = V[k_perm].  A k_perm entry
 * outside [0, N_k) latches EAR_ERR_DEVICE and row 0 is read in its place.
 */
EAR_API ear_status ear_attention_gather(const void* Q, const void* K, const void* V,
                                        ear_dtype dtype, const int32_t* q_offsets,
                                        const int32_t* k_offsets, const int32_t* q_perm,
                                        const int32_t* k_perm, const float* k_centroids,
                                        const float* v_centroids, const uint8_t* exact,
                                        const int32_t* blk_offsets, const int32_t* blk_list,
                                        int64_t bh, int64_t n_q, int64_t n_k, int32_t d,
                                        int32_t c_q, int32_t c_k, float scale, int32_t flags,
                                        void* O, float* lse, void* ws, size_t ws_bytes,
                                        void* stream);

/*
 * Clustering diagnostics (SVG-EAR §4.2: the error bound's residual
 * 8 δ_q^2 K_max^2 / (N_k d); §5.3 "Effect of clustering").
 *   X [BH][N][d] dtype, labels [BH][N] int32, centroids [BH][C][d] float
 *   mean_sq_dist [BH] double out   δ^2 = (1/N) sum_i ||x_i - c_{labels[i]}||^2
 *   max_norm     [BH] double out   max_i ||x_i|| (K_max when X = K)
 * Per row in fp32, summed over rows in fp64.  A label outside [0, C) latches
 * EAR_ERR_DEVICE and that row is skipped.  Takes no workspace.
 */
EAR_API ear_status ear_cluster_stats(const void* X, ear_dtype dtype, const int32_t* labels,
                                     const float* centroids, int64_t bh, int64_t n, int32_t d,
                                     int32_t c, double* mean_sq_dist, double* max_norm,
                                     void* stream);

/*
 * Average relative change of the softmax normalizer (SVG-EAR §5.1): per
 * slice, the mean over the N queries of |Z_sparse / Z_dense - 1| with
 * Z = e^{lse} (lse from ear_attention with the routed mask, and with every
 * block exact); a query whose two lse are equal counts 0.
 *   lse_sparse, lse_dense [BH][N] float; change [BH] double out
 */
EAR_API ear_status ear_normalizer_change(const float* lse_sparse, const float* lse_dense,
                                         int64_t bh, int64_t n, double* change, void* stream);

/*
 * Synchronizes `stream`, then returns in *out the first device-side error
 * code latched on the current device since the last call (EAR_OK if none)
 * and clears it.
 */
EAR_API ear_status ear_get_device_status(int32_t* out, void* stream);

/* Number of kernels this library has launched in this process (all devices). */
EAR_API uint64_t ear_launch_count(void);

/*
 * Failure-path self-test (the pages have no counterpart; it checks this
 * library's bounded waits).  Enqueues one warp on `stream` that waits on a
 * barrier nothing completes.  The wait gives up after its bound (about 1 s),
 * latches EAR_ERR_TIMEOUT in the device status word and the kernel returns;
 * the next ear_get_device_status() on this device reports EAR_ERR_TIMEOUT and
 * clears it, and the context stays usable.  Returns EAR_ERR_CUDA if the launch
 * fails; takes no buffers and allocates nothing.
 */
EAR_API ear_status ear_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EAR_H_ */
