/*
 * svoo.h -- C ABI of the B200 (sm_100a) library for online QK co-clustered
 * block-sparse attention in video diffusion transformers.
 *
 * The path (one attention call of one layer), after the pages that describe it:
 *
 *   1. svoo_cluster      per head, bidirectional k-means of the query and key
 *                        tokens under the query-key interaction metric
 *                        ("Attention Sparsity is Input-Stable ... Online QK
 *                        Co-Clustering" (SVOO), abstract; "iCATS" sections 3.1
 *                        and 4.1: a quadratic form in feature space, the first
 *                        query step in feature space, later query steps under
 *                        the key-cluster metric, key steps under the
 *                        just-updated query clusters).
 *   2. svoo_build_mask   per head, the estimated attention mass of every
 *                        (query cluster, key cluster) pair from the centroids,
 *                        a keep-ratio or top-p selection of pairs ("PSA"
 *                        section 2 on SVG2's centroid scores and top-k cluster
 *                        selection; iCATS section 4.2 top-p; SVOO's offline
 *                        per-layer level enters as the keep ratio), then iCATS
 *                        tail merging of the query clusters (section 4.3,
 *                        appendix E.1).
 *   3. svoo_permute      stable permutation of the tokens into cluster order
 *                        (PSA section 2, SVG2's semantic-aware permutation),
 *                        query tiles, and the gathered Q, K, V in that order.
 *   4. svoo_sparse_attn  flash-style softmax(scale Q K^T) V restricted to the
 *                        kept cluster pairs, online softmax over the kept key
 *                        tiles only, O written back in token order.
 *
 * A second source of the plan replaces steps 1-2 for heads with a static
 * pattern: svoo_psa_mask writes the stripe mask of "PSA: Parameterized Stripe
 * Attention" (section 3.2, Algorithm 1) with every PSABlock as one group;
 * steps 3-4 then run unchanged.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or synchronises. Work is enqueued on `stream` (a
 *    cudaStream_t passed as void*; NULL = legacy default stream) in call order.
 *  - Q, K, V, O are bf16 [B, H, N, d] row-major; the N tokens of a head are
 *    N - n_text video tokens followed by n_text always-kept text tokens.
 *  - Arguments are validated on the host before any launch; a bad argument
 *    returns SVOO_ERR_INVALID_ARG and enqueues nothing. Launch failures return
 *    SVOO_ERR_CUDA.
 *  - Device-side problems (a pipeline wait that exceeded its time budget,
 *    out-of-range plan metadata) set bits in the caller's int32 error word
 *    `dev_err` (device memory, may be NULL) with atomicOr; the caller reads it
 *    when it chooses: 1 = attention wait timeout, 2 = clustering wait timeout,
 *    4 = plan metadata out of range, 8 = cluster label out of range. While a
 *    timeout bit (1 or 2) is set, the pipelined kernels skip their work, so
 *    clear the word after handling a timeout.
 *  - Limits: 1 <= B*H <= 65535, B*H*N < 2^31 - 256, 1 <= N - n_text, N <= 2^20,
 *    d in {64, 128},
 *    1 <= n_qc, n_kc <= 256, block_q in {64, 128}, 0 <= n_text, iters >= 1.
 *    Inputs must be finite. Centroid member sums are exact (fp64, with
 *    components |x| < 2^-24 counted as zero, so every partial sum is a
 *    multiple of 2^-31 below 2^22), and a centroid is its exact mean rounded
 *    once to fp32, whatever the order in which the GPU added the members.
 */
#ifndef SVOO_H
#define SVOO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SVOO_OK = 0,
    SVOO_ERR_INVALID_ARG = 1,
    SVOO_ERR_WORKSPACE = 2,
    SVOO_ERR_UNSUPPORTED = 3,
    SVOO_ERR_CUDA = 4,
    SVOO_ERR_TIMEOUT = 5,
    SVOO_ERR_INTERNAL = 6
} svoo_status;

/* Shape of one attention call. */
typedef struct {
    int B;      /* batch */
    int H;      /* heads */
    int N;      /* tokens per head, video then text */
    int d;      /* head dimension: 64 or 128 */
    int n_text; /* trailing always-kept text tokens (HunyuanVideo), 0 if none */
} svoo_shape;

/* Device buffers of one call's sparse plan; every array is caller-allocated
 * with the element counts that svoo_plan_counts returns. BH = B*H,
 * Gq = n_qc + (n_text > 0), Gk = n_kc + (n_text > 0), W = ceil(Gk / 64),
 * Tcap = ceil(N / block_q) + Gq, Ucap = ceil(N / 256) + Gq. All int32 unless
 * stated. */
typedef struct {
    uint64_t *kmask;     /* [BH][Gq][W] bit b of row a: query group a attends key group b.
                            Written by svoo_build_mask (after tail merging). */
    int32_t *q_label;    /* [BH][N]   merged query group of every token (text: n_qc) */
    int32_t *q_sizes;    /* [BH][Gq]  tokens per merged query group */
    int32_t *stats;      /* [BH][8]   kept pairs, non-empty query clusters, identical-mask
                            merges, tail moves round 1, tail moves round 2, query tiles
                            before merging, query tiles after, moved tokens */
    int32_t *q_perm;     /* [BH][N]   position in cluster order -> token (svoo_permute) */
    int32_t *q_off;      /* [BH][Gq+1] group start positions in q_perm */
    int32_t *k_perm;     /* [BH][N] */
    int32_t *k_off;      /* [BH][Gk+1] */
    int32_t *tiles;      /* [BH][Tcap][4] query tile: group, start position, rows, kv length */
    int32_t *tile_count; /* [BH] tiles in use per head */
    int32_t *units;      /* [BH][Ucap][4] attention work units: up to 256 consecutive rows of
                            one query group (two 128-row MMA tiles sharing every key/value
                            tile): group, start position, rows, kv length (svoo_permute) */
    int32_t *unit_count; /* [BH] units in use per head */
} svoo_plan;

/* Element counts of the svoo_plan arrays (in field order) for a shape. */
svoo_status svoo_plan_counts(const svoo_shape *shape, int n_qc, int n_kc, int block_q,
                             int64_t counts[12]);

/* ------------------------------------------------------------------ clustering
 * Bytes of device workspace svoo_cluster / svoo_cluster_step need. */
size_t svoo_cluster_workspace_size(const svoo_shape *shape, int n_qc, int n_kc);

#define SVOO_CLUSTER_WARM 1
#define SVOO_CLUSTER_IDENTITY 2

/* Co-clusters the video tokens of every head.
 *  q, k      : bf16 [B,H,N,d] (only the first N - n_text tokens are clustered).
 *  iters     : rounds of (query step, key step), each an assignment + update.
 *  flags     : bitwise OR of
 *              SVOO_CLUSTER_WARM: start from q_cent, k_cent, k_sizes as given
 *                (e.g. the previous timestep's), first query step under the
 *                key-cluster metric; without it, start from the tokens at
 *                floor(j*Nv/C) with a feature-space first query step;
 *              SVOO_CLUSTER_IDENTITY: every step in feature space (M = I):
 *                plain k-means of queries and keys separately, the
 *                independent Euclidean clustering (SVG2's) that iCATS sec. 3.1
 *                and App. D (Table 3) compare the co-clustering against.
 *              Any other bit is SVOO_ERR_INVALID_ARG.
 *  q_assign, k_assign : int32 [BH][N - n_text] cluster of every video token.
 *  q_cent, k_cent     : fp32 [BH][n_qc|n_kc][d] centroids (in/out).
 *  q_sizes, k_sizes   : int32 [BH][n_qc|n_kc] members per cluster (k_sizes in/out).
 * Assignment: argmin_j (x - mu_j)^T M (x - mu_j), ties to the smaller j, where
 * M is the normalised second moment of the other side's clusters (identity in
 * the cold first query step, and in every step under SVOO_CLUSTER_IDENTITY);
 * M, nu_j = M mu_j and kappa_j = mu_j . nu_j in
 * fp64. Scores come from tcgen05 MMAs against nu split into two bf16 rows
 * (with kappa folded in); when more than one cluster lies within the MMA's
 * error bound of the best, those candidates (or, when there are many, all
 * clusters) are compared exactly in fp64, so the result is that of an fp64
 * evaluation. Update: member means from exact sums (see the limits above), so
 * equal labels give bit-identical centroids; an empty cluster keeps its
 * centroid. Each side's first step of a call sums all members; later steps
 * move only the tokens whose label changed (exact, so the same bits). The
 * workspace holds those kept sums, so calls sharing one workspace must not
 * overlap on the GPU. */
svoo_status svoo_cluster(const svoo_shape *shape, const void *q, const void *k, int n_qc,
                         int n_kc, int iters, int flags, int32_t *q_assign, int32_t *k_assign,
                         float *q_cent, float *k_cent, int32_t *q_sizes, int32_t *k_sizes,
                         void *workspace, size_t workspace_bytes, int32_t *dev_err,
                         void *stream);

/* One half-step of the above for one side: assigns the video tokens of x to
 * the centroids `cent` (in/out) under the metric of (metric_cent, metric_sizes)
 * (metric_C clusters; identity if metric_cent is NULL, and metric_C is then
 * ignored), then updates `cent` and `sizes`. Used for warm starts and for
 * step-level parity checks. */
svoo_status svoo_cluster_step(const svoo_shape *shape, const void *x, int C, float *cent,
                              int32_t *sizes, int32_t *assign, const float *metric_cent,
                              const int32_t *metric_sizes, int metric_C, void *workspace,
                              size_t workspace_bytes, int32_t *dev_err, void *stream);

/* Allocation-free variant of svoo_cluster_step. The paper pages have no
 * counterpart: it exists for callers that may not allocate device memory
 * themselves (code inside a host framework that owns all device memory through
 * its own pool, or a latency-critical loop that forbids allocation after
 * start-up). Arguments as svoo_cluster_step minus the workspace; the scratch
 * is a fixed array of SVOO_STATIC_SCRATCH_BYTES compiled into the library,
 * held on every GPU that loads it until the process exits. Shapes whose
 * scratch would exceed it return SVOO_ERR_WORKSPACE and enqueue nothing (16 MiB
 * covers, e.g., B*H = 12, d = 128, 128 clusters). The first call on a device
 * looks up the array's device address (make it before any stream capture).
 * All calls share the array and each clears the accumulators it uses; calls
 * that overlap on the GPU (e.g. on two streams) race. */
#define SVOO_STATIC_SCRATCH_BYTES (16u << 20)
svoo_status svoo_cluster_step_static(const svoo_shape *shape, const void *x, int C, float *cent,
                                     int32_t *sizes, int32_t *assign, const float *metric_cent,
                                     const int32_t *metric_sizes, int metric_C, int32_t *dev_err,
                                     void *stream);

/* ------------------------------------------------------------------ mask
 * Bytes of device workspace svoo_build_mask needs. */
size_t svoo_mask_workspace_size(const svoo_shape *shape, int n_qc, int n_kc);

/* Builds the key-cluster mask of every query cluster and tail-merges them.
 *  keep[BH] (fp32, device): select_mode 0 -> keep ratio r in (0, 1]: the head
 *    keeps K = ceilf(r * (n_qc*n_kc)) pairs (fp32 product), at least each query
 *    cluster's best pair; select_mode 1 -> top-p p in [0, 1]: the shortest
 *    prefix of the same order whose mass (fixed point floor(w * 2^32)) reaches
 *    ceil(p * total), again at least the per-cluster best pairs.
 *  Pair order: per-cluster best first, then w descending, then query cluster
 *    ascending, then key cluster ascending; w is the estimated attention mass
 *    n_a * n_b e^(s_ab - m_a) / Z_a with s_ab = scale * mu_a . c_b, computed
 *    in fp32 with a fixed operation order (bit-identical to the oracle).
 *  Tail merging: identical masks merge into the lowest id; then merge_rounds
 *    rounds in which mutually nearest (Hamming distance of masks) clusters
 *    whose tails (size mod block_q) fit one block move the smaller tail into
 *    the other, whose mask becomes the union. Text tokens (if any) form query
 *    group n_qc attending everything, and key group n_kc, which every query
 *    group keeps; they are outside the budget and the merging.
 *  Writes plan->kmask, q_label, q_sizes, stats. */
svoo_status svoo_build_mask(const svoo_shape *shape, const float *q_cent, const float *k_cent,
                            const int32_t *q_sizes, const int32_t *k_sizes,
                            const int32_t *q_assign, const float *keep, int n_qc, int n_kc,
                            int select_mode, int block_q, int merge_rounds, float scale,
                            const svoo_plan *plan, void *workspace, size_t workspace_bytes,
                            int32_t *dev_err, void *stream);

/* ------------------------------------------------------------------ static stripe mask
 * Number of PSABlocks, ceil(T/bt) ceil(H/bh) ceil(W/bw), of a token grid; 0
 * for a non-positive argument. */
int svoo_psa_block_count(int grid_t, int grid_h, int grid_w, int block_t, int block_h,
                         int block_w);

#define SVOO_PSA_INF 2147483647 /* stride "infinity": one diagonal band on that axis */

/* The plan of the stripe mask M(Tw, To, Ts, Sw, So, Ss) of PSA ("PSA:
 * Parameterized Stripe Attention", section 3.2 and Algorithm 1), in place of
 * svoo_cluster + svoo_build_mask.
 *  grid_t, grid_h, grid_w : the video tokens form a (T, H, W) grid in raster
 *        order (T*H*W must equal N - n_text).
 *  block_t, block_h, block_w : the PSABlock. The block grid is (T', H', W') =
 *        (ceil(T/bt), ceil(H/bh), ceil(W/bw)), nb = T'H'W' <= 256 blocks,
 *        numbered in raster order; blocks on the far edges hold only the
 *        tokens that exist (no padding).
 *  params : int32 [B*H][6], DEVICE: (Tw, To, Ts, Sw, So, Ss) of each head.
 *        Tw, Sw >= 0; Ts, Ss >= 1, SVOO_PSA_INF for infinity. A head with a
 *        parameter out of range gets no video block pair (its text group, if
 *        any, is still kept) and sets bit 4 in dev_err.
 *  Masking is at PSABlock granularity: query block a keeps key block b when
 *  Algorithm 1 holds for the block indices (frame = index / (H'W'), in-frame
 *  position = index % (H'W')), i.e. the frame distance D satisfies
 *  (|D - To| mod Ts) <= Tw - 1 and the in-frame distance E satisfies
 *  (|E - So| mod Ss) <= Sw - 1. Text tokens form group nb, which attends
 *  every group and which every group attends.
 *  Writes plan->kmask, q_label (a token's block), q_sizes and stats (kept
 *  video block pairs, nb, 0, 0, 0, query tiles, query tiles, 0), sized by
 *  svoo_plan_counts(shape, nb, nb, block_q), and k_assign (int32
 *  [B*H][N - n_text], the key block of every video token) for svoo_permute.
 *  Then call svoo_permute and svoo_sparse_attn with n_qc = n_kc = nb: the
 *  stable sort lays every block's tokens out contiguously in raster order,
 *  which is PSA's block-centric (T', H', W', bt, bh, bw) layout. */
svoo_status svoo_psa_mask(const svoo_shape *shape, int grid_t, int grid_h, int grid_w,
                          int block_t, int block_h, int block_w, const int32_t *params,
                          int block_q, svoo_plan *plan, int32_t *k_assign, int32_t *dev_err,
                          void *stream);

/* ------------------------------------------------------------------ permutation
 * Stable counting sorts of the merged query labels (plan->q_label) and of the
 * key labels (k_assign, text tokens as group n_kc): q_perm/q_off, k_perm/k_off;
 * the query tile table and per-head tile counts; and the gathered copies
 *   qp[p] = q[q_perm[p]], kp[p] = k[k_perm[p]], vp[p] = v[k_perm[p]]
 * (bf16 [B,H,N,d], caller-allocated) that svoo_sparse_attn reads. */
svoo_status svoo_permute(const svoo_shape *shape, const void *q, const void *k, const void *v,
                         const int32_t *k_assign, int n_qc, int n_kc, int block_q,
                         const svoo_plan *plan, void *qp, void *kp, void *vp, int32_t *dev_err,
                         void *stream);

/* ------------------------------------------------------------------ attention
 * o[token] = softmax(scale * q_token . K_kept^T) V_kept over the keys of the
 * key groups that the token's query group keeps, for every query tile of the
 * plan; qp/kp/vp are the cluster-ordered copies from svoo_permute; o is bf16
 * [B,H,N,d] in token order. A query whose kept key groups are all empty gets
 * o = 0. tcgen05 MMAs (bf16 in, fp32 accumulate) into tensor memory, online
 * softmax in fp32, P rounded to bf16 for the second product. */
svoo_status svoo_sparse_attn(const svoo_shape *shape, const void *qp, const void *kp,
                             const void *vp, const svoo_plan *plan, int n_qc, int n_kc,
                             int block_q, float scale, void *o, int32_t *dev_err, void *stream);

/* ------------------------------------------------------------------ top-p schedule
 * SNR-guided top-p of every call of a denoising run ("iCATS" section 4.2 and
 * appendix A: top-p follows a smooth function of the log signal-to-noise
 * ratio, fixed offline from the noise schedule, with dense attention before
 * the first sparse call; the budget stays steady early and late and falls in
 * the middle). The pages give no formula; this library reads it as
 *   s = 1 - t/steps, sigma = shift*s / (1 + (shift - 1)*s)   (flow matching),
 *   p(t) = p_min + (tau - p_min) / (1 + SNR(t)),  SNR = ((1 - sigma)/sigma)^2,
 * i.e. a logistic in log SNR: tau at pure noise, p_min in the noise-free
 * limit, (tau + p_min)/2 where SNR = 1; p(t) = 1 for t < warmup.
 * Host code only (no GPU work): writes p[0..steps-1] (HOST memory, fp32),
 * ready to be passed as the per-head keep values of svoo_build_mask with
 * select_mode 1. Requires steps >= 1, warmup >= 0, 0 <= p_min <= tau <= 1,
 * shift > 0; otherwise SVOO_ERR_INVALID_ARG and p is left untouched. */
svoo_status svoo_snr_top_p(int steps, int warmup, double p_min, double tau, double shift,
                           float *p);

const char *svoo_status_string(svoo_status s);

/* Library version, (major << 16) | minor. */
int svoo_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SVOO_H */
