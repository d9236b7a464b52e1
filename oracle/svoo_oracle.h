/*
 * svoo_oracle.h -- CPU oracle for the online QK co-clustered block-sparse
 * attention path (SVOO bidirectional co-clustering, iCATS interaction-aware
 * clustering and tail merging, cluster-pair block mask, masked softmax
 * attention).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the CUDA library links, includes or calls
 * this code; only the tests, the package's smoke check and the CPU-baseline leg
 * of the benchmark do. It is plain single-threaded C, fp64 unless a function
 * says otherwise, written for a reader to check by eye against the pages:
 *
 *   [SVOO]  "Attention Sparsity is Input-Stable: Training-Free Sparse Attention
 *           for Video Generation via Offline Sparsity Profiling and Online QK
 *           Co-Clustering" (ICML 2026 poster page), abstract.
 *   [iCATS] "iCATS: Fast Video Generation via Interaction-Aware Sparse Attention
 *           and Timestep-Adaptive Sparsity" (paperlayer.ai summary), sections
 *           3.1, 3.3, 4.1, 4.3, appendix E.1 / E.2.
 *   [PSA]   "PSA: Parameterized Stripe Attention" full text, section 2 (SVG2's
 *           k-means clustering, permutation and top-k cluster selection),
 *           section 3.2 with Algorithm 1 (the stripe mask M(Tw,To,Ts,Sw,So,Ss)
 *           at PSABlock granularity) and Table 2 (FLOP accounting).
 *
 * Readings of points the pages leave open are stated beside each function.
 * Arrays are row-major; bf16 values are passed as their uint16 bit patterns.
 * Per-head functions: the Python wrapper loops over (batch, head).
 */
#ifndef SVOO_ORACLE_H
#define SVOO_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int oracle_version(void);

/* exp of a float argument by Cody-Waite range reduction and a degree-7 Taylor
 * polynomial, every step an explicit fp32 operation (defined in the .c file). */
float oracle_exp(float x);

/* Interaction metric M (d x d, fp64) from the other side's clusters. */
void oracle_metric(const float *cent, const int32_t *sizes, int C, int d, int identity,
                   double *M);

/* Deterministic start: centroid j = token floor(j*n/C). */
void oracle_init_centroids(const uint16_t *x, int n, int d, int C, float *cent);

/* Assignment under metric M; best/second may be NULL. */
void oracle_assign(const uint16_t *x, int n, int d, const float *cent, int C, const double *M,
                   int32_t *assign, double *best, double *second);

/* Centroid update (exact fp64 sums, fp32 centroids). */
void oracle_update(const uint16_t *x, int n, int d, const int32_t *assign, int C,
                   const float *cent_old, float *cent_new, int32_t *sizes);

/* Full co-clustering of one head: `iters` rounds of (Q step, K step).
 * flags: bit 0 warm start, bit 1 identity metric in every step. */
void oracle_cluster(const uint16_t *q, const uint16_t *k, int n, int d, int Cq, int Ck, int iters,
                    int flags, int32_t *q_assign, int32_t *k_assign, float *q_cent, float *k_cent,
                    int32_t *q_sizes, int32_t *k_sizes);

/* Estimated attention mass of every (query cluster, key cluster) pair. fp32. */
void oracle_pair_mass(const float *q_cent, const float *k_cent, const int32_t *q_sizes,
                      const int32_t *k_sizes, int Cq, int Ck, int d, float scale, float *w,
                      int32_t *top1);

/* Pair selection -> packed key-cluster masks. Returns the kept pair count. */
int oracle_select(const float *w, const int32_t *top1, int Cq, int Ck, int mode, float keep,
                  float top_p, int has_text, uint64_t *kmask, int W);

/* Tail merging of query clusters (in place). Returns the number of non-empty
 * query clusters left. stats[0..5] = identical merges, moves round 1, moves
 * round 2, query tiles before, query tiles after, tokens moved. */
int oracle_tail_merge(uint64_t *kmask, int32_t *sizes, int32_t *label, int n, int Cq, int W,
                      int block_q, int rounds, int32_t *stats);

/* Stable counting sort of n labels in [0, G): perm[pos] = token, off[G+1]. */
void oracle_permute(const int32_t *label, int n, int G, int32_t *perm, int32_t *off);

/* Query tiles (group, start, rows) of at most block_q rows; returns count. */
int oracle_tiles(const int32_t *off, int G, int block_q, int32_t *tiles);

/* Masked softmax attention for selected query rows (fp64). */
void oracle_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int n, int d,
                      float scale, const int32_t *q_label, const int32_t *k_label,
                      const uint64_t *kmask, int W, const int32_t *rows, int nrows, double *out,
                      double *psum, int64_t *nkeys);

/* Textbook dense softmax attention for selected query rows (fp64). */
void oracle_dense_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int n, int d,
                            float scale, const int32_t *rows, int nrows, double *out);

/* [PSA] Alg. 1: does position i attend position j (frames of HW positions)
 * under M(Tw, To, Ts, Sw, So, Ss) = prm[0..5]; a stride INT32_MAX is infinity. */
int oracle_psa_attends(long long i, long long j, long long HW, const int32_t *prm);

/* Static stripe-mask plan of one head at PSABlock granularity: labels (the
 * token's block), block mask and block sizes; returns the block count. */
int oracle_psa_plan(int T, int H, int W, int bt, int bh, int bw, int n_text, const int32_t *prm,
                    int32_t *label, uint64_t *kmask, int32_t *sizes);

/* [iCATS] 4.2, appendix A: SNR-guided top-p of each of `steps` denoising
 * calls (a reading: the pages give the shape of the schedule, not a formula;
 * see the .c file). Writes p[0..steps-1]; returns 0, or -1 for bad arguments. */
int oracle_snr_top_p(int steps, int warmup, double p_min, double tau, double shift, float *p);

#ifdef __cplusplus
}
#endif
#endif
