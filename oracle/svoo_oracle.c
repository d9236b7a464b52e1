/*
 * svoo_oracle.c -- plain CPU oracle of the online QK co-clustered block-sparse
 * attention path. TEST INFRASTRUCTURE ONLY: the CUDA library never links or
 * calls it; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. Single-threaded, fp64 unless stated, no blocking or fusion.
 *
 * Build: cc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (see build.py).
 * -ffp-contract=off matters: every fp32 operation below is one IEEE operation,
 * fused only where fmaf() is written.
 *
 * Page references are given as [page] section. See svoo_oracle.h for the list.
 */
#include "svoo_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

int oracle_version(void) { return 1; }

static double bf16_val(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* exp used by the pair scoring.                                              */
/*                                                                            */
/* The selection of cluster pairs turns floating point into integer decisions */
/* (which pairs are kept), so the oracle and the GPU must compute the same    */
/* fp32 value. Neither may call its platform's expf (they differ), so both    */
/* implement this one definition, from mathematics only:                      */
/*   n  = rint(x * log2(e))                 fp32 multiply, round-half-even     */
/*   r  = fma(-n, LN2_HI, x); r = fma(-n, LN2_LO, r)   (Cody & Waite, 1980)    */
/*   p  = sum_{k=0..7} r^k / k!  by Horner with fmaf  (Taylor series of e^r)   */
/*   e^x = p * 2^n, 2^n built from its exponent bits                           */
/* LN2_HI = 22713 / 2^15 (ln 2 cut to 15 significant bits, so n*LN2_HI is     */
/* exact for |n| < 2^9) and LN2_LO = fp32(ln 2 - LN2_HI). Domain: x <= 0;     */
/* x < -87 returns 0.                                                          */
/* ------------------------------------------------------------------------ */
float oracle_exp(float x) {
    const float log2e = 1.4426950408889634f;
    const float ln2_hi = 22713.0f / 32768.0f;
    const float ln2_lo = (float)(0.69314718055994530942 - 22713.0 / 32768.0);
    const float c2 = (float)(1.0 / 2.0), c3 = (float)(1.0 / 6.0), c4 = (float)(1.0 / 24.0);
    const float c5 = (float)(1.0 / 120.0), c6 = (float)(1.0 / 720.0), c7 = (float)(1.0 / 5040.0);
    if (!(x >= -87.0f)) return 0.0f;
    float t = x * log2e;
    float n = rintf(t);
    float r = fmaf(-n, ln2_hi, x);
    r = fmaf(-n, ln2_lo, r);
    float p = c7;
    p = fmaf(p, r, c6);
    p = fmaf(p, r, c5);
    p = fmaf(p, r, c4);
    p = fmaf(p, r, c3);
    p = fmaf(p, r, c2);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ni = (int)n;
    uint32_t bits = (uint32_t)(ni + 127) << 23;
    float s;
    memcpy(&s, &bits, sizeof s);
    return p * s;
}

/* ------------------------------------------------------------------------ */
/* Interaction metric. [iCATS] 3.1 / 4.1: clustering should minimise the      */
/* error of the query-key dot products, and this objective is rewritten as a  */
/* quadratic form in the original feature space. Replacing a query q by its   */
/* centroid mu changes q.k by (q - mu).k for every key k; the mean squared    */
/* change over the keys is (q - mu)^T M (q - mu) with M = E_k[k k^T]. With    */
/* keys summarised by their clusters (the key clusters of the step before):   */
/*     M = sum_b n_b c_b c_b^T / sum_b n_b.                                   */
/* The key step uses the same form with the query clusters. identity != 0     */
/* gives M = I (plain feature-space k-means, [iCATS] 4.1's first step).       */
/* ------------------------------------------------------------------------ */
void oracle_metric(const float *cent, const int32_t *sizes, int C, int d, int identity,
                   double *M) {
    double total = 0.0;
    for (int b = 0; b < C; ++b) total += (double)sizes[b];
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) M[(size_t)i * d + j] = 0.0;
    if (identity || total <= 0.0) {
        for (int i = 0; i < d; ++i) M[(size_t)i * d + i] = 1.0;
        return;
    }
    for (int b = 0; b < C; ++b) {
        if (sizes[b] == 0) continue;
        const float *c = cent + (size_t)b * d;
        double wb = (double)sizes[b] / total;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j)
                M[(size_t)i * d + j] += wb * (double)c[i] * (double)c[j];
    }
}

/* Reading: the pages do not say how centroids start. Start deterministically */
/* from the tokens at indices floor(j * n / C), j = 0..C-1 (no RNG).          */
void oracle_init_centroids(const uint16_t *x, int n, int d, int C, float *cent) {
    for (int j = 0; j < C; ++j) {
        long long idx = (long long)j * n / C;
        for (int i = 0; i < d; ++i)
            cent[(size_t)j * d + i] = (float)bf16_val(x[(size_t)idx * d + i]);
    }
}

/* Assignment step of k-means under metric M: a(x) = argmin_j D_j(x),        */
/* D_j(x) = (x - mu_j)^T M (x - mu_j), exact ties to the smaller j.           */
/* Expanded as D_j = x^T M x - 2 x.nu_j + kappa_j with nu_j = M mu_j and       */
/* kappa_j = mu_j^T nu_j (the same quadratic form; the argmin is taken on     */
/* kappa_j - 2 x.nu_j since x^T M x does not depend on j).                    */
void oracle_assign(const uint16_t *x, int n, int d, const float *cent, int C, const double *M,
                   int32_t *assign, double *best, double *second) {
    double *nu = (double *)malloc(sizeof(double) * (size_t)C * d);
    double *kappa = (double *)malloc(sizeof(double) * (size_t)C);
    double *xv = (double *)malloc(sizeof(double) * (size_t)d);
    double *mx = (double *)malloc(sizeof(double) * (size_t)d);
    for (int j = 0; j < C; ++j) {
        const float *mu = cent + (size_t)j * d;
        double kap = 0.0;
        for (int i = 0; i < d; ++i) {
            double s = 0.0;
            for (int l = 0; l < d; ++l) s += M[(size_t)i * d + l] * (double)mu[l];
            nu[(size_t)j * d + i] = s;
        }
        for (int i = 0; i < d; ++i) kap += (double)mu[i] * nu[(size_t)j * d + i];
        kappa[j] = kap;
    }
    for (int t = 0; t < n; ++t) {
        for (int i = 0; i < d; ++i) xv[i] = bf16_val(x[(size_t)t * d + i]);
        double b1 = INFINITY, b2 = INFINITY;
        int arg = 0;
        for (int j = 0; j < C; ++j) {
            double dot = 0.0;
            const double *nj = nu + (size_t)j * d;
            for (int i = 0; i < d; ++i) dot += xv[i] * nj[i];
            double s = kappa[j] - 2.0 * dot;
            if (s < b1) {
                b2 = b1;
                b1 = s;
                arg = j;
            } else if (s < b2) {
                b2 = s;
            }
        }
        assign[t] = arg;
        if (best || second) {
            double xmx = 0.0;
            for (int i = 0; i < d; ++i) {
                double s = 0.0;
                for (int l = 0; l < d; ++l) s += M[(size_t)i * d + l] * xv[l];
                mx[i] = s;
            }
            for (int i = 0; i < d; ++i) xmx += xv[i] * mx[i];
            if (best) best[t] = xmx + b1;
            if (second) second[t] = xmx + b2;
        }
    }
    free(nu);
    free(kappa);
    free(xv);
    free(mx);
}

/* Update step: mu_j = mean of its members, n_j = member count. Reading: an   */
/* empty cluster keeps its previous centroid. Precision reading: sums are     */
/* fp64; components with |x| < 2^-24 count as 0, which makes every partial   */
/* sum an exact multiple of 2^-31 (exact in fp64 while |sum| < 2^22), so the  */
/* sum does not depend on the order of the members. The centroid is the fp64  */
/* quotient rounded once to fp32.                                             */
void oracle_update(const uint16_t *x, int n, int d, const int32_t *assign, int C,
                   const float *cent_old, float *cent_new, int32_t *sizes) {
    double *sum = (double *)calloc((size_t)C * d, sizeof(double));
    const double tiny = 1.0 / 16777216.0; /* 2^-24 */
    for (int j = 0; j < C; ++j) sizes[j] = 0;
    for (int t = 0; t < n; ++t) {
        int j = assign[t];
        sizes[j] += 1;
        for (int i = 0; i < d; ++i) {
            double v = bf16_val(x[(size_t)t * d + i]);
            if (fabs(v) < tiny) v = 0.0;
            sum[(size_t)j * d + i] += v;
        }
    }
    for (int j = 0; j < C; ++j) {
        for (int i = 0; i < d; ++i) {
            size_t o = (size_t)j * d + i;
            cent_new[o] = sizes[j] > 0 ? (float)(sum[o] / (double)sizes[j]) : cent_old[o];
        }
    }
    free(sum);
}

/* Bidirectional co-clustering of one head ([SVOO] abstract; [iCATS] 4.1):    */
/* round 0's query step runs in feature space (M = I); every later query     */
/* step uses the metric of the current key clusters, and each key step uses  */
/* the metric of the query clusters it has just updated. `iters` rounds of   */
/* (query step, key step), each step one assignment and one update.          */
/* flags bit 0 (warm): q_cent, k_cent and k_sizes hold a start state (e.g.  */
/* the previous timestep's clusters) and round 0's query step uses M_K too.  */
/* flags bit 1 (identity): every step uses M = I, i.e. queries and keys are  */
/* clustered independently in feature space, the Euclidean clustering that   */
/* [iCATS] 3.1 and App. D (Table 3) compare against.                         */
void oracle_cluster(const uint16_t *q, const uint16_t *k, int n, int d, int Cq, int Ck, int iters,
                    int flags, int32_t *q_assign, int32_t *k_assign, float *q_cent, float *k_cent,
                    int32_t *q_sizes, int32_t *k_sizes) {
    const int warm = flags & 1, identity = (flags >> 1) & 1;
    double *M = (double *)malloc(sizeof(double) * (size_t)d * d);
    float *tmp = (float *)malloc(sizeof(float) * (size_t)(Cq > Ck ? Cq : Ck) * d);
    if (!warm) {
        oracle_init_centroids(q, n, d, Cq, q_cent);
        oracle_init_centroids(k, n, d, Ck, k_cent);
    }
    for (int it = 0; it < iters; ++it) {
        oracle_metric(k_cent, k_sizes, Ck, d, identity || (it == 0 && !warm), M);
        oracle_assign(q, n, d, q_cent, Cq, M, q_assign, NULL, NULL);
        oracle_update(q, n, d, q_assign, Cq, q_cent, tmp, q_sizes);
        memcpy(q_cent, tmp, sizeof(float) * (size_t)Cq * d);
        oracle_metric(q_cent, q_sizes, Cq, d, identity, M);
        oracle_assign(k, n, d, k_cent, Ck, M, k_assign, NULL, NULL);
        oracle_update(k, n, d, k_assign, Ck, k_cent, tmp, k_sizes);
        memcpy(k_cent, tmp, sizeof(float) * (size_t)Ck * d);
    }
    free(M);
    free(tmp);
}

/* Cluster-pair importance ([PSA] sec. 2 on SVG2: centroid-level scores     */
/* and top-k cluster selection; [iCATS] 4, scores at the cluster level).     */
/* Reading: importance = estimated attention mass of the pair. Query cluster */
/* a puts softmax weight n_b e^{s_ab} / Z_a on key cluster b, with           */
/*   s_ab = scale * mu_a . c_b,  Z_a = sum_b n_b e^{s_ab - m_a},             */
/*   m_a = max_{b : n_b > 0} s_ab,  w_ab = n_a * n_b e^{s_ab - m_a} / Z_a,   */
/* so sum_b w_ab = n_a and sum_ab w_ab = N. Precision: fp32 with this exact  */
/* operation order (sequential fmaf dot product, sequential fmaf sum over b  */
/* in ascending order), because the kept set is an integer decision that the */
/* GPU must reproduce bit for bit. top1[a] = argmax_b w_ab, ties to lower b. */
void oracle_pair_mass(const float *q_cent, const float *k_cent, const int32_t *q_sizes,
                      const int32_t *k_sizes, int Cq, int Ck, int d, float scale, float *w,
                      int32_t *top1) {
    float *s = (float *)malloc(sizeof(float) * (size_t)Ck);
    float *e = (float *)malloc(sizeof(float) * (size_t)Ck);
    for (int a = 0; a < Cq; ++a) {
        const float *mu = q_cent + (size_t)a * d;
        int any = 0;
        float m = -INFINITY;
        for (int b = 0; b < Ck; ++b) {
            const float *c = k_cent + (size_t)b * d;
            float acc = 0.0f;
            for (int i = 0; i < d; ++i) acc = fmaf(mu[i], c[i], acc);
            s[b] = scale * acc;
            if (k_sizes[b] > 0) {
                if (!any || s[b] > m) m = s[b];
                any = 1;
            }
        }
        float Z = 0.0f;
        for (int b = 0; b < Ck; ++b) {
            e[b] = k_sizes[b] > 0 ? oracle_exp(s[b] - m) : 0.0f;
            Z = fmaf((float)k_sizes[b], e[b], Z);
        }
        int arg = 0;
        for (int b = 0; b < Ck; ++b) {
            float t = (float)k_sizes[b] * e[b];
            float u = (float)q_sizes[a] * t;
            float wab = Z > 0.0f ? u / Z : 0.0f;
            w[(size_t)a * Ck + b] = wab;
            if (wab > w[(size_t)a * Ck + arg]) arg = b;
        }
        top1[a] = arg;
    }
    free(s);
    free(e);
}

typedef struct {
    int forced;
    float w;
    int a, b;
} pair_t;

/* order: forced first, then w descending, then a ascending, then b ascending */
static int pair_cmp(const void *pa, const void *pb) {
    const pair_t *x = (const pair_t *)pa, *y = (const pair_t *)pb;
    if (x->forced != y->forced) return x->forced ? -1 : 1;
    if (x->w != y->w) return x->w > y->w ? -1 : 1;
    if (x->a != y->a) return x->a < y->a ? -1 : 1;
    if (x->b != y->b) return x->b < y->b ? -1 : 1;
    return 0;
}

/* Pair selection (spec budget; [iCATS] 4.2 top-p).                     */
/* mode 0 (keep ratio r): K = ceil(r * Cq * Ck) pairs per head, the product  */
/* taken in fp32 (so r = 0.05 of 1400 pairs gives 70, not 71). Reading: each */
/* query cluster first keeps its top-1 key cluster (so no softmax row is     */
/* empty), then pairs are taken by w descending (ties a asc, b asc) until K;  */
/* if K < Cq exactly the Cq forced pairs are kept.                            */
/* mode 1 (top-p): masses in fixed point floor(w * 2^32); keep the shortest   */
/* prefix of the same order whose mass reaches ceil(p * total), and at least  */
/* the forced pairs.                                                          */
/* has_text: the text key group (bit Ck) is kept by every query cluster and  */
/* the text query group (row Cq) keeps every key cluster and the text keys;  */
/* these are not counted in the budget.                                      */
int oracle_select(const float *w, const int32_t *top1, int Cq, int Ck, int mode, float keep,
                  float top_p, int has_text, uint64_t *kmask, int W) {
    size_t P = (size_t)Cq * Ck;
    pair_t *pairs = (pair_t *)malloc(sizeof(pair_t) * P);
    for (int a = 0; a < Cq; ++a)
        for (int b = 0; b < Ck; ++b) {
            pair_t *p = &pairs[(size_t)a * Ck + b];
            p->forced = (b == top1[a]);
            p->w = w[(size_t)a * Ck + b];
            p->a = a;
            p->b = b;
        }
    qsort(pairs, P, sizeof(pair_t), pair_cmp);
    long long L;
    if (mode == 0) {
        float kf = ceilf(keep * (float)((long long)Cq * Ck));
        L = (long long)kf;
        if (L > (long long)P) L = (long long)P;
        if (L < Cq) L = Cq;
    } else {
        long long total = 0;
        for (size_t i = 0; i < P; ++i) total += (long long)floor((double)pairs[i].w * 4294967296.0);
        long long target = (long long)ceil((double)top_p * (double)total);
        long long cum = 0;
        L = 0;
        while (L < (long long)P && cum < target) {
            cum += (long long)floor((double)pairs[L].w * 4294967296.0);
            ++L;
        }
        if (L < Cq) L = Cq;
    }
    int rows = Cq + (has_text ? 1 : 0);
    memset(kmask, 0, sizeof(uint64_t) * (size_t)rows * W);
    for (long long i = 0; i < L; ++i) {
        int a = pairs[i].a, b = pairs[i].b;
        kmask[(size_t)a * W + b / 64] |= (uint64_t)1 << (b % 64);
    }
    if (has_text) {
        for (int a = 0; a < Cq; ++a) kmask[(size_t)a * W + Ck / 64] |= (uint64_t)1 << (Ck % 64);
        for (int b = 0; b <= Ck; ++b) kmask[(size_t)Cq * W + b / 64] |= (uint64_t)1 << (b % 64);
    }
    free(pairs);
    return (int)L;
}

static int popcount64(uint64_t v) {
    int c = 0;
    while (v) {
        v &= v - 1;
        ++c;
    }
    return c;
}

static int mask_equal(const uint64_t *x, const uint64_t *y, int W) {
    for (int i = 0; i < W; ++i)
        if (x[i] != y[i]) return 0;
    return 1;
}

static int mask_hamming(const uint64_t *x, const uint64_t *y, int W) {
    int h = 0;
    for (int i = 0; i < W; ++i) h += popcount64(x[i] ^ y[i]);
    return h;
}

static long long tiles_of(const int32_t *sizes, int C, int bq) {
    long long t = 0;
    for (int a = 0; a < C; ++a) t += (sizes[a] + bq - 1) / bq;
    return t;
}

/* Tail merging ([iCATS] 3.3, 4.3, E.1), on the query clusters of one head.   */
/* (i) Query clusters whose key-cluster masks are identical are merged: the  */
/*     sizes add up and the tokens take the label of the lowest-numbered     */
/*     non-empty cluster with that mask. The attention pattern of every token */
/*     is unchanged.                                                          */
/* (ii) `rounds` (two) rounds: the tail of a cluster is t_a = n_a mod block_q */
/*     (the rows of its last, partly filled query block). Among clusters with */
/*     t > 0, a and b may pair when t_a + t_b <= block_q; each cluster's      */
/*     nearest partner is the one with the smallest Hamming distance between */
/*     masks (ties to the lower id). Mutually nearest pairs move the smaller */
/*     tail (equal tails: the higher id's) into the other cluster, whose mask */
/*     becomes the union of both. All decisions of a round use the state at  */
/*     the start of that round.                                              */
/* Readings: the tail tokens moved are the donor's t highest token indices;  */
/* clusters left empty are dropped (size 0, no query blocks).                */
int oracle_tail_merge(uint64_t *kmask, int32_t *sizes, int32_t *label, int n, int Cq, int W,
                      int block_q, int rounds, int32_t *stats) {
    int32_t *rep = (int32_t *)malloc(sizeof(int32_t) * (size_t)Cq);
    int32_t *t = (int32_t *)malloc(sizeof(int32_t) * (size_t)Cq);
    int32_t *near = (int32_t *)malloc(sizeof(int32_t) * (size_t)Cq);
    int32_t *old = (int32_t *)malloc(sizeof(int32_t) * (size_t)Cq);
    int32_t st[6] = {0, 0, 0, 0, 0, 0};
    st[3] = (int32_t)tiles_of(sizes, Cq, block_q);

    for (int a = 0; a < Cq; ++a) {
        rep[a] = a;
        if (sizes[a] == 0) continue;
        for (int a2 = 0; a2 < a; ++a2) {
            if (sizes[a2] > 0 && mask_equal(kmask + (size_t)a2 * W, kmask + (size_t)a * W, W)) {
                rep[a] = a2;
                break;
            }
        }
    }
    for (int i = 0; i < n; ++i) label[i] = rep[label[i]];
    memcpy(old, sizes, sizeof(int32_t) * (size_t)Cq);
    for (int a = 0; a < Cq; ++a) sizes[a] = 0;
    for (int a = 0; a < Cq; ++a) {
        sizes[rep[a]] += old[a];
        if (rep[a] != a) st[0] += 1;
    }

    for (int r = 0; r < rounds; ++r) {
        for (int a = 0; a < Cq; ++a) t[a] = sizes[a] % block_q;
        for (int a = 0; a < Cq; ++a) {
            near[a] = -1;
            if (t[a] == 0) continue;
            int best = 1 << 30;
            for (int b = 0; b < Cq; ++b) {
                if (b == a || t[b] == 0 || t[a] + t[b] > block_q) continue;
                int h = mask_hamming(kmask + (size_t)a * W, kmask + (size_t)b * W, W);
                if (h < best) {
                    best = h;
                    near[a] = b;
                }
            }
        }
        for (int a = 0; a < Cq; ++a) {
            int b = near[a];
            if (b <= a || near[b] != a) continue;
            int donor, recv;
            if (t[a] < t[b]) {
                donor = a;
                recv = b;
            } else {
                donor = b;
                recv = a;
            }
            int moved = 0;
            for (int i = n - 1; i >= 0 && moved < t[donor]; --i) {
                if (label[i] == donor) {
                    label[i] = recv;
                    ++moved;
                }
            }
            sizes[recv] += moved;
            sizes[donor] -= moved;
            for (int wi = 0; wi < W; ++wi) kmask[(size_t)recv * W + wi] |= kmask[(size_t)donor * W + wi];
            st[1 + (r < 1 ? 0 : 1)] += 1;
            st[5] += moved;
        }
    }
    st[4] = (int32_t)tiles_of(sizes, Cq, block_q);
    int nonempty = 0;
    for (int a = 0; a < Cq; ++a) nonempty += sizes[a] > 0;
    if (stats) memcpy(stats, st, sizeof st);
    free(rep);
    free(t);
    free(near);
    free(old);
    return nonempty;
}

/* Token permutation into cluster order ([PSA] sec. 2 on SVG2's semantic-    */
/* aware permutation): a stable counting sort by label, so each group is one */
/* contiguous range in ascending token order. off has G + 1 entries.         */
void oracle_permute(const int32_t *label, int n, int G, int32_t *perm, int32_t *off) {
    int32_t *cnt = (int32_t *)calloc((size_t)G + 1, sizeof(int32_t));
    for (int i = 0; i < n; ++i) cnt[label[i]] += 1;
    off[0] = 0;
    for (int g = 0; g < G; ++g) off[g + 1] = off[g] + cnt[g];
    for (int g = 0; g < G; ++g) cnt[g] = off[g];
    for (int i = 0; i < n; ++i) perm[cnt[label[i]]++] = i;
    free(cnt);
}

/* Query blocks: each group cut into tiles of at most block_q rows. */
int oracle_tiles(const int32_t *off, int G, int block_q, int32_t *tiles) {
    int c = 0;
    for (int g = 0; g < G; ++g) {
        int ng = off[g + 1] - off[g];
        for (int s = 0; s < ng; s += block_q) {
            tiles[3 * c + 0] = g;
            tiles[3 * c + 1] = off[g] + s;
            tiles[3 * c + 2] = ng - s < block_q ? ng - s : block_q;
            ++c;
        }
    }
    return c;
}

/* Block-sparse attention, restated per query row: row i of query group     */
/* a = q_label[i] attends to every key j whose group k_label[j] has its bit  */
/* set in kmask[a]: o_i = sum_j softmax_j(scale * q_i.k_j) v_j over those   */
/* keys, in fp64. A row with no kept key gets o_i = 0. psum[i] is the sum of */
/* the normalised probabilities, nkeys[i] the number of keys attended.      */
void oracle_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int n, int d,
                      float scale, const int32_t *q_label, const int32_t *k_label,
                      const uint64_t *kmask, int W, const int32_t *rows, int nrows, double *out,
                      double *psum, int64_t *nkeys) {
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double *qi = (double *)malloc(sizeof(double) * (size_t)d);
    double sc = (double)scale;
    for (int r = 0; r < nrows; ++r) {
        int i = rows[r];
        const uint64_t *mrow = kmask + (size_t)q_label[i] * W;
        for (int c = 0; c < d; ++c) qi[c] = bf16_val(q[(size_t)i * d + c]);
        double m = -INFINITY;
        long long cnt = 0;
        for (int j = 0; j < n; ++j) {
            int b = k_label[j];
            if (!((mrow[b / 64] >> (b % 64)) & 1)) {
                s[j] = NAN;
                continue;
            }
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qi[c] * bf16_val(k[(size_t)j * d + c]);
            s[j] = sc * dot;
            if (s[j] > m) m = s[j];
            ++cnt;
        }
        double *o = out + (size_t)r * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (nkeys) nkeys[r] = cnt;
        if (cnt == 0) {
            if (psum) psum[r] = 0.0;
            continue;
        }
        double Z = 0.0;
        for (int j = 0; j < n; ++j)
            if (!isnan(s[j])) Z += exp(s[j] - m);
        double ps = 0.0;
        for (int j = 0; j < n; ++j) {
            if (isnan(s[j])) continue;
            double p = exp(s[j] - m) / Z;
            ps += p;
            for (int c = 0; c < d; ++c) o[c] += p * bf16_val(v[(size_t)j * d + c]);
        }
        if (psum) psum[r] = ps;
    }
    free(s);
    free(qi);
}

/* Dense softmax attention o_i = softmax(scale * q_i K^T) V, fp64. */
void oracle_dense_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int n, int d,
                            float scale, const int32_t *rows, int nrows, double *out) {
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double sc = (double)scale;
    for (int r = 0; r < nrows; ++r) {
        int i = rows[r];
        double m = -INFINITY;
        for (int j = 0; j < n; ++j) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += bf16_val(q[(size_t)i * d + c]) * bf16_val(k[(size_t)j * d + c]);
            s[j] = sc * dot;
            if (s[j] > m) m = s[j];
        }
        double Z = 0.0;
        for (int j = 0; j < n; ++j) Z += exp(s[j] - m);
        double *o = out + (size_t)r * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int j = 0; j < n; ++j) {
            double p = exp(s[j] - m) / Z;
            for (int c = 0; c < d; ++c) o[c] += p * bf16_val(v[(size_t)j * d + c]);
        }
    }
    free(s);
}

/* [PSA] sec. 3.2, Alg. 1 (mask definition): 1 if position i attends position */
/* j under M(Tw, To, Ts, Sw, So, Ss) = prm[0..5], the sequence being frames   */
/* of HW positions. Frame and in-frame index of both, then the inter-frame    */
/* band test on the frame distance and the intra-frame band test on the       */
/* in-frame distance. A stride of INT32_MAX stands for infinity: the distance */
/* never wraps, leaving one diagonal band on that axis.                       */
int oracle_psa_attends(long long i, long long j, long long HW, const int32_t *prm) {
    const long long tq = i / HW, sq = i % HW;
    const long long tk = j / HW, sk = j % HW;
    const long long dt = tk - tq;
    if (llabs(dt - prm[1]) % prm[2] > (long long)prm[0] - 1) return 0;
    const long long ds = sk - sq;
    return llabs(ds - prm[4]) % prm[5] <= (long long)prm[3] - 1;
}

/* [PSA] sec. 3.2 (PSABlock; block-centric layout) and Alg. 1: the sparse    */
/* plan of one head for a static stripe mask. Video tokens lie in (T, H, W)   */
/* raster order, n_text text tokens follow them. A token's label is its       */
/* PSABlock (t / bt, y / bh, x / bw), numbered in raster order over the grid  */
/* (T', H', W') = (ceil(T / bt), ceil(H / bh), ceil(W / bw)); blocks on the   */
/* far edges are smaller (no padding tokens are made). Text tokens take label */
/* nb = T'H'W'. Masking is at PSABlock granularity: bit b of row a is Alg. 1  */
/* with i = a, j = b and HW = H'W' (block distances). The text row attends    */
/* every group and every row attends the text group. Writes label[N],         */
/* kmask[G][Wd] (G = nb + (n_text > 0), Wd = ceil(G / 64)) and sizes[G];      */
/* returns nb.                                                                */
int oracle_psa_plan(int T, int H, int W, int bt, int bh, int bw, int n_text, const int32_t *prm,
                    int32_t *label, uint64_t *kmask, int32_t *sizes) {
    const int Tb = (T + bt - 1) / bt, Hb = (H + bh - 1) / bh, Wb = (W + bw - 1) / bw;
    const int nb = Tb * Hb * Wb;
    const int G = nb + (n_text > 0), Wd = (G + 63) / 64;
    const long long nv = (long long)T * H * W;
    for (int g = 0; g < G; ++g) sizes[g] = 0;
    for (long long i = 0; i < nv; ++i) {
        const int t = (int)(i / ((long long)H * W));
        const int y = (int)((i / W) % H);
        const int x = (int)(i % W);
        const int a = ((t / bt) * Hb + y / bh) * Wb + x / bw;
        label[i] = a;
        sizes[a] += 1;
    }
    for (int e = 0; e < n_text; ++e) {
        label[nv + e] = nb;
        sizes[nb] += 1;
    }
    memset(kmask, 0, sizeof(uint64_t) * (size_t)G * Wd);
    for (int a = 0; a < G; ++a) {
        for (int b = 0; b < G; ++b) {
            int keep;
            if (a == nb || b == nb) keep = 1; /* text row / text column */
            else keep = oracle_psa_attends(a, b, (long long)Hb * Wb, prm);
            if (keep) kmask[(size_t)a * Wd + b / 64] |= 1ull << (b % 64);
        }
    }
    return nb;
}

/* ------------------------------------------------------------------------ */
/* [iCATS] 4.2 and appendix A: the top-p of each denoising call follows a     */
/* smooth function of log SNR, fixed offline from the noise schedule; calls   */
/* before the first sparse one stay dense; the budget is steady early and     */
/* late and falls in the middle; tau and p_min are its parameters. The pages  */
/* give no formula. Reading (parity unpinned by the pages):                   */
/*   noise level of call t (flow matching, t = 0 is pure noise, `shift` the   */
/*   usual timestep shift):  s = 1 - t/steps,  sigma = shift s / (1 + (shift-1) s) */
/*   lambda = log SNR = 2 ln((1 - sigma) / sigma)                             */
/*   p(t) = p_min + (tau - p_min) / (1 + e^lambda)   for t >= warmup,         */
/*   p(t) = 1                                        for t <  warmup.         */
/* So p = tau at pure noise, p_min in the noise-free limit, and the midpoint  */
/* (tau + p_min) / 2 where SNR = 1; the logistic in lambda keeps both ends    */
/* flat. The value is rounded once to fp32 (build_mask takes an fp32 p).      */
/* ------------------------------------------------------------------------ */
int oracle_snr_top_p(int steps, int warmup, double p_min, double tau, double shift, float *p) {
    if (steps < 1 || warmup < 0 || !(p_min >= 0.0) || !(tau >= p_min) || !(tau <= 1.0) ||
        !(shift > 0.0) || !p)
        return -1;
    for (int t = 0; t < steps; ++t) {
        if (t < warmup) {
            p[t] = 1.0f;
            continue;
        }
        double s = 1.0 - (double)t / (double)steps;
        double sigma = shift * s / (1.0 + (shift - 1.0) * s);
        double noisy_share;
        if (sigma >= 1.0) {
            noisy_share = 1.0; /* lambda = -infinity */
        } else {
            double lambda = 2.0 * log((1.0 - sigma) / sigma);
            noisy_share = 1.0 / (1.0 + exp(lambda));
        }
        p[t] = (float)(p_min + (tau - p_min) * noisy_share);
    }
    return 0;
}
