/*
 * scope_oracle.c -- plain, slow, fp64 CPU oracle for centroid-guided sparse
 * attention in the SCOPE formulation.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  It shares no
 * code, header, table or constant with the CUDA path and never calls it.
 *
 * Sources (by page title and section):
 *   [SCOPE]   "SCOPE: Subspace Clustering with Online Per-Head Top-K
 *             Estimation for Sparse Video Attention", abstract.
 *   [CLUSTER] "ClusterAttention: A training-free speedup of bidirectional
 *             attention", abstract.
 * The pages are abstract-level; every concrete choice below that they leave
 * open is a stated reading (R1..R16) listed beside the function it affects.
 *
 * Conventions: one (batch, head) at a time; row-major [rows][D] arrays of
 * double; labels int32; counts int64.  Every function is single-threaded and
 * uses plain loops, qsort and libm only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* 3D rotary position embedding [SCOPE: "post-RoPE keys", "3D-RoPE-aligned  */
/* key subspace"].                                                          */
/* R1: token n sits at (t, y, x) with n = (t*Hh + y)*W + x, positions from 0;*/
/*     pair i of an axis block occupies dims (off+2i, off+2i+1) and turns by */
/*     pos * theta^(-2i/d_s).                                               */
/* R2: the head dim is split into contiguous [t | h | w] blocks of sizes     */
/*     d_t, d_h, d_w (each even, summing to D).                             */
/* ------------------------------------------------------------------------ */
int orc_rope3d(double *x, int64_t N, int64_t D, const int32_t *grid,
               const int32_t *dsplit, double theta)
{
    const int64_t T = grid[0], Hh = grid[1], W = grid[2];
    if (T == 0) return 0; /* no grid: identity */
    if (T * Hh * W != N) return 1;
    if ((int64_t)dsplit[0] + dsplit[1] + dsplit[2] != D) return 2;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t pos[3] = {n / (Hh * W), (n / W) % Hh, n % W};
        int64_t off = 0;
        for (int s = 0; s < 3; ++s) {
            const int64_t ds = dsplit[s];
            for (int64_t i = 0; i < ds / 2; ++i) {
                const double phi = (double)pos[s] * pow(theta, -2.0 * (double)i / (double)ds);
                const double c = cos(phi), sn = sin(phi);
                double *p = x + n * D + off + 2 * i;
                const double x0 = p[0], x1 = p[1];
                p[0] = x0 * c - x1 * sn;
                p[1] = x0 * sn + x1 * c;
            }
            off += ds;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* k-means (Lloyd) [SCOPE: keys "clusters them independently" per subspace, */
/* queries grouped into "query clusters"].                                  */
/* R3: Lloyd iterations on squared Euclidean distance.                      */
/* R5: init c_j = x[off + j*floor(N/C)], off = seed mod floor(N/C).         */
/* R6: argmin ties go to the lowest centroid index.                         */
/* R7: an empty cluster keeps its previous centroid.                        */
/* R8: `iters` rounds of (assign, update), then one final assign; labels are */
/*     that final assign, centroids those after the last update.            */
/* ------------------------------------------------------------------------ */
static double sqdist(const double *a, const double *b, int64_t D)
{
    double s = 0.0;
    for (int64_t k = 0; k < D; ++k) {
        const double t = a[k] - b[k];
        s += t * t;
    }
    return s;
}

/* labels[n] = argmin_j ||x_n - c_j||^2.  d1/d2 (optional) receive the best
 * and second-best squared distance, for near-tie accounting in tests. */
void orc_kmeans_assign(const double *x, int64_t N, int64_t ldx, int64_t D,
                       const double *cent, int64_t C, int64_t ldc,
                       int32_t *labels, double *d1, double *d2)
{
    for (int64_t n = 0; n < N; ++n) {
        double best = INFINITY, second = INFINITY;
        int64_t arg = 0;
        for (int64_t j = 0; j < C; ++j) {
            const double d = sqdist(x + n * ldx, cent + j * ldc, D);
            if (d < best) {
                second = best;
                best = d;
                arg = j;
            } else if (d < second) {
                second = d;
            }
        }
        labels[n] = (int32_t)arg;
        if (d1) d1[n] = best;
        if (d2) d2[n] = second;
    }
}

/* cent_j <- mean of the rows labelled j (R7: empty keeps cent_j). */
void orc_kmeans_update(const double *x, int64_t N, int64_t ldx, int64_t D,
                       const int32_t *labels, int64_t C, double *cent,
                       int64_t ldc, int64_t *sizes)
{
    double *sum = (double *)calloc((size_t)(C * (D > 0 ? D : 1)), sizeof(double));
    int64_t *cnt = (int64_t *)calloc((size_t)C, sizeof(int64_t));
    for (int64_t n = 0; n < N; ++n) {
        const int64_t j = labels[n];
        cnt[j] += 1;
        for (int64_t k = 0; k < D; ++k) sum[j * D + k] += x[n * ldx + k];
    }
    for (int64_t j = 0; j < C; ++j) {
        if (sizes) sizes[j] = cnt[j];
        if (cnt[j] == 0) continue;
        for (int64_t k = 0; k < D; ++k) cent[j * ldc + k] = sum[j * D + k] / (double)cnt[j];
    }
    free(sum);
    free(cnt);
}

/* Sum of squared distances to the assigned centroid (the k-means objective). */
double orc_kmeans_objective(const double *x, int64_t N, int64_t ldx, int64_t D,
                            const int32_t *labels, const double *cent, int64_t ldc)
{
    double J = 0.0;
    for (int64_t n = 0; n < N; ++n) J += sqdist(x + n * ldx, cent + labels[n] * ldc, D);
    return J;
}

int orc_kmeans(const double *x, int64_t N, int64_t ldx, int64_t D, int64_t C,
               int iters, uint32_t seed, int32_t *labels, double *cent,
               int64_t *sizes)
{
    if (C < 1 || C > N) return 1;
    const int64_t stride = N / C;
    const int64_t off = (int64_t)(seed % (uint64_t)stride);
    for (int64_t j = 0; j < C; ++j)
        for (int64_t k = 0; k < D; ++k) cent[j * D + k] = x[(off + j * stride) * ldx + k];
    for (int it = 0; it < iters; ++it) {
        orc_kmeans_assign(x, N, ldx, D, cent, C, D, labels, NULL, NULL);
        orc_kmeans_update(x, N, ldx, D, labels, C, cent, D, NULL);
    }
    orc_kmeans_assign(x, N, ldx, D, cent, C, D, labels, NULL, NULL);
    for (int64_t j = 0; j < C; ++j) sizes[j] = 0;
    for (int64_t n = 0; n < N; ++n) sizes[labels[n]] += 1;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Centroid-score lookup table [SCOPE: "aggregates the corresponding        */
/* centroid scores through lookup tables"]: lut[c][a] is the dot product of */
/* query centroid c, restricted to one key subspace, with key centroid a of */
/* that subspace.                                                           */
/* ------------------------------------------------------------------------ */
void orc_lut(const double *qc, int64_t Cq, int64_t ldq, const double *kc,
             int64_t Ck, int64_t ldk, int64_t Ds, double *lut)
{
    for (int64_t c = 0; c < Cq; ++c)
        for (int64_t a = 0; a < Ck; ++a) {
            double s = 0.0;
            for (int64_t k = 0; k < Ds; ++k) s += qc[c * ldq + k] * kc[a * ldk + k];
            lut[c * Ck + a] = s;
        }
}

/* Per-key proxy score of one query cluster: the sum of its three subspace
 * table entries selected by the key's subspace codes [SCOPE]. */
void orc_proxy_scores(const double *lut_t, const double *lut_h, const double *lut_w,
                      const int32_t *a_t, const int32_t *a_h, const int32_t *a_w,
                      int64_t N, double *s)
{
    for (int64_t j = 0; j < N; ++j) s[j] = lut_t[a_t[j]] + lut_h[a_h[j]] + lut_w[a_w[j]];
}

/* ------------------------------------------------------------------------ */
/* Key order used by every selection: score descending, then key index      */
/* ascending (R6 applied to selection ties).                                */
/* ------------------------------------------------------------------------ */
static const double *g_sort_scores; /* qsort has no context argument */

static int cmp_desc(const void *pa, const void *pb)
{
    const int64_t a = *(const int64_t *)pa, b = *(const int64_t *)pb;
    const double sa = g_sort_scores[a], sb = g_sort_scores[b];
    if (sa > sb) return -1;
    if (sa < sb) return 1;
    return (a > b) - (a < b);
}

void orc_order(const double *s, int64_t N, int64_t *order)
{
    for (int64_t j = 0; j < N; ++j) order[j] = j;
    g_sort_scores = s;
    qsort(order, (size_t)N, sizeof(int64_t), cmp_desc);
}

/* ------------------------------------------------------------------------ */
/* Top-p [SCOPE: "existing hybrid Top-p/fixed Top-k selection"]: the number  */
/* of keys in the shortest prefix of the order above whose softmax(scale*s)  */
/* mass reaches p of the total (R9: scale = 1/sqrt(d); R14: ">= p").         */
/* p >= 1 keeps every key.  `mass_out` (optional) gets the prefix mass       */
/* fraction at the cut, for near-tie accounting.                            */
/* ------------------------------------------------------------------------ */
int64_t orc_topp_count(const double *s, int64_t N, double p, double scale,
                       double *mass_out)
{
    if (N <= 0) return 0;
    int64_t *order = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    orc_order(s, N, order);
    const double smax = s[order[0]];
    double total = 0.0;
    for (int64_t j = 0; j < N; ++j) total += exp((s[j] - smax) * scale);
    int64_t m = N;
    double cum = 0.0;
    if (p < 1.0) {
        const double target = p * total;
        for (int64_t i = 0; i < N; ++i) {
            cum += exp((s[order[i]] - smax) * scale);
            if (cum >= target) {
                m = i + 1;
                break;
            }
        }
    } else {
        cum = total;
    }
    if (mass_out) *mass_out = cum / total;
    free(order);
    return m;
}

/* Prefix mass fraction of the first m keys of the order (near-tie checks). */
double orc_prefix_mass(const double *s, int64_t N, int64_t m, double scale)
{
    int64_t *order = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    orc_order(s, N, order);
    const double smax = s[order[0]];
    double total = 0.0, cum = 0.0;
    for (int64_t j = 0; j < N; ++j) total += exp((s[j] - smax) * scale);
    for (int64_t i = 0; i < m && i < N; ++i) cum += exp((s[order[i]] - smax) * scale);
    free(order);
    return cum / total;
}

/* ------------------------------------------------------------------------ */
/* Online per-head Top-k [SCOPE: a head-specific Top-k is the average of the */
/* initial retained counts weighted by query-cluster size; extra keys go    */
/* only to clusters whose initial count falls below it].                    */
/* r[c] is the initial (hybrid) count max(|P_c|, k_min) capped at N.         */
/* R10: K_h = ceil(sum_c |c| r_c / sum_c |c|) in exact integers; since r_c   */
/*      is an integer, r_c < mean  <=>  r_c < ceil(mean), so topping up to  */
/*      K_h changes exactly the clusters below the mean.  n_c = 0 for empty  */
/*      clusters (no query reads their list).                               */
/* ------------------------------------------------------------------------ */
int64_t orc_online_topk(const int64_t *sizes, const int64_t *r, int64_t C,
                        int64_t N, int online, int64_t *n)
{
    int64_t num = 0, den = 0;
    for (int64_t c = 0; c < C; ++c) {
        num += sizes[c] * r[c];
        den += sizes[c];
    }
    const int64_t K = den > 0 ? (num + den - 1) / den : 0;
    for (int64_t c = 0; c < C; ++c) {
        int64_t v = r[c];
        if (online && K > v) v = K;
        if (v > N) v = N;
        n[c] = sizes[c] > 0 ? v : 0;
    }
    return online ? K : 0;
}

/* ------------------------------------------------------------------------ */
/* EG-Sparse ["EG-Sparse", abstract: low-entropy heads are routed to a       */
/* grouped cross-head pool, high-entropy heads keep per-row selection, using */
/* only scores the sparse pipeline already has].  Readings (R17):           */
/*  - a row is a query cluster c of head h; its proxy distribution is        */
/*    pi_c(j) = softmax_j(scale * s_c(j)) over all N keys;                   */
/*  - head entropy E_h = sum_c |c| H(pi_c) / (sum_c |c| * ln N), H in nats,  */
/*    so 0 <= E_h <= 1 (1: uniform rows);                                    */
/*  - head h is low-entropy iff E_h < tau; heads are grouped G at a time in  */
/*    index order, and a group's low-entropy heads form one pool;           */
/*  - in a pool every (h, c, j) competes at once: entries ranked by pi_c(j)  */
/*    descending (ties: h, then c, then the row's own key order), each       */
/*    carrying mass |c| pi_c(j); the shortest prefix reaching p of the       */
/*    pool's total mass (sum over its heads of sum_c |c|) is kept, and       */
/*    |P_c| = the number of kept entries of row c -- a prefix of that row's  */
/*    own key order, so lists, k_min and the online Top-k follow as before.  */
/* ------------------------------------------------------------------------ */

/* Normalised entropy of one head: s [C][N] proxy scores, sizes [C]. */
double orc_head_entropy(const double *s, const int64_t *sizes, int64_t C, int64_t N, double scale)
{
    if (N <= 1) return 0.0;
    double num = 0.0, den = 0.0;
    for (int64_t c = 0; c < C; ++c) {
        if (sizes[c] <= 0) continue;
        const double *sc = s + c * N;
        double mx = sc[0];
        for (int64_t j = 1; j < N; ++j) mx = sc[j] > mx ? sc[j] : mx;
        double Z = 0.0;
        for (int64_t j = 0; j < N; ++j) Z += exp((sc[j] - mx) * scale);
        double H = 0.0;
        for (int64_t j = 0; j < N; ++j) {
            const double pj = exp((sc[j] - mx) * scale) / Z;
            if (pj > 0.0) H -= pj * log(pj);
        }
        num += (double)sizes[c] * H;
        den += (double)sizes[c];
    }
    return den > 0.0 ? num / (den * log((double)N)) : 0.0;
}

typedef struct {
    double logp;     /* ln pi of the entry */
    double mass;     /* |c| pi */
    int64_t h, c, pos; /* pool head, row, place in the row's own order */
} pool_entry;

static int cmp_pool(const void *pa, const void *pb)
{
    const pool_entry *a = (const pool_entry *)pa, *b = (const pool_entry *)pb;
    if (a->logp > b->logp) return -1;
    if (a->logp < b->logp) return 1;
    if (a->h != b->h) return (a->h > b->h) - (a->h < b->h);
    if (a->c != b->c) return (a->c > b->c) - (a->c < b->c);
    return (a->pos > b->pos) - (a->pos < b->pos);
}

/* Pooled Top-p counts of one pool: s [Hp][C][N] proxy scores of the pool's
 * heads, sizes [Hp][C]; counts [Hp][C] receives |P_c| (N when p >= 1).  A
 * cluster with no queries has no rows to pool: it keeps its own per-row
 * Top-p count.  Returns the kept mass fraction (for near-tie accounting). */
double orc_pooled_topp(const double *s, const int64_t *sizes, int64_t Hp, int64_t C, int64_t N, double p,
                       double scale, int64_t *counts)
{
    int64_t E = 0;
    for (int64_t i = 0; i < Hp * C; ++i) {
        counts[i] = p >= 1.0 ? N : 0;
        if (sizes[i] > 0) E += N;
        else if (p < 1.0) counts[i] = orc_topp_count(s + i * N, N, p, scale, NULL);
    }
    if (p >= 1.0 || E == 0) return 1.0;
    pool_entry *e = (pool_entry *)malloc((size_t)E * sizeof(pool_entry));
    int64_t *order = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    double total = 0.0;
    int64_t m = 0;
    for (int64_t h = 0; h < Hp; ++h)
        for (int64_t c = 0; c < C; ++c) {
            if (sizes[h * C + c] <= 0) continue;
            const double *sc = s + (h * C + c) * N;
            orc_order(sc, N, order);
            const double mx = sc[order[0]];
            double Z = 0.0;
            for (int64_t j = 0; j < N; ++j) Z += exp((sc[j] - mx) * scale);
            const double lnZ = log(Z);
            for (int64_t i = 0; i < N; ++i) {
                const double a = (sc[order[i]] - mx) * scale - lnZ;
                e[m].logp = a;
                e[m].mass = (double)sizes[h * C + c] * exp(a);
                e[m].h = h;
                e[m].c = c;
                e[m].pos = i;
                total += e[m].mass;
                ++m;
            }
        }
    qsort(e, (size_t)E, sizeof(pool_entry), cmp_pool);
    const double target = p * total;  /* total = sum over the pooled rows of |c| */
    double cum = 0.0;
    for (int64_t i = 0; i < E; ++i) {
        cum += e[i].mass;
        counts[e[i].h * C + e[i].c] += 1;
        if (cum >= target) break;
    }
    free(order);
    free(e);
    return total > 0.0 ? cum / total : 1.0;
}

/* ------------------------------------------------------------------------ */
/* VMoBA block-granular selection ["VMoBA: Mixture-of-Block Attention for    */
/* Video Diffusion Models", abstract items (1) a layer-wise recurrent 1D-2D- */
/* 3D block partition and (3) threshold selection of blocks by cumulative    */
/* similarity].  Readings (R18):                                           */
/*  - kind 1: runs of bt*bh*bw consecutive tokens in raster order; kind 2:  */
/*    bh x bw tiles inside each frame; kind 3: bt x bh x bw cubes; ragged   */
/*    edge blocks; blocks numbered in raster order of their corners.  The   */
/*    caller cycles the kind with the layer index (the recurrent scheme).   */
/*  - a key block's representative is the mean of its post-RoPE keys; query */
/*    cluster c scores block b by s_c(b) = qbar_c . kbar_b;                  */
/*  - blocks are ranked by s_c(b) descending; each weighs |b| e^{scale s};   */
/*    the shortest prefix whose weight reaches p of the total is kept, and  */
/*    blocks tied with the last kept one are kept too (whole blocks only).  */
/* ------------------------------------------------------------------------ */

/* Block id of every token of a T x Hh x W grid; returns the block count. */
int64_t orc_block_ids(int32_t T, int32_t Hh, int32_t W, int kind, int32_t bt, int32_t bh, int32_t bw,
                      int32_t *ids)
{
    const int64_t N = (int64_t)T * Hh * W;
    if (kind == 1) {
        const int64_t len = (int64_t)bt * bh * bw;
        for (int64_t n = 0; n < N; ++n) ids[n] = (int32_t)(n / len);
        return (N + len - 1) / len;
    }
    const int64_t nbt = kind == 2 ? T : (T + bt - 1) / bt;
    const int64_t nbh = (Hh + bh - 1) / bh, nbw = (W + bw - 1) / bw;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t t = n / ((int64_t)Hh * W), y = (n / W) % Hh, x = n % W;
        const int64_t tb = kind == 2 ? t : t / bt;
        ids[n] = (int32_t)((tb * nbh + y / bh) * nbw + x / bw);
    }
    return nbt * nbh * nbw;
}

/* Keys kept by one query cluster: s [Nb] block scores, sizes [Nb]; keep[b]
 * set to 1 for kept blocks; returns the kept key count. */
int64_t orc_block_select(const double *s, const int64_t *sizes, int64_t Nb, double p, double scale, int8_t *keep)
{
    int64_t *order = (int64_t *)malloc((size_t)(Nb > 0 ? Nb : 1) * sizeof(int64_t));
    orc_order(s, Nb, order);
    double mx = -INFINITY, total = 0.0;
    for (int64_t b = 0; b < Nb; ++b)
        if (sizes[b] > 0 && s[b] > mx) mx = s[b];
    for (int64_t b = 0; b < Nb; ++b) total += (double)sizes[b] * exp((s[b] - mx) * scale);
    for (int64_t b = 0; b < Nb; ++b) keep[b] = 0;
    int64_t kept = 0;
    double cum = 0.0, cut = INFINITY;
    for (int64_t i = 0; i < Nb; ++i) {
        const int64_t b = order[i];
        if (sizes[b] <= 0) continue;
        if (cum >= p * total && s[b] < cut) break;  /* reached, and past the last kept score */
        keep[b] = 1;
        kept += sizes[b];
        cum += (double)sizes[b] * exp((s[b] - mx) * scale);
        if (cum >= p * total && cut == INFINITY) cut = s[b];
    }
    free(order);
    return kept;
}

/* Selected keys of one cluster: the first n keys of the order, written in
 * ascending key index (R11). */
void orc_emit(const double *s, int64_t N, int64_t n, int32_t *out)
{
    int64_t *order = (int64_t *)malloc((size_t)(N > 0 ? N : 1) * sizeof(int64_t));
    orc_order(s, N, order);
    char *take = (char *)calloc((size_t)(N > 0 ? N : 1), 1);
    for (int64_t i = 0; i < n && i < N; ++i) take[order[i]] = 1;
    int64_t w = 0;
    for (int64_t j = 0; j < N; ++j)
        if (take[j]) out[w++] = (int32_t)j;
    free(take);
    free(order);
}

/* ------------------------------------------------------------------------ */
/* Sparse attention [SCOPE: "computed over the selected original keys and   */
/* values"]: o = sum_{j in S} softmax_j(scale * q.k_j) v_j (R12: post-RoPE q */
/* and k, original v, scale 1/sqrt(d)).                                     */
/* ------------------------------------------------------------------------ */
void orc_attn_rows(const double *q, int64_t nq, const double *K, const double *V,
                   int64_t D, const int32_t *sel, int64_t n, double scale, double *o)
{
    double *lg = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    for (int64_t i = 0; i < nq; ++i) {
        const double *qi = q + i * D;
        double mx = -INFINITY;
        for (int64_t t = 0; t < n; ++t) {
            double dot = 0.0;
            const double *kj = K + (int64_t)sel[t] * D;
            for (int64_t k = 0; k < D; ++k) dot += qi[k] * kj[k];
            lg[t] = dot * scale;
            if (lg[t] > mx) mx = lg[t];
        }
        double den = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            lg[t] = exp(lg[t] - mx);
            den += lg[t];
        }
        double *oi = o + i * D;
        for (int64_t k = 0; k < D; ++k) oi[k] = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            const double *vj = V + (int64_t)sel[t] * D;
            const double w = lg[t] / den;
            for (int64_t k = 0; k < D; ++k) oi[k] += w * vj[k];
        }
    }
    free(lg);
}

/* ------------------------------------------------------------------------ */
/* Compensation of excluded clusters [CLUSTER: "compensation of excluded     */
/* clusters through their mean"].                                            */
/* R16: key cluster k (klab) has mean key mu_k and mean value vbar_k over    */
/*      all of its members.  For one query cluster with selected keys S, m_k */
/*      is the number of members of k not in S; every such key enters the   */
/*      softmax through its cluster's mean:                                  */
/*        o = (sum_{j in S} e^{a_j} v_j + sum_k m_k e^{b_k} vbar_k)          */
/*          / (sum_{j in S} e^{a_j} + sum_k m_k e^{b_k}),                    */
/*      a_j = scale q.k_j, b_k = scale q.mu_k.  With every cluster a single  */
/*      key, or with identical keys and values inside each cluster, this is  */
/*      dense attention.                                                    */
/* ------------------------------------------------------------------------ */
void orc_attn_rows_comp(const double *q, int64_t nq, const double *K, const double *V, int64_t N, int64_t D,
                        const int32_t *sel, int64_t n, const int32_t *klab, int64_t C, double scale, double *o)
{
    double *mu = (double *)calloc((size_t)(C * D), sizeof(double));
    double *vb = (double *)calloc((size_t)(C * D), sizeof(double));
    int64_t *size = (int64_t *)calloc((size_t)C, sizeof(int64_t));
    int64_t *m = (int64_t *)calloc((size_t)C, sizeof(int64_t));
    for (int64_t j = 0; j < N; ++j) {
        const int64_t k = klab[j];
        size[k] += 1;
        for (int64_t d = 0; d < D; ++d) {
            mu[k * D + d] += K[j * D + d];
            vb[k * D + d] += V[j * D + d];
        }
    }
    for (int64_t k = 0; k < C; ++k)
        for (int64_t d = 0; d < D; ++d) {
            if (size[k] > 0) {
                mu[k * D + d] /= (double)size[k];
                vb[k * D + d] /= (double)size[k];
            }
        }
    for (int64_t k = 0; k < C; ++k) m[k] = size[k];
    for (int64_t t = 0; t < n; ++t) m[klab[sel[t]]] -= 1;
    double *lg = (double *)malloc((size_t)(n + C > 0 ? n + C : 1) * sizeof(double));
    for (int64_t i = 0; i < nq; ++i) {
        const double *qi = q + i * D;
        double mx = -INFINITY;
        for (int64_t t = 0; t < n; ++t) {
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d) dot += qi[d] * K[(int64_t)sel[t] * D + d];
            lg[t] = dot * scale;
            if (lg[t] > mx) mx = lg[t];
        }
        for (int64_t k = 0; k < C; ++k) {
            if (m[k] <= 0) continue;
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d) dot += qi[d] * mu[k * D + d];
            lg[n + k] = dot * scale;
            if (lg[n + k] > mx) mx = lg[n + k];
        }
        double den = 0.0;
        double *oi = o + i * D;
        for (int64_t d = 0; d < D; ++d) oi[d] = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            const double w = exp(lg[t] - mx);
            den += w;
            for (int64_t d = 0; d < D; ++d) oi[d] += w * V[(int64_t)sel[t] * D + d];
        }
        for (int64_t k = 0; k < C; ++k) {
            if (m[k] <= 0) continue;
            const double w = (double)m[k] * exp(lg[n + k] - mx);
            den += w;
            for (int64_t d = 0; d < D; ++d) oi[d] += w * vb[k * D + d];
        }
        for (int64_t d = 0; d < D; ++d) oi[d] /= den;
    }
    free(lg);
    free(m);
    free(size);
    free(vb);
    free(mu);
}

/* ------------------------------------------------------------------------ */
/* Balanced recursive bisection [CLUSTER: "fast attention-aware recursive    */
/* clustering" with "power-of-two cluster sizes" for block-sparse attention].*/
/* R13: at a node of n points (members in token order) run 2-means seeded   */
/*      with members 0 and n/2; each assign ranks the members by             */
/*      delta = ||x-c0||^2 - ||x-c1||^2 (ties: lower token index first) and  */
/*      sends the first n/2 to child 0; each update takes the two means.     */
/*      `iters` rounds of (assign, update), then a final assign decides the  */
/*      children.  Recurse until n == leaf; leaves are numbered depth-first, */
/*      child 0 first.                                                      */
/* ------------------------------------------------------------------------ */
typedef struct {
    const double *x;
    int64_t D, leaf;
    int iters;
    int32_t *labels;
    double *cent;
    int64_t *perm;
    int64_t perm_pos;
    int32_t next_leaf;
} bisect_ctx;

static const double *g_delta;
static const int64_t *g_members;

static int cmp_delta(const void *pa, const void *pb)
{
    const int64_t a = *(const int64_t *)pa, b = *(const int64_t *)pb;
    const double da = g_delta[a], db = g_delta[b];
    if (da < db) return -1;
    if (da > db) return 1;
    const int64_t ta = g_members[a], tb = g_members[b];
    return (ta > tb) - (ta < tb);
}

static void bisect_split(const bisect_ctx *cx, const int64_t *mem, int64_t n,
                         const double *c0, const double *c1, char *side,
                         double *delta, int64_t *idx)
{
    for (int64_t i = 0; i < n; ++i) {
        const double *xi = cx->x + mem[i] * cx->D;
        delta[i] = sqdist(xi, c0, cx->D) - sqdist(xi, c1, cx->D);
        idx[i] = i;
    }
    g_delta = delta;
    g_members = mem;
    qsort(idx, (size_t)n, sizeof(int64_t), cmp_delta);
    for (int64_t r = 0; r < n; ++r) side[idx[r]] = r < n / 2 ? 0 : 1;
}

static void mean_rows(const bisect_ctx *cx, const int64_t *mem, int64_t n,
                      const char *side, int which, double *c)
{
    int64_t cnt = 0;
    for (int64_t k = 0; k < cx->D; ++k) c[k] = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        if (side && side[i] != which) continue;
        for (int64_t k = 0; k < cx->D; ++k) c[k] += cx->x[mem[i] * cx->D + k];
        ++cnt;
    }
    for (int64_t k = 0; k < cx->D; ++k) c[k] /= (double)cnt;
}

static void bisect_node(bisect_ctx *cx, const int64_t *mem, int64_t n)
{
    const int64_t D = cx->D;
    if (n <= cx->leaf) {
        const int32_t id = cx->next_leaf++;
        for (int64_t i = 0; i < n; ++i) {
            cx->labels[mem[i]] = id;
            cx->perm[cx->perm_pos++] = mem[i];
        }
        mean_rows(cx, mem, n, NULL, 0, cx->cent + (int64_t)id * D);
        return;
    }
    double *c0 = (double *)malloc((size_t)D * sizeof(double));
    double *c1 = (double *)malloc((size_t)D * sizeof(double));
    double *delta = (double *)malloc((size_t)n * sizeof(double));
    int64_t *idx = (int64_t *)malloc((size_t)n * sizeof(int64_t));
    char *side = (char *)malloc((size_t)n);
    memcpy(c0, cx->x + mem[0] * D, (size_t)D * sizeof(double));
    memcpy(c1, cx->x + mem[n / 2] * D, (size_t)D * sizeof(double));
    for (int it = 0; it < cx->iters; ++it) {
        bisect_split(cx, mem, n, c0, c1, side, delta, idx);
        mean_rows(cx, mem, n, side, 0, c0);
        mean_rows(cx, mem, n, side, 1, c1);
    }
    bisect_split(cx, mem, n, c0, c1, side, delta, idx);
    int64_t *child = (int64_t *)malloc((size_t)n * sizeof(int64_t));
    int64_t n0 = 0;
    for (int64_t i = 0; i < n; ++i)
        if (side[i] == 0) child[n0++] = mem[i];
    int64_t n1 = n0;
    for (int64_t i = 0; i < n; ++i)
        if (side[i] == 1) child[n1++] = mem[i];
    free(c0);
    free(c1);
    free(delta);
    free(idx);
    free(side);
    bisect_node(cx, child, n0);
    bisect_node(cx, child + n0, n - n0);
    free(child);
}

/* labels[N], cent[(N/leaf)*D] (leaf means), perm[N] (members leaf by leaf). */
int orc_bisect(const double *x, int64_t N, int64_t D, int64_t leaf, int iters,
               int32_t *labels, double *cent, int64_t *perm)
{
    if (leaf < 1 || N % leaf) return 1;
    for (int64_t m = N / leaf; m > 1; m >>= 1)
        if (m & 1) return 1; /* N must be leaf * 2^L */
    bisect_ctx cx = {x, D, leaf, iters, labels, cent, perm, 0, 0};
    int64_t *mem = (int64_t *)malloc((size_t)N * sizeof(int64_t));
    for (int64_t i = 0; i < N; ++i) mem[i] = i;
    bisect_node(&cx, mem, N);
    free(mem);
    return 0;
}
