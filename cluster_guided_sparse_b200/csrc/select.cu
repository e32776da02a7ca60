// Steps 3-4 of SCOPE (abstract): per-(query cluster, key) proxy scores from
// centroid-dot lookup tables, hybrid Top-p / fixed Top-k counts, the online
// per-head Top-k and the per-cluster selected-key lists.
//
// Readings: a key's proxy score for cluster c is
//   s = (LUT_t[c][a_t] + LUT_h[c][a_h]) + LUT_w[c][a_w]        (fp32, this order)
// keys are ranked by (s desc, index asc); the Top-p count is the shortest
// prefix of that order whose softmax(s/sqrt(D)) mass reaches p of the total;
// r_c = min(N, max(count, k_min)); K_h = ceil(sum_c |c| r_c / N);
// n_c = min(N, max(r_c, K_h)) for non-empty clusters (0 for empty ones);
// the list of c holds the first n_c keys of the order, ascending.
//
// A key's score depends only on its code triple (a_t, a_h, a_w), so the
// selection runs over the distinct triples of a head, each weighted by how
// many keys carry it (16 384 triples instead of 118 800 keys at 720p).  The
// Top-p cut is an exact select over the order-preserving 32-bit image of the
// score: a coarse histogram over the row's score range, then the crossing
// bucket's triples gathered and ranked (radix passes when the bucket is
// full), carrying key counts and softmax masses; masses are 64-bit fixed
// point (2^40 units) so their sums are exact and order-free.
#include "common.cuh"

namespace scope {

constexpr int kSelThreads = 512;
constexpr double kMassScale = 1099511627776.0;  // 2^40

struct SelArgs {
    const float *lut;         // [BH][Cq][Csum]
    const int32_t *codes;     // [3][BH][N]
    const int32_t *item_id;   // [BH][Pcap] distinct code triples, ascending
    const int32_t *item_cnt;  // [BH][Pcap]
    const int32_t *item_n;    // [BH]
    const uint16_t *key_item; // [BH][N] rank of each key's triple among the head's items
    int Pcap, N, Cq, Ct, Ch, Cw, BH;
    float top_p, inv_sqrt_d;
    int k_min;
    int whole_items;          // block mode: the cut takes every key tied at the cut score
    int entropy;              // EG-Sparse: topp_kernel also records each row's entropy and ln Z
    int32_t *err;             // device error word
};

// -------------------------------------------------------------- LUT
// lut[c][e] for e over (t: 0..Ct-1, h: Ct.., w: Ct+Ch..): fp64 dot of the
// query centroid's subspace slice with the key centroid, summed in dimension
// order, stored as fp32.  A CTA takes kLutQ query centroids of one head and
// walks the key centroids of each subspace in tiles of kLutRows rows, each
// tile staged in shared memory by coalesced loads (rows padded to an odd
// stride, so the row-per-lane reads are conflict-free); a thread owns one
// row and kLutQ / kLutGroups of the query centroids.
constexpr int kLutQ = 16, kLutRows = 64, kLutGroups = 4, kLutThreads = kLutRows * kLutGroups;

__global__ void __launch_bounds__(kLutThreads)
    lut_kernel(const float *qcent, const float *kc_t, const float *kc_h, const float *kc_w, float *lut, int Cq, int D,
               int dt, int dh, int dw, int Ct, int Ch, int Cw)
{
    extern __shared__ double lsm_d[];
    constexpr int QPT = kLutQ / kLutGroups;  // query centroids per thread
    const int c0 = blockIdx.x * kLutQ, bh = blockIdx.y;
    const int nq = min(kLutQ, Cq - c0);
    double *q = lsm_d;                                      // [kLutQ][D], converted once
    float *kt = reinterpret_cast<float *>(lsm_d + kLutQ * D);  // [kLutRows][stride]
    for (int i = threadIdx.x; i < kLutQ * D; i += kLutThreads)
        q[i] = i / D < nq ? (double)qcent[((int64_t)bh * Cq + c0) * D + i] : 0.0;
    const int Csum = Ct + Ch + Cw;
    const int row = threadIdx.x % kLutRows, grp = threadIdx.x / kLutRows;
    const float *segs[3] = {kc_t, kc_h, kc_w};
    const int dss[3] = {dt, dh, dw}, Cs[3] = {Ct, Ch, Cw}, offs[3] = {0, dt, dt + dh};
    int col = 0;
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        const int ds = dss[s], stride = ds | 1;
        for (int e0 = 0; e0 < Cs[s]; e0 += kLutRows) {
            const int rows = min(kLutRows, Cs[s] - e0);
            __syncthreads();  // q staged / previous tile consumed
            const float *src = segs[s] + ((int64_t)bh * Cs[s] + e0) * ds;
            for (int i = threadIdx.x; i < rows * ds; i += kLutThreads) kt[(i / ds) * stride + i % ds] = src[i];
            __syncthreads();
            if (row < rows) {
                double acc[QPT];
#pragma unroll
                for (int u = 0; u < QPT; ++u) acc[u] = 0.0;
                const float *kr = kt + row * stride;
                const double *qs = q + grp * QPT * D + offs[s];
                for (int k = 0; k < ds; ++k) {
                    const double kv = (double)kr[k];
#pragma unroll
                    for (int u = 0; u < QPT; ++u) acc[u] += qs[u * D + k] * kv;
                }
#pragma unroll
                for (int u = 0; u < QPT; ++u) {
                    const int c = grp * QPT + u;
                    if (c < nq) lut[((int64_t)bh * Cq + c0 + c) * Csum + col + e0 + row] = (float)acc[u];
                }
            }
        }
        col += Cs[s];
    }
}

// -------------------------------------------------------------- code-triple histogram
__global__ void item_hist_kernel(const int32_t *codes, int32_t *hist, int N, int BH, int Ch, int Cw, int P)
{
    const int bh = blockIdx.y;
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const int64_t plane = (int64_t)BH * N;
    const int64_t i = (int64_t)bh * N + n;
    const int id = (codes[i] * Ch + codes[plane + i]) * Cw + codes[2 * plane + i];
    atomicAdd(&hist[(int64_t)bh * P + id], 1);
}

// Ordered compaction of the non-empty triples of one head; the histogram
// entry of each non-empty triple is replaced by its item rank.
__global__ void __launch_bounds__(1024) item_compact_kernel(int32_t *hist, int32_t *item_id, int32_t *item_cnt,
                                                            int32_t *item_n, int P, int Pcap)
{
    __shared__ int tmp[33];
    const int bh = blockIdx.x;
    int32_t *h = hist + (int64_t)bh * P;
    int carry = 0;
    for (int base = 0; base < P; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int cnt = i < P ? h[i] : 0;
        int tot;
        const int ex = block_excl_scan(cnt > 0 ? 1 : 0, tmp, tot);
        if (cnt > 0) {
            item_id[(int64_t)bh * Pcap + carry + ex] = i;
            item_cnt[(int64_t)bh * Pcap + carry + ex] = cnt;
            h[i] = carry + ex;
        }
        carry += tot;
    }
    if (threadIdx.x == 0) item_n[bh] = carry;
}

// Item rank of every key (P <= 65536, so a rank fits 16 bits).
__global__ void key_item_kernel(const int32_t *codes, const int32_t *rank, uint16_t *key_item, int N, int BH, int Ch,
                                int Cw, int P)
{
    const int bh = blockIdx.y;
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const int64_t plane = (int64_t)BH * N;
    const int64_t i = (int64_t)bh * N + n;
    const int id = (codes[i] * Ch + codes[plane + i]) * Cw + codes[2 * plane + i];
    key_item[i] = (uint16_t)rank[(int64_t)bh * P + id];
}

// -------------------------------------------------------------- Top-p select
// The order of a cluster's keys is (score desc, index asc); a key's place in
// it depends only on its item's 32-bit order key u = ordered_key(score).
//
// The select runs in two stages.  Coarse: every item goes to one of kBuckets
// buckets by a monotone map of its score onto [smin, smax] of the cluster
// (so the buckets spread over the scores actually present, instead of
// crowding into the few exponent bits they share), carrying key counts and
// softmax masses; the bucket where the running metric from the top reaches
// the target is found by a scan.  Refine: a radix select on the exact order
// key (11/11/10 bits) among that bucket's items alone.  Masses are 64-bit
// fixed point (2^40 units), so every sum is exact and order-free.
//
// Items' order keys are computed once per kernel and kept in shared memory
// when the head has at most kItemCache distinct items (720p: <= 16 384).
// The Top-p kernel stores, per cluster, the score range, the coarse count
// histogram and its cut, so the list emission can skip the coarse pass and,
// when a cluster's final count equals its Top-p count, the whole select.
constexpr int kBuckets = 2048;
constexpr int kItemCache = 16384;

struct SelShared {
    unsigned long long met[kBuckets];
    int cnt[kBuckets];
    unsigned long long utmp[33];
    int itmp[33];
    float fmin[32], fmax[32];
    double dz[32], da[32];
    uint32_t prefix;
    int coarse;  // the coarse bucket being refined (-1: none)
    unsigned long long above_met, run_met, bucket_met, new_above_met;
    int above_cnt, run_cnt, bucket_cnt, new_above_cnt, bucket;
    int nlist;  // refine: items gathered from the coarse bucket
};

__device__ __forceinline__ float item_score(const float *L, int id, int Ch, int Cw, int Ct)
{
    const int a_w = id % Cw, a_h = (id / Cw) % Ch, a_t = id / (Cw * Ch);
    return (L[a_t] + L[Ct + a_h]) + L[Ct + Ch + a_w];
}

__device__ __forceinline__ float key_score(uint32_t u)
{
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

__device__ __forceinline__ unsigned long long item_mass(float s, float smax, float inv_sqrt_d)
{
    const float w = expf((s - smax) * inv_sqrt_d);
    return (unsigned long long)__double2ll_rn((double)w * kMassScale);
}

// Monotone (non-decreasing) map of a score onto the coarse buckets; the same
// fp32 operations in every kernel, so every kernel places an item alike.
struct CoarseMap {
    float smin, scale;
    __device__ __forceinline__ CoarseMap(float lo, float hi)
    {
        smin = lo;
        const float sc = hi > lo ? __fdiv_rn((float)kBuckets, __fsub_rn(hi, lo)) : 0.f;
        scale = isfinite(sc) ? sc : 0.f;
    }
    __device__ __forceinline__ int operator()(float s) const
    {
        const float t = __fmul_rn(__fsub_rn(s, smin), scale);
        return t < (float)(kBuckets - 1) ? (int)t : kBuckets - 1;
    }
};

// Per cluster, written by the Top-p kernel for the list emission.
struct ClusterCut {
    float smin, smax;
    uint32_t key;     // order key of the last key the Top-p prefix takes
    int32_t need;     // keys it takes at that key
    int32_t taken;    // the Top-p count |P_c| (-1: set by a pooled selection)
    float ent;        // entropy (nats) of the row's proxy softmax
    float lnz;        // ln of its normaliser sum_j e^{(s_j - smax) / sqrt(D)}
    int32_t pad;
};

// The order key of item i (cached, or recomputed from the table row).
struct ItemKeys {
    const uint32_t *cache;  // null when not cached
    const float *L;
    const int32_t *ids;
    int Ct, Ch, Cw;
    __device__ __forceinline__ uint32_t operator()(int i) const
    {
        return cache ? cache[i] : ordered_key(item_score(L, ids[i], Ch, Cw, Ct));
    }
};

// Scans the histogram S.met / S.cnt (nb buckets) from the top bucket down
// for the bucket where the running metric first reaches `target`, on top of
// S.above_met / S.above_cnt.  Sets S.bucket (-1 if none), S.bucket_met,
// S.bucket_cnt and moves S.above_* to the keys strictly above that bucket.
__device__ void pick_bucket(SelShared &S, int nb, unsigned long long target)
{
    if (threadIdx.x == 0) {
        S.run_met = 0ull;
        S.run_cnt = 0;
        S.bucket = -1;
    }
    __syncthreads();
    for (int top = nb - 1; top >= 0; top -= blockDim.x) {
        const int b = top - (int)threadIdx.x;
        const unsigned long long v = b >= 0 ? S.met[b] : 0ull;
        const int k = b >= 0 ? S.cnt[b] : 0;
        unsigned long long tv;
        int tk;
        const unsigned long long ev = block_excl_scan(v, S.utmp, tv);
        const int ek = block_excl_scan(k, S.itmp, tk);
        const unsigned long long before = S.above_met + S.run_met + ev;
        if (b >= 0 && v > 0ull && before < target && target <= before + v) {
            S.bucket = b;
            S.bucket_met = v;
            S.bucket_cnt = k;
            S.new_above_met = before;
            S.new_above_cnt = S.above_cnt + S.run_cnt + ek;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            S.run_met += tv;
            S.run_cnt += tk;
        }
        __syncthreads();
        if (S.bucket >= 0) break;
    }
    __syncthreads();
    if (threadIdx.x == 0 && S.bucket >= 0) {
        S.above_met = S.new_above_met;
        S.above_cnt = S.new_above_cnt;
    }
    __syncthreads();
}

// One refine pass over `width` bits below `shift + width` of the order key,
// among the items of coarse bucket S.coarse whose key matches S.prefix above.
__device__ bool refine_pass(SelShared &S, const ItemKeys &K, const int32_t *cnts, int n_items, const CoarseMap &cm,
                            float smax, float inv_sqrt_d, bool by_mass, unsigned long long target, int shift,
                            int width)
{
    const int nb = 1 << width;
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        S.met[i] = 0ull;
        S.cnt[i] = 0;
    }
    __syncthreads();
    const uint32_t pre = S.prefix;
    const int hi = shift + width, cb = S.coarse;
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const uint32_t u = K(i);
        if (hi < 32 && (u >> hi) != (pre >> hi)) continue;
        const float sc = key_score(u);
        if (cm(sc) != cb) continue;
        const int d = (int)((u >> shift) & (uint32_t)(nb - 1));
        atomicAdd(&S.cnt[d], cnts[i]);
        atomicAdd(&S.met[d], by_mass ? (unsigned long long)cnts[i] * item_mass(sc, smax, inv_sqrt_d)
                                     : (unsigned long long)cnts[i]);
    }
    __syncthreads();
    pick_bucket(S, nb, target);
    const bool ok = S.bucket >= 0;
    if (threadIdx.x == 0 && ok) S.prefix = pre | ((uint32_t)S.bucket << shift);
    __syncthreads();
    return ok;
}

// After the coarse bucket is chosen (S.coarse, S.above_*): the exact order
// key of the cut and the number of keys taken (-1 if the invariant broke,
// which exact integer metrics rule out).  The coarse bucket's items are
// gathered first (key, count, metric; at most kRefineList of them, in the
// select's bucket arrays, free by then): each gathered item then sums the
// metric and count of the gathered items with a larger key and with its own
// key, and the key where the running metric reaches the target is the cut,
// exactly as the radix passes would find it.  A fuller bucket takes three
// radix passes (11/11/10 bits of the order key) over every item instead.
constexpr int kRefineList = 1024;

__device__ int refine(SelShared &S, const ItemKeys &K, const int32_t *cnts, int n_items, const CoarseMap &cm,
                      float smax, float inv_sqrt_d, bool by_mass, unsigned long long target, uint32_t *cut_key,
                      int *need_at_cut, bool whole = false)
{
    static_assert(kBuckets >= 2 * kRefineList, "the gathered items live in the bucket arrays");
    unsigned long long *lw = S.met;                                         // metric
    uint32_t *lk = reinterpret_cast<uint32_t *>(S.met + kRefineList);      // order key
    int *lc = S.cnt;                                                        // key count
    if (threadIdx.x == 0) {
        S.nlist = 0;
        S.bucket = -1;
        S.prefix = 0u;
    }
    __syncthreads();
    const int cb = S.coarse;
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const uint32_t u = K(i);
        const float sc = key_score(u);
        if (cm(sc) != cb) continue;
        const int slot = atomicAdd(&S.nlist, 1);
        if (slot < kRefineList) {
            lk[slot] = u;
            lc[slot] = cnts[i];
            lw[slot] = by_mass ? (unsigned long long)cnts[i] * item_mass(sc, smax, inv_sqrt_d)
                               : (unsigned long long)cnts[i];
        }
    }
    __syncthreads();
    const int m = S.nlist;
    if (m <= kRefineList) {
        for (int p = threadIdx.x; p < m; p += blockDim.x) {
            const uint32_t u = lk[p];
            unsigned long long wg = 0ull, we = 0ull;
            int cg = 0, ce = 0;
            for (int q = 0; q < m; ++q) {
                const uint32_t v = lk[q];
                if (v > u) {
                    wg += lw[q];
                    cg += lc[q];
                } else if (v == u) {
                    we += lw[q];
                    ce += lc[q];
                }
            }
            const unsigned long long before = S.above_met + wg;
            if (before < target && target <= before + we) {  // every item of the cut key writes the same
                S.bucket = 0;
                S.prefix = u;
                S.bucket_met = we;
                S.bucket_cnt = ce;
                S.new_above_met = before;
                S.new_above_cnt = S.above_cnt + cg;
            }
        }
        __syncthreads();
        if (S.bucket < 0) return -1;
        if (threadIdx.x == 0) {
            S.above_met = S.new_above_met;
            S.above_cnt = S.new_above_cnt;
        }
        __syncthreads();
    } else {
        if (!refine_pass(S, K, cnts, n_items, cm, smax, inv_sqrt_d, by_mass, target, 21, 11)) return -1;
        if (!refine_pass(S, K, cnts, n_items, cm, smax, inv_sqrt_d, by_mass, target, 10, 11)) return -1;
        if (!refine_pass(S, K, cnts, n_items, cm, smax, inv_sqrt_d, by_mass, target, 0, 10)) return -1;
    }
    // every key in the final bucket has the same score, hence the same metric
    const unsigned long long per = S.bucket_met / (unsigned long long)S.bucket_cnt;
    const unsigned long long rest = target - S.above_met;
    const int need = whole ? S.bucket_cnt : (int)((rest + per - 1) / per);
    *cut_key = S.prefix;
    *need_at_cut = need;
    return S.above_cnt + need;
}

// Order keys of the head's items (into the cache when there is one) and the
// block's score range.
__device__ void item_keys_and_range(SelShared &S, const float *L, const int32_t *ids, int n_items, uint32_t *cache,
                                    int Ct, int Ch, int Cw, float *smin, float *smax)
{
    float lo = INFINITY, hi = -INFINITY;
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const float sc = item_score(L, ids[i], Ch, Cw, Ct);
        if (cache) cache[i] = ordered_key(sc);
        lo = fminf(lo, sc);
        hi = fmaxf(hi, sc);
    }
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if ((threadIdx.x & 31) == 0) {
        S.fmin[threadIdx.x >> 5] = lo;
        S.fmax[threadIdx.x >> 5] = hi;
    }
    __syncthreads();
    lo = INFINITY;
    hi = -INFINITY;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
        lo = fminf(lo, S.fmin[w]);
        hi = fmaxf(hi, S.fmax[w]);
    }
    *smin = lo;
    *smax = hi;
    __syncthreads();
}

// -------------------------------------------------------------- Top-p counts
__global__ void __launch_bounds__(kSelThreads) topp_kernel(SelArgs a, int32_t *r_out, ClusterCut *cuts,
                                                           int32_t *coarse_hist)
{
    extern __shared__ __align__(16) float L[];
    __shared__ SelShared S;
    const int c = blockIdx.x, bh = blockIdx.y;
    const int64_t bhc = (int64_t)bh * a.Cq + c;
    const int Csum = a.Ct + a.Ch + a.Cw;
    uint32_t *cache = reinterpret_cast<uint32_t *>(L + ((Csum + 3) & ~3));
    const float *lrow = a.lut + bhc * Csum;
    for (int e = threadIdx.x; e < Csum; e += blockDim.x) L[e] = lrow[e];
    __syncthreads();
    const int n_items = a.item_n[bh];
    const int32_t *ids = a.item_id + (int64_t)bh * a.Pcap;
    const int32_t *cnts = a.item_cnt + (int64_t)bh * a.Pcap;
    if (n_items > kItemCache) cache = nullptr;
    float smin, smax;
    item_keys_and_range(S, L, ids, n_items, cache, a.Ct, a.Ch, a.Cw, &smin, &smax);
    const ItemKeys K{cache, L, ids, a.Ct, a.Ch, a.Cw};
    const CoarseMap cm(smin, smax);
    int m = a.N;
    uint32_t key = 0u;
    int need = 0;
    // coarse histogram by count and by mass, over every item
    for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) {
        S.met[i] = 0ull;
        S.cnt[i] = 0;
    }
    __syncthreads();
    const bool sel = a.top_p < 1.0f;
    unsigned long long wsum = 0ull;
    double zs = 0.0, as = 0.0;  // sum cnt e^x and sum cnt e^x x, x = (s - smax) / sqrt(D): the row entropy
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const float sc = key_score(K(i));
        const int b = cm(sc);
        atomicAdd(&S.cnt[b], cnts[i]);
        if (sel) {
            const unsigned long long w = (unsigned long long)cnts[i] * item_mass(sc, smax, a.inv_sqrt_d);
            atomicAdd(&S.met[b], w);
            wsum += w;
            if (a.entropy) {
                const float x = (sc - smax) * a.inv_sqrt_d;
                const double e = (double)cnts[i] * (double)expf(x);
                zs += e;
                as += e * (double)x;
            }
        }
    }
    for (int o = 16; o > 0; o >>= 1) {
        zs += __shfl_xor_sync(0xffffffffu, zs, o);
        as += __shfl_xor_sync(0xffffffffu, as, o);
    }
    if ((threadIdx.x & 31) == 0) {
        S.dz[threadIdx.x >> 5] = zs;
        S.da[threadIdx.x >> 5] = as;
    }
    __syncthreads();
    int32_t *hist_out = coarse_hist + bhc * kBuckets;
    for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) hist_out[i] = S.cnt[i];
    if (sel) {
        unsigned long long Wt;
        block_excl_scan(wsum, S.utmp, Wt);
        unsigned long long target = (unsigned long long)ceil((double)a.top_p * (double)Wt);
        if (target < 1ull) target = 1ull;
        if (target > Wt) target = Wt;
        if (threadIdx.x == 0) {
            S.above_met = 0ull;
            S.above_cnt = 0;
        }
        __syncthreads();
        pick_bucket(S, kBuckets, target);
        if (threadIdx.x == 0) S.coarse = S.bucket;
        __syncthreads();
        m = S.coarse >= 0 ? refine(S, K, cnts, n_items, cm, smax, a.inv_sqrt_d, true, target, &key, &need,
                                   a.whole_items != 0)
                          : -1;
        if (m < 0) {
            if (threadIdx.x == 0) set_error(a.err, kErrRange, 0x100 + c);
            m = a.N;
        }
    }
    if (threadIdx.x == 0) {
        int r = m > a.k_min ? m : a.k_min;
        r = r < a.N ? r : a.N;
        r_out[bhc] = r;
        ClusterCut cut;
        cut.smin = smin;
        cut.smax = smax;
        cut.key = key;
        cut.need = need;
        cut.taken = sel ? m : a.N;
        double Z = 0.0, A = 0.0;  // fixed combination order: deterministic
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            Z += S.dz[w];
            A += S.da[w];
        }
        cut.lnz = a.entropy && sel && Z > 0.0 ? (float)log(Z) : 0.f;
        cut.ent = a.entropy && sel && Z > 0.0 ? (float)(log(Z) - A / Z) : 0.f;
        cut.pad = 0;
        cuts[bhc] = cut;
    }
}

// -------------------------------------------------------------- EG-Sparse
// "EG-Sparse" (abstract): low-entropy heads are routed to a grouped
// cross-head pool, high-entropy heads keep per-row selection, using only
// scores the sparse pipeline already has.  Reading: a head's entropy is the
// query-weighted mean of its rows' proxy-softmax entropies over ln N; heads
// below eg_tau are grouped eg_group at a time (per batch entry) and a group's
// low-entropy heads form one pool, in which every (head, cluster, key) entry
// competes by ln pi = (s - smax) / sqrt(D) - ln Z of its row and carries mass
// |c| pi; the shortest prefix reaching top_p of the pool's mass is kept (ties:
// head, then cluster, then the row's own key order), and a row's Top-p count
// is its number of kept entries.  Clusters without queries stay out of the
// pool and keep their own count.
//
// The pooled select mirrors the per-row one across CTAs: coarse buckets of
// ln pi over [-kLambdaSpan, 0] (entries below share bucket 0), then a radix
// refine on the exact fp32 order key of ln pi, each pass a histogram that the
// clusters' CTAs add into the pool's buffer and one CTA per pool reads.  Pool
// masses are 64-bit fixed point in 2^-32 units (a pool of 64 heads of 2^24
// queries stays below 2^63).
constexpr float kLambdaSpan = 64.f;
constexpr double kPoolMassScale = 4294967296.0;  // 2^32

struct PoolSel {
    unsigned long long met[kBuckets];  // histogram of the pass in progress
    int cnt[kBuckets];
    unsigned long long target;         // ceil(top_p * pool mass)
    unsigned long long above_met;      // mass strictly above the chosen range
    uint32_t prefix;                   // order-key bits fixed so far
    int coarse;                        // chosen coarse bucket (-1: none)
    int ok;
    int pad;
};

__device__ __forceinline__ int lambda_bucket(float lam)
{
    const float t = __fmul_rn(__fadd_rn(lam, kLambdaSpan), (float)kBuckets / kLambdaSpan);
    return t <= 0.f ? 0 : (t < (float)(kBuckets - 1) ? (int)t : kBuckets - 1);
}

// ln pi of an item of row (c, bh): the same fp32 operations in every pass
__device__ __forceinline__ float item_lambda(float sc, const ClusterCut &cut, float inv_sqrt_d)
{
    return __fsub_rn((sc - cut.smax) * inv_sqrt_d, cut.lnz);
}

// Head entropies and routing, one CTA per batch entry, one warp per head.
__global__ void __launch_bounds__(1024) eg_route_kernel(const ClusterCut *cuts, const int32_t *sizes, float *entropy,
                                                        int32_t *pool, int H, int Cq, int N, float tau, int group)
{
    const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ngroups = (H + group - 1) / group;
    for (int h = warp; h < H; h += blockDim.x >> 5) {
        const int64_t bh = (int64_t)b * H + h;
        double num = 0.0, den = 0.0;
        for (int c = lane; c < Cq; c += 32) {
            const int z = sizes[bh * Cq + c];
            num += (double)z * (double)cuts[bh * Cq + c].ent;
            den += (double)z;
        }
        for (int o = 16; o > 0; o >>= 1) {
            num += __shfl_xor_sync(0xffffffffu, num, o);
            den += __shfl_xor_sync(0xffffffffu, den, o);
        }
        if (lane == 0) {
            const float e = den > 0.0 && N > 1 ? (float)(num / (den * log((double)N))) : 0.f;
            entropy[bh] = e;
            pool[bh] = e < tau ? b * ngroups + h / group : -1;
        }
    }
}

// One pass over the items of one pooled cluster: the coarse histogram
// (pass < 0) or the refine digit [shift, shift + width) among the chosen
// range, added into the pool's histogram.
__global__ void __launch_bounds__(kSelThreads) eg_hist_kernel(SelArgs a, const ClusterCut *cuts,
                                                              const int32_t *sizes, const int32_t *pool,
                                                              PoolSel *pools, int shift, int width)
{
    extern __shared__ __align__(16) float L[];
    __shared__ unsigned long long hmet[kBuckets];
    __shared__ int hcnt[kBuckets];
    const int c = blockIdx.x, bh = blockIdx.y;
    const int64_t bhc = (int64_t)bh * a.Cq + c;
    const int pid = pool[bh];
    const int sz = sizes[bhc];
    if (pid < 0 || sz <= 0) return;
    PoolSel &P = pools[pid];
    const bool coarse = shift < 0;
    if (!coarse && (P.coarse < 0 || !P.ok)) return;
    const int Csum = a.Ct + a.Ch + a.Cw;
    const float *lrow = a.lut + bhc * Csum;
    for (int e = threadIdx.x; e < Csum; e += blockDim.x) L[e] = lrow[e];
    const int nb = coarse ? kBuckets : 1 << width;
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        hmet[i] = 0ull;
        hcnt[i] = 0;
    }
    __syncthreads();
    const ClusterCut cut = cuts[bhc];
    const int n_items = a.item_n[bh];
    const int32_t *ids = a.item_id + (int64_t)bh * a.Pcap;
    const int32_t *cnts = a.item_cnt + (int64_t)bh * a.Pcap;
    const int hi = shift + width;
    const uint32_t pre = P.prefix;
    const int cb = P.coarse;
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const float lam = item_lambda(item_score(L, ids[i], a.Ch, a.Cw, a.Ct), cut, a.inv_sqrt_d);
        const int lb = lambda_bucket(lam);
        int d;
        if (coarse) {
            d = lb;
        } else {
            const uint32_t u = ordered_key(lam);
            if (lb != cb || (hi < 32 && (u >> hi) != (pre >> hi))) continue;
            d = (int)((u >> shift) & (uint32_t)(nb - 1));
        }
        const unsigned long long m =
            (unsigned long long)sz * (unsigned long long)llrint((double)cnts[i] * (double)expf(lam) * kPoolMassScale);
        atomicAdd(&hcnt[d], cnts[i]);
        atomicAdd(&hmet[d], m);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nb; i += blockDim.x)
        if (hcnt[i]) {
            atomicAdd(&P.cnt[i], hcnt[i]);
            atomicAdd(&P.met[i], hmet[i]);
        }
}

// One CTA per pool: reads the pass's histogram (and clears it for the next
// pass), then picks the bucket where the pool's running mass reaches the
// target; the coarse pass (shift < 0) first sets the target.
__global__ void __launch_bounds__(kSelThreads) eg_pick_kernel(PoolSel *pools, float top_p, int shift, int width,
                                                              int32_t *err)
{
    __shared__ SelShared S;
    PoolSel &P = pools[blockIdx.x];
    const bool coarse = shift < 0;
    if (!coarse && (P.coarse < 0 || !P.ok)) return;
    const int nb = coarse ? kBuckets : 1 << width;
    unsigned long long w = 0ull;
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        S.met[i] = P.met[i];
        S.cnt[i] = P.cnt[i];
        w += S.met[i];
        P.met[i] = 0ull;
        P.cnt[i] = 0;
    }
    unsigned long long W;
    block_excl_scan(w, S.utmp, W);
    if (coarse) {
        if (W == 0ull) {  // no pooled rows in this group
            if (threadIdx.x == 0) {
                P.coarse = -1;
                P.ok = 1;
            }
            return;
        }
        unsigned long long t = (unsigned long long)ceil((double)top_p * (double)W);
        t = t < 1ull ? 1ull : (t > W ? W : t);
        if (threadIdx.x == 0) {
            P.target = t;
            P.above_met = 0ull;
            P.prefix = 0u;
        }
    }
    if (threadIdx.x == 0) {
        S.above_met = P.above_met;
        S.above_cnt = 0;
    }
    __syncthreads();
    pick_bucket(S, nb, P.target);
    if (threadIdx.x == 0) {
        if (S.bucket < 0) {
            P.ok = 0;
            P.coarse = -1;
            set_error(err, kErrRange, 0x400 + (int)blockIdx.x);
        } else {
            P.ok = 1;
            P.above_met = S.above_met;
            if (coarse) P.coarse = S.bucket;
            else P.prefix |= (uint32_t)S.bucket << shift;
        }
    }
}

// Keys of every pooled cluster above and at the pool's cut (order key of ln pi).
__global__ void __launch_bounds__(kSelThreads) eg_count_kernel(SelArgs a, const ClusterCut *cuts,
                                                               const int32_t *sizes, const int32_t *pool,
                                                               const PoolSel *pools, int2 *above_at)
{
    extern __shared__ __align__(16) float L[];
    __shared__ int tmp[33];
    const int c = blockIdx.x, bh = blockIdx.y;
    const int64_t bhc = (int64_t)bh * a.Cq + c;
    const int pid = pool[bh];
    if (pid < 0 || sizes[bhc] <= 0) return;
    const PoolSel &P = pools[pid];
    if (P.coarse < 0 || !P.ok) return;
    const int Csum = a.Ct + a.Ch + a.Cw;
    const float *lrow = a.lut + bhc * Csum;
    for (int e = threadIdx.x; e < Csum; e += blockDim.x) L[e] = lrow[e];
    __syncthreads();
    const ClusterCut cut = cuts[bhc];
    const uint32_t key = P.prefix;
    const int n_items = a.item_n[bh];
    const int32_t *ids = a.item_id + (int64_t)bh * a.Pcap;
    const int32_t *cnts = a.item_cnt + (int64_t)bh * a.Pcap;
    int above = 0, at = 0;
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const uint32_t u = ordered_key(item_lambda(item_score(L, ids[i], a.Ch, a.Cw, a.Ct), cut, a.inv_sqrt_d));
        above += u > key ? cnts[i] : 0;
        at += u == key ? cnts[i] : 0;
    }
    int ta, tt;
    block_excl_scan(above, tmp, ta);
    block_excl_scan(at, tmp, tt);
    if (threadIdx.x == 0) above_at[bhc] = make_int2(ta, tt);
}

// One CTA per pool: the keys at the cut go to the pool's rows in (head,
// cluster) order until the mass target is met; every pooled row's Top-p count
// becomes (keys above) + (its keys taken at the cut), then the hybrid rule.
__global__ void __launch_bounds__(1024) eg_assign_kernel(const PoolSel *pools, const int32_t *sizes,
                                                         const int32_t *pool, const int2 *above_at, int32_t *r_out,
                                                         ClusterCut *cuts, int H, int group, int Cq, int N, int k_min)
{
    __shared__ unsigned long long utmp[33];
    __shared__ unsigned long long carry_sh;
    const int pid = blockIdx.x;
    const PoolSel &P = pools[pid];
    if (P.coarse < 0 || !P.ok) return;
    const int ngroups = (H + group - 1) / group;
    const int b = pid / ngroups, g = pid % ngroups;
    const int h0 = g * group, h1 = min(H, h0 + group);
    const unsigned long long rest = P.target - P.above_met;  // > 0: mass still needed at the cut
    const unsigned long long per_key = (unsigned long long)llrint((double)expf(key_score(P.prefix)) * kPoolMassScale);
    if (threadIdx.x == 0) carry_sh = 0ull;
    __syncthreads();
    for (int h = h0; h < h1; ++h) {
        const int64_t bh = (int64_t)b * H + h;
        if (pool[bh] != pid) continue;
        for (int c0 = 0; c0 < Cq; c0 += blockDim.x) {
            const int c = c0 + threadIdx.x;
            const int64_t bhc = bh * Cq + c;
            const bool in = c < Cq && sizes[bhc] > 0;
            const int2 aa = in ? above_at[bhc] : make_int2(0, 0);
            const unsigned long long unit = in ? (unsigned long long)sizes[bhc] * per_key : 0ull;
            const unsigned long long v = unit * (unsigned long long)aa.y;
            unsigned long long tot;
            const unsigned long long ex = block_excl_scan(v, utmp, tot);
            const unsigned long long before = carry_sh + ex;
            if (in) {
                int take;
                if (before >= rest) take = 0;
                else if (before + v <= rest || unit == 0ull) take = aa.y;
                else take = (int)min((unsigned long long)aa.y, (rest - before + unit - 1) / unit);
                int r = aa.x + take;
                r = r > k_min ? r : k_min;
                r = r < N ? r : N;
                r_out[bhc] = r;
                cuts[bhc].taken = -1;  // the list emission selects by count
            }
            __syncthreads();
            if (threadIdx.x == 0) carry_sh += tot;
            __syncthreads();
        }
    }
}

// -------------------------------------------------------------- online Top-k + offsets
__global__ void __launch_bounds__(1024) topk_kernel(const int32_t *sizes, const int32_t *r, int32_t *n_out,
                                                    int32_t *kh_out, long long *offsets, int BH, int Cq, int N,
                                                    int online)
{
    __shared__ long long ltmp[33];
    long long carry = 0;
    for (int bh = 0; bh < BH; ++bh) {
        long long num = 0;
        for (int c = threadIdx.x; c < Cq; c += blockDim.x)
            num += (long long)sizes[(int64_t)bh * Cq + c] * r[(int64_t)bh * Cq + c];
        long long tot;
        block_excl_scan(num, ltmp, tot);
        const long long K = online ? (tot + N - 1) / N : 0;
        if (threadIdx.x == 0) kh_out[bh] = (int32_t)K;
        for (int base = 0; base < Cq; base += blockDim.x) {
            const int c = base + threadIdx.x;
            long long v = 0;
            if (c < Cq) {
                const int64_t i = (int64_t)bh * Cq + c;
                long long x = r[i];
                if (x < K) x = K;
                if (x > N) x = N;
                v = sizes[i] > 0 ? x : 0;
                n_out[i] = (int32_t)v;
            }
            long long t2;
            const long long ex = block_excl_scan(v, ltmp, t2);
            if (c < Cq) offsets[(int64_t)bh * Cq + c] = carry + ex;
            carry += t2;
        }
    }
    if (threadIdx.x == 0) offsets[(int64_t)BH * Cq] = carry;
}

// -------------------------------------------------------------- list emission
// The first n_c keys of the (score desc, index asc) order: every key strictly
// above the cut, then the lowest-index `need` keys at the cut.  When n_c is
// the cluster's Top-p count the cut is the Top-p kernel's; otherwise a count
// select runs from that kernel's coarse histogram.  Written in ascending key
// order: the output slot of key j is
// (#keys above the cut before j) + min(#keys at the cut before j, need).
// A key's side of the cut is its item's: each key costs one 16-bit load of its
// item rank and one shared-memory lookup (the item's order key, or a class
// byte when the keys are not cached).

__global__ void __launch_bounds__(kSelThreads) emit_kernel(SelArgs a, const int32_t *n_in, const long long *offsets,
                                                           const ClusterCut *cuts, const int32_t *coarse_hist,
                                                           int32_t *indices)
{
    extern __shared__ __align__(16) float L[];
    __shared__ SelShared S;
    const int c = blockIdx.x, bh = blockIdx.y;
    const int64_t bhc = (int64_t)bh * a.Cq + c;
    const int n = n_in[bhc];
    if (n == 0) return;
    int32_t *out = indices + offsets[bhc];
    if (n >= a.N) {
        for (int j = threadIdx.x; j < a.N; j += blockDim.x) out[j] = j;
        return;
    }
    const int Csum = a.Ct + a.Ch + a.Cw;
    unsigned char *region = reinterpret_cast<unsigned char *>(L + ((Csum + 3) & ~3));  // 64 KB
    const float *lrow = a.lut + bhc * Csum;
    for (int e = threadIdx.x; e < Csum; e += blockDim.x) L[e] = lrow[e];
    __syncthreads();
    const int n_items = a.item_n[bh];
    const int32_t *ids = a.item_id + (int64_t)bh * a.Pcap;
    const int32_t *cnts = a.item_cnt + (int64_t)bh * a.Pcap;
    const bool cached = n_items <= kItemCache;
    uint32_t *cache = cached ? reinterpret_cast<uint32_t *>(region) : nullptr;
    if (cached)
        for (int i = threadIdx.x; i < n_items; i += blockDim.x)
            cache[i] = ordered_key(item_score(L, ids[i], a.Ch, a.Cw, a.Ct));
    __syncthreads();
    const ItemKeys K{cache, L, ids, a.Ct, a.Ch, a.Cw};
    const ClusterCut cut = cuts[bhc];
    uint32_t key = cut.key;
    int need = cut.need;
    if (n != cut.taken) {
        // count select for n: coarse bucket from the stored histogram, then refine
        const int32_t *hist = coarse_hist + bhc * kBuckets;
        for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) {
            const int k = hist[i];
            S.cnt[i] = k;
            S.met[i] = (unsigned long long)k;
        }
        if (threadIdx.x == 0) {
            S.above_met = 0ull;
            S.above_cnt = 0;
        }
        __syncthreads();
        pick_bucket(S, kBuckets, (unsigned long long)n);
        if (threadIdx.x == 0) S.coarse = S.bucket;
        __syncthreads();
        const CoarseMap cm(cut.smin, cut.smax);
        if (S.coarse < 0 ||
            refine(S, K, cnts, n_items, cm, cut.smax, a.inv_sqrt_d, false, (unsigned long long)n, &key, &need) < 0) {
            if (threadIdx.x == 0) set_error(a.err, kErrRange, 0x200 + c);
            return;
        }
    }
    // every item's class once: 2 above the cut, 1 at it, 0 below (a byte per
    // item after the 64 KB region; without cached keys, in the region itself)
    uint8_t *cls = cached ? region + (size_t)kItemCache * 4 : region;
    __syncthreads();  // the refine above may still read the cached keys
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const uint32_t u = K(i);
        cls[i] = u > key ? 2 : (u == key ? 1 : 0);
    }
    __syncthreads();
    // Key walk without block-wide scans: warp w owns a contiguous chunk of the
    // keys (a multiple of 256).  Each lane takes eight adjacent keys per step
    // (one 16-byte load of their item ranks), gathers their class bytes into
    // two words and turns them into 8-bit masks of keys above and at the cut
    // (one multiply packs four bytes' low bits), so counting is two popcounts.
    // Pass 1 counts the chunk; after one barrier every warp knows its chunk's
    // output base, and pass 2 walks the chunk again, placing each lane's
    // selected keys (those above the cut, and those at it while fewer than
    // `need` came before) after an exclusive warp scan of the lanes' counts.
    const uint16_t *ki = a.key_item + (int64_t)bh * a.N;
    const bool vec8 = (((int64_t)bh * a.N) & 7) == 0;  // 16-byte aligned runs of eight ranks
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int chunk = (((a.N + nwarps - 1) / nwarps) + 255) & ~255;
    const int j_begin = min(a.N, warp * chunk), j_end = min(a.N, j_begin + chunk);
    __shared__ int wgt[32], weq[32];
    // bit b of the result = bit `sh` of byte b of x (b < 4)
    auto pack4 = [](uint32_t x, int sh) { return (((x >> sh) & 0x01010101u) * 0x01020408u) >> 24 & 0xfu; };
    // masks of keys j .. j+7 above (bits of *ab) and at (*at) the cut; keys past the chunk are below
    auto masks8 = [&](int j, uint32_t &ab, uint32_t &at) {
        uint32_t lo, hi;
        if (vec8 && j + 8 <= j_end) {
            const uint4 w = *reinterpret_cast<const uint4 *>(ki + j);
            lo = (uint32_t)cls[w.x & 0xffffu] | (uint32_t)cls[w.x >> 16] << 8 | (uint32_t)cls[w.y & 0xffffu] << 16 |
                 (uint32_t)cls[w.y >> 16] << 24;
            hi = (uint32_t)cls[w.z & 0xffffu] | (uint32_t)cls[w.z >> 16] << 8 | (uint32_t)cls[w.w & 0xffffu] << 16 |
                 (uint32_t)cls[w.w >> 16] << 24;
        } else {
            lo = hi = 0u;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                if (j + t < j_end) lo |= (uint32_t)cls[ki[j + t]] << (8 * t);
                if (j + 4 + t < j_end) hi |= (uint32_t)cls[ki[j + 4 + t]] << (8 * t);
            }
        }
        ab = pack4(lo, 1) | pack4(hi, 1) << 4;
        at = pack4(lo, 0) | pack4(hi, 0) << 4;
    };
    int g_cnt = 0, e_cnt = 0;
    for (int j0 = j_begin; j0 < j_end; j0 += 256) {
        uint32_t ab, at;
        masks8(j0 + 8 * lane, ab, at);
        g_cnt += __popc(ab);
        e_cnt += __popc(at);
    }
    for (int o = 16; o > 0; o >>= 1) {
        g_cnt += __shfl_xor_sync(0xffffffffu, g_cnt, o);
        e_cnt += __shfl_xor_sync(0xffffffffu, e_cnt, o);
    }
    if (lane == 0) {
        wgt[warp] = g_cnt;
        weq[warp] = e_cnt;
    }
    __syncthreads();
    unsigned g = 0, e = 0;  // keys above / at the cut before this warp's chunk
    for (int w = 0; w < warp; ++w) {
        g += wgt[w];
        e += weq[w];
    }
    // staging rows (256 keys per warp step) in the select's bucket array,
    // which the count select above no longer needs
    int *stage = reinterpret_cast<int *>(S.met) + warp * 256;
    for (int j0 = j_begin; j0 < j_end; j0 += 256) {
        const int j = j0 + 8 * lane;
        uint32_t ab, at;
        masks8(j, ab, at);
        const unsigned lg = __popc(ab), le = __popc(at);
        // exclusive scan of the lanes' (above, at) counts, packed in one word
        const unsigned packed = lg | (le << 16);
        unsigned incl = packed;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const unsigned tot = __shfl_sync(0xffffffffu, incl, 31);
        const unsigned ex = incl - packed;
        // output slot of a selected key = selected keys before it
        const unsigned base = g + min(e, (unsigned)need);  // selected keys before this step
        const unsigned gl = g + (ex & 0xffffu), el = e + (ex >> 16);
        uint32_t sel = ab;
        if (el < (unsigned)need) {
            if (el + le <= (unsigned)need) {
                sel |= at;
            } else {  // the lane where the keys at the cut run out
                uint32_t m = at;
                for (unsigned k = el; k < (unsigned)need; ++k) {
                    sel |= m & (0u - m);
                    m &= m - 1u;
                }
            }
        }
        unsigned pos = gl + min(el, (unsigned)need) - base;
        while (sel) {
            const int t = __ffs(sel) - 1;
            sel &= sel - 1u;
            stage[pos++] = j + t;
        }
        g += tot & 0xffffu;
        e += tot >> 16;
        const unsigned step_sel = g + min(e, (unsigned)need) - base;
        __syncwarp();
        for (unsigned i = lane; i < step_sel; i += 32) {
            if (base + i < (unsigned)n) out[base + i] = stage[i];
            else set_error(a.err, kErrRange, 0x300 + c);
        }
        __syncwarp();
    }
}

// dynamic shared memory of topp_kernel and emit_kernel: the table row and a
// 64 KB region (cached order keys, or item class bytes)
static size_t sel_smem(int Csum) { return (size_t)((Csum + 3) & ~3) * sizeof(float) + (size_t)kItemCache * 4; }
// emit_kernel also keeps a class byte per item after the region
static size_t emit_smem(int Csum) { return sel_smem(Csum) + (size_t)kItemCache; }

cudaError_t select_configure()
{
    static_assert(kItemCache * 4 >= kMaxItems, "the 64 KB region must hold a class byte per item");
    static_assert(kBuckets * 2 >= (kSelThreads / 32) * 256, "emit stages 256 keys per warp in SelShared::met");
    // the table kernel's staging at D = 128: fp64 query centroids + one padded key tile
    cudaError_t el = cudaFuncSetAttribute(lut_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)(kLutQ * 128 * sizeof(double) + kLutRows * 129 * sizeof(float)));
    if (el != cudaSuccess) return el;
    const int max_csum = kMaxBlocks + 2 > 3 * kMaxClusters ? kMaxBlocks + 2 : 3 * kMaxClusters;
    cudaError_t e = cudaFuncSetAttribute(emit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)emit_smem(max_csum));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(eg_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(3 * kMaxClusters * sizeof(float)));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(eg_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(3 * kMaxClusters * sizeof(float)));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(topp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem(max_csum));
}

// -------------------------------------------------------------- launchers
void launch_lut(const float *qcent, const float *kc_t, const float *kc_h, const float *kc_w, float *lut, int BH,
                int Cq, int D, int dt, int dh, int dw, int Ct, int Ch, int Cw, cudaStream_t st)
{
    const int dmax = max(dt, max(dh, dw));
    const size_t smem = (size_t)kLutQ * D * sizeof(double) + (size_t)kLutRows * (dmax | 1) * sizeof(float);
    lut_kernel<<<dim3((Cq + kLutQ - 1) / kLutQ, BH), kLutThreads, smem, st>>>(qcent, kc_t, kc_h, kc_w, lut, Cq, D, dt,
                                                                             dh, dw, Ct, Ch, Cw);
    count_launches(1);
}

void launch_items(const int32_t *codes, int32_t *hist, int32_t *item_id, int32_t *item_cnt, int32_t *item_n,
                  uint16_t *key_item, int BH, int N, int Ch, int Cw, int P, int Pcap, cudaStream_t st)
{
    cudaMemsetAsync(hist, 0, (size_t)BH * P * sizeof(int32_t), st);
    item_hist_kernel<<<dim3((N + 255) / 256, BH), 256, 0, st>>>(codes, hist, N, BH, Ch, Cw, P);
    count_launches(1);
    item_compact_kernel<<<BH, 1024, 0, st>>>(hist, item_id, item_cnt, item_n, P, Pcap);
    count_launches(1);
    key_item_kernel<<<dim3((N + 255) / 256, BH), 256, 0, st>>>(codes, hist, key_item, N, BH, Ch, Cw, P);
    count_launches(1);
}

void launch_topp(const SelArgs &a, int32_t *r_out, ClusterCut *cuts, int32_t *coarse_hist, cudaStream_t st)
{
    topp_kernel<<<dim3(a.Cq, a.BH), kSelThreads, sel_smem(a.Ct + a.Ch + a.Cw), st>>>(a, r_out, cuts, coarse_hist);
    count_launches(1);
}

void launch_topk(const int32_t *sizes, const int32_t *r, int32_t *n_out, int32_t *kh, long long *offsets, int BH,
                 int Cq, int N, int online, cudaStream_t st)
{
    topk_kernel<<<1, 1024, 0, st>>>(sizes, r, n_out, kh, offsets, BH, Cq, N, online);
    count_launches(1);
}

void launch_emit(const SelArgs &a, const int32_t *n_in, const long long *offsets, const ClusterCut *cuts,
                 const int32_t *coarse_hist, int32_t *indices, cudaStream_t st)
{
    emit_kernel<<<dim3(a.Cq, a.BH), kSelThreads, emit_smem(a.Ct + a.Ch + a.Cw), st>>>(a, n_in, offsets, cuts,
                                                                                  coarse_hist, indices);
    count_launches(1);
}

// Bytes of per-cluster selection state (cut record + coarse histogram) and,
// with EG-Sparse routing, of the head entropies, pool ids, per-cluster cut
// counts and per-pool histograms.
size_t selection_state_bytes(int64_t clusters) { return (size_t)clusters * (sizeof(ClusterCut) + kBuckets * 4); }
size_t eg_state_bytes(int64_t B, int64_t H, int64_t Cq, int group)
{
    const int64_t pools = B * ((H + group - 1) / group);
    return (size_t)(B * H * 8 + B * H * Cq * 8 + 256) + (size_t)pools * sizeof(PoolSel);
}

void run_selection(const float *lut, const int32_t *codes, const int32_t *item_id, const int32_t *item_cnt,
                   const int32_t *item_n, const uint16_t *key_item, int Pcap, int N, int Cq, int Ct, int Ch,
                   int Cw, int BH, float top_p, float inv_sqrt_d, int k_min, int32_t *err, const int32_t *sizes,
                   int32_t *r, int32_t *n, int32_t *kh, long long *offsets, int32_t *indices, int online,
                   void *state, int B, float eg_tau, int eg_group, void *eg_state, int whole_items, cudaStream_t st)
{
    SelArgs a;
    a.lut = lut;
    a.codes = codes;
    a.item_id = item_id;
    a.item_cnt = item_cnt;
    a.item_n = item_n;
    a.key_item = key_item;
    a.Pcap = Pcap;
    a.N = N;
    a.Cq = Cq;
    a.Ct = Ct;
    a.Ch = Ch;
    a.Cw = Cw;
    a.BH = BH;
    a.top_p = top_p;
    a.inv_sqrt_d = inv_sqrt_d;
    a.k_min = k_min;
    a.whole_items = whole_items;
    a.entropy = (eg_tau > 0.f && top_p < 1.0f) ? 1 : 0;
    a.err = err;
    ClusterCut *cuts = reinterpret_cast<ClusterCut *>(state);
    int32_t *coarse_hist = reinterpret_cast<int32_t *>(cuts + (int64_t)BH * Cq);
    launch_topp(a, r, cuts, coarse_hist, st);
    if (eg_tau > 0.f && top_p < 1.0f) {
        // EG-Sparse: entropies, routing, then the pooled Top-p of every group
        const int H = BH / B;
        const int npools = B * ((H + eg_group - 1) / eg_group);
        float *entropy = reinterpret_cast<float *>(eg_state);
        int32_t *pool = reinterpret_cast<int32_t *>(entropy + BH);
        int2 *above_at = reinterpret_cast<int2 *>(pool + BH);
        PoolSel *pools = reinterpret_cast<PoolSel *>(
            (reinterpret_cast<uintptr_t>(above_at + (int64_t)BH * Cq) + 255) & ~(uintptr_t)255);
        cudaMemsetAsync(pools, 0, (size_t)npools * sizeof(PoolSel), st);
        eg_route_kernel<<<B, 1024, 0, st>>>(cuts, sizes, entropy, pool, H, Cq, N, eg_tau, eg_group);
        const size_t lsm = (size_t)((Ct + Ch + Cw + 3) & ~3) * sizeof(float);
        const dim3 grid(Cq, BH);
        eg_hist_kernel<<<grid, kSelThreads, lsm, st>>>(a, cuts, sizes, pool, pools, -1, 11);
        eg_pick_kernel<<<npools, kSelThreads, 0, st>>>(pools, top_p, -1, 11, err);
        const int shifts[3] = {21, 10, 0}, widths[3] = {11, 11, 10};
        for (int i = 0; i < 3; ++i) {
            eg_hist_kernel<<<grid, kSelThreads, lsm, st>>>(a, cuts, sizes, pool, pools, shifts[i], widths[i]);
            eg_pick_kernel<<<npools, kSelThreads, 0, st>>>(pools, top_p, shifts[i], widths[i], err);
        }
        eg_count_kernel<<<grid, kSelThreads, lsm, st>>>(a, cuts, sizes, pool, pools, above_at);
        eg_assign_kernel<<<npools, 1024, 0, st>>>(pools, sizes, pool, above_at, r, cuts, H, eg_group, Cq, N, k_min);
        count_launches(11);
    }
    launch_topk(sizes, r, n, kh, offsets, BH, Cq, N, online, st);
    launch_emit(a, n, offsets, cuts, coarse_hist, indices, st);
}

}  // namespace scope
