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
// Top-p cut is a radix select over the order-preserving 32-bit image of the
// score, carrying per-bucket key counts and softmax masses; masses are 64-bit
// fixed point (2^40 units) so their sums are exact and order-free.
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
    int32_t *err;             // device error word
};

// -------------------------------------------------------------- LUT
// lut[c][e] for e over (t: 0..Ct-1, h: Ct.., w: Ct+Ch..): fp64 dot of the
// query centroid's subspace slice with the key centroid, stored as fp32.
__global__ void lut_kernel(const float *qcent, const float *kc_t, const float *kc_h, const float *kc_w,
                           float *lut, int Cq, int D, int dt, int dh, int dw, int Ct, int Ch, int Cw)
{
    extern __shared__ float q[];
    const int c = blockIdx.x, bh = blockIdx.y;
    const float *qc = qcent + ((int64_t)bh * Cq + c) * D;
    for (int k = threadIdx.x; k < D; k += blockDim.x) q[k] = qc[k];
    __syncthreads();
    const int Csum = Ct + Ch + Cw;
    for (int e = threadIdx.x; e < Csum; e += blockDim.x) {
        const float *kc;
        int off, ds;
        if (e < Ct) {
            kc = kc_t + ((int64_t)bh * Ct + e) * dt; off = 0; ds = dt;
        } else if (e < Ct + Ch) {
            kc = kc_h + ((int64_t)bh * Ch + (e - Ct)) * dh; off = dt; ds = dh;
        } else {
            kc = kc_w + ((int64_t)bh * Cw + (e - Ct - Ch)) * dw; off = dt + dh; ds = dw;
        }
        double s = 0.0;
        for (int k = 0; k < ds; ++k) s += (double)q[off + k] * (double)kc[k];
        lut[((int64_t)bh * Cq + c) * Csum + e] = (float)s;
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

// -------------------------------------------------------------- radix select
// Candidates are keys whose 32-bit order key matches `prefix` above the bits
// still open.  Invariant: above_met < target <= above_met + (candidates'
// metric), where above_* sum the keys strictly above the candidate range.
struct SelShared {
    unsigned long long met[2048];
    int cnt[2048];
    unsigned long long utmp[33];
    int itmp[33];
    float fred[32];
    uint32_t prefix;
    unsigned long long above_met, run_met, bucket_met, new_above_met;
    int above_cnt, run_cnt, bucket_cnt, new_above_cnt, bucket;
};

__device__ __forceinline__ float item_score(const float *L, int id, int Ch, int Cw, int Ct)
{
    const int a_w = id % Cw, a_h = (id / Cw) % Ch, a_t = id / (Cw * Ch);
    return (L[a_t] + L[Ct + a_h]) + L[Ct + Ch + a_w];
}

__device__ __forceinline__ unsigned long long item_mass(float s, float smax, float inv_sqrt_d)
{
    const float w = expf((s - smax) * inv_sqrt_d);
    return (unsigned long long)__double2ll_rn((double)w * kMassScale);
}

// One pass over `width` more bits below `shift + width`; returns false if no
// bucket satisfied the invariant (cannot happen with exact integer metrics).
__device__ bool radix_pass(SelShared &S, const float *L, const int32_t *ids, const int32_t *cnts, int n_items,
                           const SelArgs &a, float smax, bool by_mass, unsigned long long target, int shift,
                           int width)
{
    const int nb = 1 << width;
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        S.met[i] = 0ull;
        S.cnt[i] = 0;
    }
    if (threadIdx.x == 0) {
        S.run_met = 0ull;
        S.run_cnt = 0;
        S.bucket = -1;
    }
    __syncthreads();
    const uint32_t pre = S.prefix;
    const int hi = shift + width;
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const float s = item_score(L, ids[i], a.Ch, a.Cw, a.Ct);
        const uint32_t u = ordered_key(s);
        if (hi < 32 && (u >> hi) != (pre >> hi)) continue;
        const int d = (int)((u >> shift) & (uint32_t)(nb - 1));
        atomicAdd(&S.cnt[d], cnts[i]);
        atomicAdd(&S.met[d], by_mass ? (unsigned long long)cnts[i] * item_mass(s, smax, a.inv_sqrt_d)
                                     : (unsigned long long)cnts[i]);
    }
    __syncthreads();
    // Buckets from the largest key down, blockDim at a time.
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
    const bool ok = S.bucket >= 0;
    __syncthreads();
    if (threadIdx.x == 0 && ok) {
        S.above_met = S.new_above_met;
        S.above_cnt = S.new_above_cnt;
        S.prefix = pre | ((uint32_t)S.bucket << shift);
    }
    __syncthreads();
    return ok;
}

// Finds the key at which the running metric (from the largest key down)
// first reaches `target`.  Returns the number of keys taken: all keys above
// that cut key plus `need` keys at it (-1 if the invariant broke).
__device__ int radix_select(SelShared &S, const float *L, const int32_t *ids, const int32_t *cnts, int n_items,
                            const SelArgs &a, float smax, bool by_mass, unsigned long long target,
                            uint32_t *cut_key, int *need_at_cut)
{
    if (threadIdx.x == 0) {
        S.prefix = 0u;
        S.above_met = 0ull;
        S.above_cnt = 0;
    }
    __syncthreads();
    if (!radix_pass(S, L, ids, cnts, n_items, a, smax, by_mass, target, 21, 11)) return -1;
    if (!radix_pass(S, L, ids, cnts, n_items, a, smax, by_mass, target, 10, 11)) return -1;
    if (!radix_pass(S, L, ids, cnts, n_items, a, smax, by_mass, target, 0, 10)) return -1;
    // Every key in the final bucket has the same score, hence the same metric.
    const unsigned long long per = S.bucket_met / (unsigned long long)S.bucket_cnt;
    const unsigned long long rest = target - S.above_met;
    const int need = (int)((rest + per - 1) / per);
    *cut_key = S.prefix;
    *need_at_cut = need;
    return S.above_cnt + need;
}

__device__ float block_max_score(SelShared &S, const float *L, const int32_t *ids, int n_items, const SelArgs &a)
{
    float m = -INFINITY;
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) m = fmaxf(m, item_score(L, ids[i], a.Ch, a.Cw, a.Ct));
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) S.fred[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? S.fred[threadIdx.x] : -INFINITY;
        v = warp_max(v);
        if (threadIdx.x == 0) S.fred[0] = v;
    }
    __syncthreads();
    const float r = S.fred[0];
    __syncthreads();
    return r;
}

// -------------------------------------------------------------- Top-p counts
__global__ void __launch_bounds__(kSelThreads) topp_kernel(SelArgs a, int32_t *r_out)
{
    extern __shared__ float L[];
    __shared__ SelShared S;
    const int c = blockIdx.x, bh = blockIdx.y;
    const int Csum = a.Ct + a.Ch + a.Cw;
    const float *lrow = a.lut + ((int64_t)bh * a.Cq + c) * Csum;
    for (int e = threadIdx.x; e < Csum; e += blockDim.x) L[e] = lrow[e];
    __syncthreads();
    const int n_items = a.item_n[bh];
    const int32_t *ids = a.item_id + (int64_t)bh * a.Pcap;
    const int32_t *cnts = a.item_cnt + (int64_t)bh * a.Pcap;
    int m = a.N;
    if (a.top_p < 1.0f) {
        const float smax = block_max_score(S, L, ids, n_items, a);
        unsigned long long W = 0ull;
        for (int i = threadIdx.x; i < n_items; i += blockDim.x)
            W += (unsigned long long)cnts[i] * item_mass(item_score(L, ids[i], a.Ch, a.Cw, a.Ct), smax, a.inv_sqrt_d);
        unsigned long long Wt;
        block_excl_scan(W, S.utmp, Wt);
        unsigned long long target = (unsigned long long)ceil((double)a.top_p * (double)Wt);
        if (target < 1ull) target = 1ull;
        if (target > Wt) target = Wt;
        uint32_t key;
        int need;
        m = radix_select(S, L, ids, cnts, n_items, a, smax, true, target, &key, &need);
        if (m < 0) {
            if (threadIdx.x == 0) set_error(a.err, kErrRange, 0x100 + c);
            m = a.N;
        }
    }
    if (threadIdx.x == 0) {
        int r = m > a.k_min ? m : a.k_min;
        r = r < a.N ? r : a.N;
        r_out[(int64_t)bh * a.Cq + c] = r;
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
// above the cut score, then the lowest-index `need` keys at the cut score.
// Written in ascending key order: the output slot of key j is
// (#keys above the cut before j) + min(#keys at the cut before j, need).
// A key's side of the cut is its item's, so the items are classed once in
// shared memory (2 above, 1 at, 0 below) and each key costs one 16-bit load.
constexpr int kEmitPer = 8;

__global__ void __launch_bounds__(kSelThreads) emit_kernel(SelArgs a, const int32_t *n_in,
                                                           const long long *offsets, int32_t *indices)
{
    extern __shared__ __align__(16) float L[];
    __shared__ SelShared S;
    __shared__ unsigned ptmp[33];
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
    uint8_t *cls = reinterpret_cast<uint8_t *>(L + ((Csum + 3) & ~3));
    const float *lrow = a.lut + bhc * Csum;
    for (int e = threadIdx.x; e < Csum; e += blockDim.x) L[e] = lrow[e];
    __syncthreads();
    const int n_items = a.item_n[bh];
    const int32_t *ids = a.item_id + (int64_t)bh * a.Pcap;
    const int32_t *cnts = a.item_cnt + (int64_t)bh * a.Pcap;
    uint32_t cut;
    int need;
    if (radix_select(S, L, ids, cnts, n_items, a, 0.f, false, (unsigned long long)n, &cut, &need) < 0) {
        if (threadIdx.x == 0) set_error(a.err, kErrRange, 0x200 + c);
        return;
    }
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
        const uint32_t u = ordered_key(item_score(L, ids[i], a.Ch, a.Cw, a.Ct));
        cls[i] = u > cut ? 2 : (u == cut ? 1 : 0);
    }
    __syncthreads();
    const uint16_t *ki = a.key_item + (int64_t)bh * a.N;
    const bool vec = (((int64_t)bh * a.N) & 7) == 0;  // 16-byte aligned rows of 8 ranks
    int gt_run = 0, eq_run = 0;
    for (int base = 0; base < a.N; base += kSelThreads * kEmitPer) {
        const int j0 = base + threadIdx.x * kEmitPer;
        unsigned gt = 0, eq = 0;
        uint8_t k[kEmitPer];
        if (vec && j0 + kEmitPer <= a.N) {
            const uint4 w = *reinterpret_cast<const uint4 *>(ki + j0);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int t = 0; t < kEmitPer; ++t) k[t] = cls[(ws[t >> 1] >> (16 * (t & 1))) & 0xffffu];
        } else {
#pragma unroll
            for (int t = 0; t < kEmitPer; ++t) k[t] = j0 + t < a.N ? cls[ki[j0 + t]] : 0;
        }
#pragma unroll
        for (int t = 0; t < kEmitPer; ++t) {
            gt += k[t] == 2;
            eq += k[t] == 1;
        }
        unsigned tot;
        const unsigned ex = block_excl_scan(gt | (eq << 16), ptmp, tot);
        unsigned g = gt_run + (ex & 0xffffu), e = eq_run + (ex >> 16);
#pragma unroll
        for (int t = 0; t < kEmitPer; ++t) {
            const int j = j0 + t;
            if (k[t] == 2) {
                const unsigned slot = g + (e < (unsigned)need ? e : (unsigned)need);
                if (slot < (unsigned)n) out[slot] = j;
                else set_error(a.err, kErrRange, 0x300 + c);
                ++g;
            } else if (k[t] == 1) {
                if (e < (unsigned)need) {
                    if (g + e < (unsigned)n) out[g + e] = j;
                    else set_error(a.err, kErrRange, 0x300 + c);
                }
                ++e;
            }
        }
        gt_run += tot & 0xffffu;
        eq_run += tot >> 16;
    }
}

static size_t emit_smem(int Csum, int Pcap) { return (size_t)((Csum + 3) & ~3) * sizeof(float) + (size_t)Pcap; }

cudaError_t select_configure()
{
    return cudaFuncSetAttribute(emit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)emit_smem(3 * kMaxClusters, kMaxItems));
}

// -------------------------------------------------------------- launchers
void launch_lut(const float *qcent, const float *kc_t, const float *kc_h, const float *kc_w, float *lut, int BH,
                int Cq, int D, int dt, int dh, int dw, int Ct, int Ch, int Cw, cudaStream_t st)
{
    lut_kernel<<<dim3(Cq, BH), 128, D * sizeof(float), st>>>(qcent, kc_t, kc_h, kc_w, lut, Cq, D, dt, dh, dw, Ct,
                                                            Ch, Cw);
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

void launch_topp(const SelArgs &a, int32_t *r_out, cudaStream_t st)
{
    const size_t smem = (size_t)(a.Ct + a.Ch + a.Cw) * sizeof(float);
    topp_kernel<<<dim3(a.Cq, a.BH), kSelThreads, smem, st>>>(a, r_out);
    count_launches(1);
}

void launch_topk(const int32_t *sizes, const int32_t *r, int32_t *n_out, int32_t *kh, long long *offsets, int BH,
                 int Cq, int N, int online, cudaStream_t st)
{
    topk_kernel<<<1, 1024, 0, st>>>(sizes, r, n_out, kh, offsets, BH, Cq, N, online);
    count_launches(1);
}

void launch_emit(const SelArgs &a, const int32_t *n_in, const long long *offsets, int32_t *indices, cudaStream_t st)
{
    const size_t smem = emit_smem(a.Ct + a.Ch + a.Cw, a.Pcap);
    emit_kernel<<<dim3(a.Cq, a.BH), kSelThreads, smem, st>>>(a, n_in, offsets, indices);
    count_launches(1);
}

void run_selection(const float *lut, const int32_t *codes, const int32_t *item_id, const int32_t *item_cnt,
                   const int32_t *item_n, const uint16_t *key_item, int Pcap, int N, int Cq, int Ct, int Ch,
                   int Cw, int BH, float top_p, float inv_sqrt_d, int k_min, int32_t *err, const int32_t *sizes,
                   int32_t *r, int32_t *n, int32_t *kh, long long *offsets, int32_t *indices, int online,
                   cudaStream_t st)
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
    a.err = err;
    launch_topp(a, r, st);
    launch_topk(sizes, r, n, kh, offsets, BH, Cq, N, online, st);
    launch_emit(a, n, offsets, indices, st);
}

}  // namespace scope
