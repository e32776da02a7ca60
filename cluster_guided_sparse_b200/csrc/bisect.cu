// ClusterAttention variant ("ClusterAttention: A training-free speedup of
// bidirectional attention", abstract: recursive clustering with power-of-two
// cluster sizes, so block-sparse attention runs at dense per-pair throughput).
//
// Reading: balanced recursive 2-means bisection.  At a node of n rows (its
// members in token order) the two centroids start at members 0 and n/2;
// every assign ranks the members by delta = ||x-c0||^2 - ||x-c1||^2 (ties:
// lower token first) and sends the first n/2 to child 0; every update takes
// the two means.  `iters` (assign, update) rounds, then a final assign
// decides the children.  Recursion stops at `leaf` rows; leaves are numbered
// depth-first, child 0 first, which is the order of the member array after
// the last level.
//
// delta is formed in fp64 (dims in order) and the member sums are exact in
// fp64 (bf16 inputs), so the split agrees with an fp64 evaluation except at
// ties below 1e-15.  The median cut is an exact select on the order-preserving
// 64-bit image of delta (equal keys taken in member order): min and max, a
// histogram of equal-width value buckets (the bucket is a non-decreasing
// function of delta), then the crossing bucket's keys alone, ranked by one
// warp when there are at most 32 of them and by a radix select otherwise (a
// radix select over all members when the bucket is too full).  Members go to
// their side by a plain comparison unless some keys at the cut are left out;
// the children are written by a stable partition (a block scan per tile).
// Nodes of 2048 rows and more run each round as four kernels over all
// members (delta, cut, side sums, means); smaller nodes as one CTA per node
// with every round inside.  The queries' and the keys' row sets of a call are
// bisected together (2*BH row sets), so the top levels' few nodes fill more
// of the GPU.
#include "common.cuh"

namespace scope {

namespace {

constexpr int kBT = 1024;
constexpr int kSplitNodes = 64;  // most nodes per head on a split level

__device__ __forceinline__ unsigned long long dkey(double d)
{
    const unsigned long long u = (unsigned long long)__double_as_longlong(d);
    return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

struct BisectShared {
    double c[2][128];
    double sum[2][128];
    int hist[256];
    int tmp[33];
    unsigned long long prefix;
    int below, need, bucket, eq;
};

// A node's median cut: members with keys below `key` go to child 0, and of
// the `eq` members at exactly `key` the first `need` in member order.
struct Cut {
    unsigned long long key;
    int need, eq;
};

// Selects the `k` smallest of n ordered 64-bit keys (key(i), member index
// asc): the cut key, how many keys equal it and how many of those are
// taken.  Eight 8-bit radix passes.
template <class Key>
__device__ void radix_select(BisectShared &S, Key key, int n, int k, Cut &c)
{
    if (threadIdx.x == 0) {
        S.prefix = 0ull;
        S.below = 0;
    }
    __syncthreads();
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) S.hist[i] = 0;
        __syncthreads();
        const unsigned long long pre = S.prefix;
        const int hi = shift + 8;
        // A node's deltas share their leading bytes, so most keys fall in one
        // bucket: add per warp (one atomic per distinct bucket) instead of
        // per key, which would serialise on that bucket.
        const int step = 4 * blockDim.x;
        for (int i0 = 0; i0 < n; i0 += step) {
            unsigned long long u[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = i0 + e * blockDim.x + threadIdx.x;
                u[e] = i < n ? key(i) : 0ull;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = i0 + e * blockDim.x + threadIdx.x;
                int b = -1;
                if (i < n && (hi >= 64 || (u[e] >> hi) == (pre >> hi))) b = (int)((u[e] >> shift) & 255ull);
                const unsigned peers = __match_any_sync(0xffffffffu, b);
                if (b >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&S.hist[b], __popc(peers));
            }
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // the first bucket b (< 255) where the running count reaches k,
            // else 255: lane L scans buckets 8L..8L+7 from its exclusive prefix
            const int lane = threadIdx.x;
            int h[8], loc = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                h[e] = S.hist[lane * 8 + e];
                loc += h[e];
            }
            const int before = S.below + warp_incl_scan(loc) - loc;
            const unsigned hit = __ballot_sync(0xffffffffu, before + loc >= k);
            if (lane == (hit ? __ffs(hit) - 1 : 31)) {
                int acc = before, b = lane * 8, cnt = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e, ++b) {
                    cnt = h[e];
                    if (b == 255 || acc + h[e] >= k) break;
                    acc += h[e];
                }
                S.below = acc;
                S.eq = cnt;
                S.prefix = pre | ((unsigned long long)b << shift);
            }
        }
        __syncthreads();
    }
    c.key = S.prefix;
    c.need = k - S.below;
    c.eq = S.eq;  // the last pass's bucket holds exactly the keys equal to the cut
}

__device__ __forceinline__ void select_k(BisectShared &S, const double *delta, int n, int k, Cut &c)
{
    radix_select(S, [&](int i) { return dkey(delta[i]); }, n, k, c);
}

// The same selection for large nodes in fewer passes over the deltas:
// min and max, a histogram of 4096 equal-width buckets of the delta value
// (the bucket is a non-decreasing function of delta, so every key of an
// earlier bucket is below every key of a later one), the bucket where the
// running count reaches k, and the radix select among that bucket's keys
// only, gathered in shared memory.  A bucket holding more than kCoarseCap
// keys falls back to the radix select over all n.
constexpr int kCoarse = 4096, kCoarseCap = 2048;
template <int NB, int CAP>
struct CoarseT {
    int hist[NB];
    unsigned long long list[CAP];
    double red[2][32];
    double lo, scale;
    int nlist, bucket, below;
};
using CoarseShared = CoarseT<kCoarse, kCoarseCap>;  // top-level nodes (one CTA per node)
using CoarseSmall = CoarseT<2048, 256>;            // nodes of up to 2048 rows

// The exact cut among m <= 32 keys, by one warp: a lane's key is the cut when
// fewer than k keys are below it and at least k are at or below it.
__device__ void small_select(BisectShared &S, const unsigned long long *list, int m, int k, Cut &c)
{
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const unsigned long long u = lane < m ? list[lane] : ~0ull;
        int lt = 0, le = 0;
        for (int i = 0; i < m; ++i) {
            const unsigned long long v = __shfl_sync(0xffffffffu, u, i);
            lt += v < u ? 1 : 0;
            le += v <= u ? 1 : 0;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, lane < m && lt < k && k <= le);
        if (lane == __ffs(hit) - 1) {
            S.prefix = u;
            S.need = k - lt;
            S.eq = le - lt;
        }
    }
    __syncthreads();
    c.key = S.prefix;
    c.need = S.need;
    c.eq = S.eq;
}

// The same for m <= a few hundred keys, block-wide: every key counts the keys
// below it and at or below it.
__device__ void block_rank_select(BisectShared &S, const unsigned long long *list, int m, int k, Cut &c)
{
    for (int p = threadIdx.x; p < m; p += blockDim.x) {
        const unsigned long long u = list[p];
        int lt = 0, le = 0;
        for (int q = 0; q < m; ++q) {
            const unsigned long long v = list[q];
            lt += v < u ? 1 : 0;
            le += v <= u ? 1 : 0;
        }
        if (lt < k && k <= le) {  // every key equal to the cut writes the same values
            S.prefix = u;
            S.need = k - lt;
            S.eq = le - lt;
        }
    }
    __syncthreads();
    c.key = S.prefix;
    c.need = S.need;
    c.eq = S.eq;
}

template <int NB, int CAP>
__device__ void select_k_coarse(BisectShared &S, CoarseT<NB, CAP> &C, const double *delta, int n, int k, Cut &c)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    double lo = INFINITY, hi = -INFINITY;
    for (int i = tid; i < n; i += blockDim.x) {
        const double d = delta[i];
        lo = fmin(lo, d);
        hi = fmax(hi, d);
    }
    for (int o = 16; o > 0; o >>= 1) {
        lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
        C.red[0][warp] = lo;
        C.red[1][warp] = hi;
    }
    for (int b = tid; b < NB; b += blockDim.x) C.hist[b] = 0;
    __syncthreads();
    if (tid == 0) {
        double l = C.red[0][0], h = C.red[1][0];
        for (int w = 1; w < nw; ++w) {
            l = fmin(l, C.red[0][w]);
            h = fmax(h, C.red[1][w]);
        }
        C.lo = l;
        C.scale = h > l ? (double)NB / (h - l) : 0.0;
        C.nlist = 0;
    }
    __syncthreads();
    const double l = C.lo, sc = C.scale;
    auto bucket_of = [&](double d) { return min(NB - 1, (int)((d - l) * sc)); };
    for (int i0 = 0; i0 < n; i0 += blockDim.x) {
        const int i = i0 + tid;
        const int b = i < n ? bucket_of(delta[i]) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, b);
        if (b >= 0 && lane == __ffs(peers) - 1) atomicAdd(&C.hist[b], __popc(peers));
    }
    __syncthreads();
    // the first bucket where the running count reaches k: thread t scans
    // buckets [t*per, (t+1)*per) from its exclusive prefix
    const int per = (NB + blockDim.x - 1) / blockDim.x;
    const int b0 = min(NB, tid * per), b1 = min(NB, b0 + per);
    int loc = 0;
    for (int b = b0; b < b1; ++b) loc += C.hist[b];
    int tot;
    const int before = block_excl_scan(loc, S.tmp, tot);
    if (before < k && before + loc >= k) {
        int acc = before, b = b0;
        for (; acc + C.hist[b] < k; ++b) acc += C.hist[b];
        C.bucket = b;
        C.below = acc;
    }
    __syncthreads();
    const int bk = C.bucket, below = C.below, m = C.hist[bk];
    if (m > CAP) {
        select_k(S, delta, n, k, c);
        return;
    }
    for (int i = tid; i < n; i += blockDim.x) {
        const double d = delta[i];
        if (bucket_of(d) == bk) C.list[atomicAdd(&C.nlist, 1)] = dkey(d);
    }
    __syncthreads();
    if (m <= 32) small_select(S, C.list, m, k - below, c);
    else if (m <= 512) block_rank_select(S, C.list, m, k - below, c);
    else radix_select(S, [&](int i) { return C.list[i]; }, m, k - below, c);
}

// delta = ||x - c0||^2 - ||x - c1||^2 in fp64, dims in order.  The row is
// read 8 dims (16 bytes) at a time (rows are 16-byte aligned).
template <int D>
__device__ __forceinline__ double split_delta(const __nv_bfloat16 *x, const double *c0, const double *c1)
{
    double d0 = 0.0, d1 = 0.0;
#pragma unroll 2
    for (int k0 = 0; k0 < D; k0 += 8) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(x + k0);
        const __nv_bfloat16 *xv8 = reinterpret_cast<const __nv_bfloat16 *>(&raw);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double xv = (double)__bfloat162float(xv8[e]);
            const double t0 = xv - c0[k0 + e], t1 = xv - c1[k0 + e];
            d0 = fma(t0, t0, d0);
            d1 = fma(t1, t1, d1);
        }
    }
    return d0 - d1;
}

// Member sides under a cut, block-wide: f(i, side0) once for every member
// i < n, where side0 says member i goes to child 0.  Without ties at the cut
// (every member at the cut is taken) that is a plain comparison; otherwise
// the members are visited in tiles of blockDim in member order and a block
// scan ranks the members at the cut.
template <class F>
__device__ void mark_sides(BisectShared &S, const double *delta, int n, const Cut &c, F &&f)
{
    if (c.need == c.eq) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) f(i, dkey(delta[i]) <= c.key);
        return;
    }
    int eq_run = 0;
    for (int b0 = 0; b0 < n; b0 += blockDim.x) {
        const int i = b0 + threadIdx.x;
        const unsigned long long u = i < n ? dkey(delta[i]) : ~0ull;
        const int eq = (i < n && u == c.key) ? 1 : 0;
        int tot;
        const int ex = block_excl_scan(eq, S.tmp, tot);
        if (i < n) f(i, u < c.key || (eq && eq_run + ex < c.need));
        eq_run += tot;
    }
}

// Stable partition of a node's members by side: child 0 in member order,
// then child 1.  Tiles of 4 members per thread; one block scan per tile
// places child 0 (a second one ranks the members at the cut when some of
// them are left out).
__device__ void partition_node(BisectShared &S, const double *delta, int n, const Cut &c, const int32_t *mem,
                               int32_t *out)
{
    constexpr int E = 4;
    const int half = n >> 1;
    const bool ties = c.need != c.eq;
    int s0_run = 0, eq_run = 0;
    for (int b0 = 0; b0 < n; b0 += E * blockDim.x) {
        const int i0 = b0 + threadIdx.x * E;
        unsigned long long u[E];
        int neq = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            u[e] = i0 + e < n ? dkey(delta[i0 + e]) : ~0ull;
            neq += (i0 + e < n && u[e] == c.key) ? 1 : 0;
        }
        int eq_rank = 0;
        if (ties) {
            int tot;
            eq_rank = eq_run + block_excl_scan(neq, S.tmp, tot);
            eq_run += tot;
        }
        bool side0[E];
        int ns0 = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const bool eq = i0 + e < n && u[e] == c.key;
            side0[e] = i0 + e < n && (u[e] < c.key || (eq && (!ties || eq_rank < c.need)));
            if (eq) ++eq_rank;
            ns0 += side0[e] ? 1 : 0;
        }
        int tot0;
        int pos0 = s0_run + block_excl_scan(ns0, S.tmp, tot0);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int i = i0 + e;
            if (i < n) {
                if (side0[e]) out[pos0++] = mem[i];
                else out[half + (i - pos0)] = mem[i];
            }
        }
        s0_run += tot0;
    }
}

// Adds member i's row into its side's sums, warp-wide: every lane holds
// D/32 consecutive dims of both sides' running sums.  The sums of bf16
// values in fp64 are exact, so the order of the additions does not matter.
template <int D>
__device__ __forceinline__ void add_row(const __nv_bfloat16 *x, bool side0, double (&s0)[D / 32], double (&s1)[D / 32])
{
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    float v[PER];
    if constexpr (PER == 4) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(x + lane * 4);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
        v[0] = __low2float(a);
        v[1] = __high2float(a);
        v[2] = __low2float(b);
        v[3] = __high2float(b);
    } else {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(x + lane * 2);
        v[0] = __low2float(a);
        v[1] = __high2float(a);
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        if (side0) s0[e] += (double)v[e];
        else s1[e] += (double)v[e];
    }
}

}  // namespace

struct BisectArgs {
    const __nv_bfloat16 *X;   // [BH][N][D]
    int32_t *order;           // [BH][N] members, node by node (in/out)
    int32_t *order_tmp;       // [BH][N]
    double *delta;            // [BH][N]
    uint8_t *side;            // [BH][N] child of each member (split levels)
    double *cent;             // [BH][kSplitNodes][2][D] node centroids (split levels)
    double *gsum;             // [BH][kSplitNodes][2][D] side sums, zero between rounds
    int N, D, level, iters;
};

// One CTA per (node, bh) of this level: 2-means split of the node's members.
template <int D>
__global__ void __launch_bounds__(kBT) bisect_level_kernel(BisectArgs a)
{
    __shared__ BisectShared S;
    __shared__ CoarseSmall C;
    const int node = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int n = a.N >> a.level, half = n >> 1;
    const int lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    constexpr int PER = D / 32;
    int32_t *mem = a.order + (int64_t)bh * a.N + (int64_t)node * n;
    int32_t *out = a.order_tmp + (int64_t)bh * a.N + (int64_t)node * n;
    double *delta = a.delta + (int64_t)bh * a.N + (int64_t)node * n;
    const __nv_bfloat16 *X = a.X + (int64_t)bh * a.N * D;

    for (int k = tid; k < 2 * D; k += blockDim.x) {
        const int which = k / D, dim = k % D;
        S.c[which][dim] = (double)__bfloat162float(X[(int64_t)mem[which ? half : 0] * D + dim]);
    }
    __syncthreads();
    Cut cut;
    for (int r = 0; r <= a.iters; ++r) {
        // delta of every member
        for (int i = tid; i < n; i += blockDim.x) delta[i] = split_delta<D>(X + (int64_t)mem[i] * D, S.c[0], S.c[1]);
        __syncthreads();
        select_k_coarse(S, C, delta, n, half, cut);
        if (r == a.iters) break;
        // mark sides, reusing delta as the side flag for the sums (a thread
        // reads and then overwrites only its own member's entry)
        mark_sides(S, delta, n, cut, [&](int i, bool side0) { delta[i] = side0 ? 0.0 : 1.0; });
        for (int k = tid; k < 2 * D; k += blockDim.x) S.sum[k / D][k % D] = 0.0;
        __syncthreads();
        // update: each warp adds whole rows into its registers, then the
        // warps' sums meet in shared memory (exact, so in any order)
        double s0[PER], s1[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) s0[e] = s1[e] = 0.0;
#pragma unroll 4
        for (int i = warp; i < n; i += nw) add_row<D>(X + (int64_t)mem[i] * D, delta[i] == 0.0, s0, s1);
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            atomicAdd(&S.sum[0][lane * PER + e], s0[e]);
            atomicAdd(&S.sum[1][lane * PER + e], s1[e]);
        }
        __syncthreads();
        for (int k = tid; k < 2 * D; k += blockDim.x) S.c[k / D][k % D] = S.sum[k / D][k % D] / (double)half;
        __syncthreads();
    }
    // stable partition by the final cut: side 0 (member order), then side 1
    partition_node(S, delta, n, cut, mem, out);
}

// ---------------------------------------------------------------- split levels
// The top levels have few nodes (one per head at level 0), so one CTA per
// node would leave most SMs idle.  There each round runs as separate
// kernels: deltas and side sums over all members of all nodes, the select
// (and the side marks or the final partition) one CTA per node.  The
// arithmetic is the fused kernel's: the same fp64 delta, the same select,
// exact fp64 side sums (now added across CTAs), so the children are the same.
constexpr int kSplitRows = 256;

__global__ void __launch_bounds__(128) bis_init_kernel(BisectArgs a)
{
    const int node = blockIdx.x, bh = blockIdx.y, nodes = gridDim.x;
    const int n = a.N >> a.level, D = a.D;
    const int32_t *mem = a.order + (int64_t)bh * a.N + (int64_t)node * n;
    const __nv_bfloat16 *X = a.X + (int64_t)bh * a.N * D;
    double *c = a.cent + ((int64_t)bh * nodes + node) * 2 * D;
    for (int k = threadIdx.x; k < 2 * D; k += blockDim.x) {
        const int which = k / D, dim = k % D;
        c[k] = (double)__bfloat162float(X[(int64_t)mem[which ? n >> 1 : 0] * D + dim]);
    }
}

template <int D>
__global__ void __launch_bounds__(kSplitRows) bis_delta_kernel(BisectArgs a, int nodes)
{
    __shared__ double c[2 * D];
    const int bh = blockIdx.y;
    const int p0 = blockIdx.x * kSplitRows, p = p0 + threadIdx.x;
    const int n = a.N >> a.level;  // n >= kSplitRows and n % kSplitRows == 0 on split levels
    const double *cg = a.cent + ((int64_t)bh * nodes + p0 / n) * 2 * D;
    for (int k = threadIdx.x; k < 2 * D; k += kSplitRows) c[k] = cg[k];
    __syncthreads();
    if (p >= a.N) return;
    const int32_t m = a.order[(int64_t)bh * a.N + p];
    a.delta[(int64_t)bh * a.N + p] = split_delta<D>(a.X + ((int64_t)bh * a.N + m) * D, c, c + D);
}

// last == 0: mark each member's child; last == 1: write the children.
__global__ void __launch_bounds__(kBT) bis_select_kernel(BisectArgs a, int last)
{
    __shared__ BisectShared S;
    __shared__ CoarseShared C;
    const int node = blockIdx.x, bh = blockIdx.y;
    const int n = a.N >> a.level;
    const int64_t base = (int64_t)bh * a.N + (int64_t)node * n;
    const double *delta = a.delta + base;
    Cut cut;
    select_k_coarse(S, C, delta, n, n >> 1, cut);
    if (last) {
        partition_node(S, delta, n, cut, a.order + base, a.order_tmp + base);
    } else {
        uint8_t *side = a.side + base;
        mark_sides(S, delta, n, cut, [&](int i, bool side0) { side[i] = side0 ? 0 : 1; });
    }
}

// Side sums of kSplitRows consecutive members (all of one node): a warp takes
// 32 members, adds their rows into its registers (add_row), the CTA's warps
// meet in shared memory, and one fp64 atomic per (side, dim) adds the CTA's
// sums to the node's.
template <int D>
__global__ void __launch_bounds__(kSplitRows) bis_sums_kernel(BisectArgs a, int nodes)
{
    __shared__ double sum[2][D];
    constexpr int PER = D / 32;
    const int bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int p0 = blockIdx.x * kSplitRows;
    const int node = p0 / (a.N >> a.level);
    for (int k = tid; k < 2 * D; k += kSplitRows) sum[k / D][k % D] = 0.0;
    const int i = p0 + warp * 32 + lane;  // N is a multiple of kSplitRows here
    const int mi = a.order[(int64_t)bh * a.N + i];
    const int si = a.side[(int64_t)bh * a.N + i];
    const __nv_bfloat16 *X = a.X + (int64_t)bh * a.N * D;
    double s0[PER], s1[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) s0[e] = s1[e] = 0.0;
#pragma unroll 8
    for (int r = 0; r < 32; ++r) {
        const int m = __shfl_sync(0xffffffffu, mi, r), sd = __shfl_sync(0xffffffffu, si, r);
        add_row<D>(X + (int64_t)m * D, sd == 0, s0, s1);
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        atomicAdd(&sum[0][lane * PER + e], s0[e]);
        atomicAdd(&sum[1][lane * PER + e], s1[e]);
    }
    __syncthreads();
    double *g = a.gsum + ((int64_t)bh * nodes + node) * 2 * D;
    for (int k = tid; k < 2 * D; k += kSplitRows) atomicAdd(g + k, sum[k / D][k % D]);
}

__global__ void __launch_bounds__(256) bis_means_kernel(BisectArgs a)
{
    const int node = blockIdx.x, bh = blockIdx.y, nodes = gridDim.x;
    const int half = (a.N >> a.level) >> 1;
    const int64_t o = ((int64_t)bh * nodes + node) * 2 * a.D;
    for (int k = threadIdx.x; k < 2 * a.D; k += blockDim.x) {
        a.cent[o + k] = a.gsum[o + k] / (double)half;
        a.gsum[o + k] = 0.0;
    }
}

// After the last level: labels (leaf id of each token), leaf centroids (fp32
// means), leaf starts and sizes; `order` becomes the cluster-major permutation.
__global__ void __launch_bounds__(256) bisect_leaves_kernel(const __nv_bfloat16 *X, const int32_t *order, int N,
                                                            int D, int leaf, int32_t *labels, float *cent,
                                                            float *cn, int32_t *start, int32_t *sizes, int32_t *perm)
{
    __shared__ double part[4][64];
    const int c = blockIdx.x, bh = blockIdx.y, C = N / leaf;
    const int32_t *mem = order + (int64_t)bh * N + (int64_t)c * leaf;
    for (int i = threadIdx.x; i < leaf; i += blockDim.x) {
        labels[(int64_t)bh * N + mem[i]] = c;
        perm[(int64_t)bh * N + (int64_t)c * leaf + i] = mem[i];
    }
    const int dim = threadIdx.x & 63, slice = threadIdx.x >> 6;
    const __nv_bfloat16 *Xb = X + (int64_t)bh * N * D;
    float *cc = cent + ((int64_t)bh * C + c) * D;
    for (int d0 = 0; d0 < D; d0 += 64) {
        double s = 0.0;
        if (d0 + dim < D)
            for (int i = slice; i < leaf; i += 4) s += (double)__bfloat162float(Xb[(int64_t)mem[i] * D + d0 + dim]);
        part[slice][dim] = s;
        __syncthreads();
        if (threadIdx.x < 64 && d0 + threadIdx.x < D)
            cc[d0 + threadIdx.x] = (float)((part[0][threadIdx.x] + part[1][threadIdx.x] + part[2][threadIdx.x] +
                                            part[3][threadIdx.x]) /
                                           (double)leaf);
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        float s = 0.f;
        for (int k = 0; k < D; ++k) s = fmaf(cc[k], cc[k], s);
        cn[(int64_t)bh * C + c] = s;
        sizes[(int64_t)bh * C + c] = leaf;
        start[(int64_t)bh * (C + 1) + c] = c * leaf;
        if (c == C - 1) start[(int64_t)bh * (C + 1) + C] = N;
    }
}

__global__ void iota_kernel(int32_t *order, int N, int64_t total)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < total) order[i] = (int32_t)(i % N);
}

// Bytes of the split-level scratch (member sides, node centroids, side sums).
size_t bisect_aux_bytes(int BH, int N, int D)
{
    return (((size_t)BH * N + 255) & ~(size_t)255) + 2 * (size_t)BH * kSplitNodes * 2 * D * sizeof(double);
}

// Bisection of every (bh) row set of X into N/leaf leaves.  `aux` holds
// bisect_aux_bytes(BH, N, D) bytes (256-byte aligned).  The BH row sets are
// nout consecutive parts of BH / nout (the queries and the keys of a call,
// bisected together so that the top levels' few nodes fill more of the
// GPU); part p's leaves go to out[p].
void launch_bisect(const __nv_bfloat16 *X, int BH, int N, int D, int leaf, int iters, int32_t *order,
                   int32_t *order_tmp, double *delta, void *aux, const BisectOut *out, int nout, cudaStream_t st)
{
    const int64_t total = (int64_t)BH * N;
    iota_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(order, N, total);
    count_launches(1);
    BisectArgs a;
    a.X = X;
    a.N = N;
    a.D = D;
    a.iters = iters;
    a.delta = delta;
    a.side = (uint8_t *)aux;
    a.cent = (double *)((char *)aux + (((size_t)BH * N + 255) & ~(size_t)255));
    a.gsum = a.cent + (size_t)BH * kSplitNodes * 2 * D;
    cudaMemsetAsync(a.gsum, 0, (size_t)BH * kSplitNodes * 2 * D * sizeof(double), st);
    int32_t *cur = order, *nxt = order_tmp;
    int level = 0;
    for (int n = N; n > leaf; n >>= 1, ++level) {
        a.order = cur;
        a.order_tmp = nxt;
        a.level = level;
        const int nodes = 1 << level;
        if (nodes <= kSplitNodes && nodes * BH < 2 * 148 && n >= 2048 && n % kSplitRows == 0) {
            const dim3 rows((unsigned)(N / kSplitRows), BH), per_node(nodes, BH);
            bis_init_kernel<<<per_node, 128, 0, st>>>(a);
            count_launches(1);
            for (int r = 0; r <= iters; ++r) {
                if (D == 64) bis_delta_kernel<64><<<rows, kSplitRows, 0, st>>>(a, nodes);
                else bis_delta_kernel<128><<<rows, kSplitRows, 0, st>>>(a, nodes);
                bis_select_kernel<<<per_node, kBT, 0, st>>>(a, r == iters ? 1 : 0);
                count_launches(2);
                if (r == iters) break;
                if (D == 64) bis_sums_kernel<64><<<rows, kSplitRows, 0, st>>>(a, nodes);
                else bis_sums_kernel<128><<<rows, kSplitRows, 0, st>>>(a, nodes);
                bis_means_kernel<<<per_node, 256, 0, st>>>(a);
                count_launches(2);
            }
        } else {
            // a CTA as wide as its node (128..1024 threads): deep levels have many
            // small nodes, and idle threads would only wait at the barriers
            const int threads = n >= kBT ? kBT : (n > 128 ? (n + 63) & ~63 : 128);
            if (D == 64) bisect_level_kernel<64><<<dim3(nodes, BH), threads, 0, st>>>(a);
            else bisect_level_kernel<128><<<dim3(nodes, BH), threads, 0, st>>>(a);
            count_launches(1);
        }
        int32_t *t = cur;
        cur = nxt;
        nxt = t;
    }
    const int per = BH / nout;
    for (int q = 0; q < nout; ++q) {
        const BisectOut &o = out[q];
        bisect_leaves_kernel<<<dim3(N / leaf, per), 256, 0, st>>>(X + (int64_t)q * per * N * D,
                                                                  cur + (int64_t)q * per * N, N, D, leaf, o.labels,
                                                                  o.cent, o.cn, o.start, o.sizes, o.perm);
        count_launches(1);
    }
}

}  // namespace scope
