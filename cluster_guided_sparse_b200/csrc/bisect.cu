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
// One CTA per node per level.  delta is formed in fp64 and the member sums
// are exact in fp64 (bf16 inputs), so the split agrees with an fp64
// evaluation except at ties below 1e-15.  The median cut is a radix select on
// the order-preserving 64-bit image of delta, and the children are written by
// a stable partition (a packed block scan per 1024-member tile).
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
    double part[2][16][64];
    int hist[256];
    int tmp[33];
    unsigned long long prefix;
    int below, need, bucket;
};

// Selects the `k` smallest keys (delta asc, member index asc) among n keys:
// returns the cut key and how many members at exactly that key are taken.
__device__ void select_k(BisectShared &S, const double *delta, int n, int k, unsigned long long *cut, int *need)
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
        for (int i0 = 0; i0 < n; i0 += blockDim.x) {
            const int i = i0 + threadIdx.x;
            int b = -1;
            if (i < n) {
                const unsigned long long u = dkey(delta[i]);
                if (hi >= 64 || (u >> hi) == (pre >> hi)) b = (int)((u >> shift) & 255ull);
            }
            const unsigned peers = __match_any_sync(0xffffffffu, b);
            if (b >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&S.hist[b], __popc(peers));
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int acc = S.below, b = 0;
            for (; b < 255; ++b) {
                if (acc + S.hist[b] >= k) break;
                acc += S.hist[b];
            }
            S.below = acc;
            S.prefix = pre | ((unsigned long long)b << shift);
        }
        __syncthreads();
    }
    *cut = S.prefix;
    *need = k - S.below;
}

// delta = ||x - c0||^2 - ||x - c1||^2 in fp64, dims in order.
__device__ __forceinline__ double split_delta(const __nv_bfloat16 *x, const double *c0, const double *c1, int D)
{
    double d0 = 0.0, d1 = 0.0;
    for (int k = 0; k < D; ++k) {
        const double xv = (double)__bfloat162float(x[k]);
        const double t0 = xv - c0[k], t1 = xv - c1[k];
        d0 = fma(t0, t0, d0);
        d1 = fma(t1, t1, d1);
    }
    return d0 - d1;
}

// One ordered pass over a node's members: f(i, side0) for every thread and
// every block of members (i >= n gives side0 = false), where side0 says
// member i goes to child 0 under (cut, need) -- keys below the cut, then the
// first `need` members at the cut in member order.  Block-wide.
template <class F>
__device__ void each_side(BisectShared &S, const double *delta, int n, unsigned long long cut, int need, F &&f)
{
    int eq_run = 0;
    for (int b0 = 0; b0 < n; b0 += blockDim.x) {
        const int i = b0 + threadIdx.x;
        const unsigned long long u = i < n ? dkey(delta[i]) : ~0ull;
        const int eq = (i < n && u == cut) ? 1 : 0;
        int tot;
        const int ex = block_excl_scan(eq, S.tmp, tot);
        f(i, i < n && (u < cut || (eq && eq_run + ex < need)));
        eq_run += tot;
    }
}

// Stable partition of a node's members by side: child 0 in member order, then child 1.
__device__ void partition_node(BisectShared &S, const double *delta, int n, unsigned long long cut, int need,
                               const int32_t *mem, int32_t *out)
{
    const int half = n >> 1;
    int s0_run = 0;
    each_side(S, delta, n, cut, need, [&](int i, bool side0) {
        int tot0;
        const int ex0 = block_excl_scan(side0 ? 1 : 0, S.tmp, tot0);
        if (i < n) {
            const int pos0 = s0_run + ex0;
            out[side0 ? pos0 : half + (i - pos0)] = mem[i];
        }
        s0_run += tot0;
    });
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
__global__ void __launch_bounds__(kBT) bisect_level_kernel(BisectArgs a)
{
    __shared__ BisectShared S;
    const int node = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int n = a.N >> a.level, D = a.D, half = n >> 1;
    const int nsl = blockDim.x >> 6;  // member slices of the update (blockDim in 128..1024)
    int32_t *mem = a.order + (int64_t)bh * a.N + (int64_t)node * n;
    int32_t *out = a.order_tmp + (int64_t)bh * a.N + (int64_t)node * n;
    double *delta = a.delta + (int64_t)bh * a.N + (int64_t)node * n;
    const __nv_bfloat16 *X = a.X + (int64_t)bh * a.N * D;

    for (int k = tid; k < 2 * D; k += blockDim.x) {
        const int which = k / D, dim = k % D;
        S.c[which][dim] = (double)__bfloat162float(X[(int64_t)mem[which ? half : 0] * D + dim]);
    }
    __syncthreads();
    unsigned long long cut = 0;
    int need = 0;
    for (int r = 0; r <= a.iters; ++r) {
        // delta of every member
        for (int i = tid; i < n; i += blockDim.x) delta[i] = split_delta(X + (int64_t)mem[i] * D, S.c[0], S.c[1], D);
        __syncthreads();
        select_k(S, delta, n, half, &cut, &need);
        if (r == a.iters) break;
        // mark sides, reusing delta as the side flag for the sums (a thread
        // reads and then overwrites only its own member's entry)
        each_side(S, delta, n, cut, need, [&](int i, bool side0) {
            if (i < n) delta[i] = side0 ? 0.0 : 1.0;
        });
        __syncthreads();
        // update: exact fp64 sums of each side (64 dims x blockDim/64 member
        // slices per pass; exact, so the slicing does not change the sums)
        for (int d0 = 0; d0 < D; d0 += 64) {
            const int dim = tid & 63, slice = tid >> 6;
            double s0 = 0.0, s1 = 0.0;
            if (d0 + dim < D) {
                for (int i = slice; i < n; i += nsl) {
                    const double xv = (double)__bfloat162float(X[(int64_t)mem[i] * D + d0 + dim]);
                    if (delta[i] == 0.0) s0 += xv;
                    else s1 += xv;
                }
            }
            S.part[0][slice][dim] = s0;
            S.part[1][slice][dim] = s1;
            __syncthreads();
            if (tid < 128) {
                const int which = tid >> 6, dd = tid & 63;
                if (d0 + dd < D) {
                    double sum = 0.0;
                    for (int q = 0; q < nsl; ++q) sum += S.part[which][q][dd];
                    S.c[which][d0 + dd] = sum / (double)half;
                }
            }
            __syncthreads();
        }
    }
    // stable partition by the final cut: side 0 (member order), then side 1
    partition_node(S, delta, n, cut, need, mem, out);
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

__global__ void __launch_bounds__(kSplitRows) bis_delta_kernel(BisectArgs a, int nodes)
{
    const int bh = blockIdx.y, D = a.D;
    const int p = blockIdx.x * kSplitRows + threadIdx.x;
    if (p >= a.N) return;
    const int n = a.N >> a.level, node = p / n;
    const int32_t m = a.order[(int64_t)bh * a.N + p];
    const double *c = a.cent + ((int64_t)bh * nodes + node) * 2 * D;
    a.delta[(int64_t)bh * a.N + p] = split_delta(a.X + ((int64_t)bh * a.N + m) * D, c, c + D, D);
}

// last == 0: mark each member's child; last == 1: write the children.
__global__ void __launch_bounds__(kBT) bis_select_kernel(BisectArgs a, int last)
{
    __shared__ BisectShared S;
    const int node = blockIdx.x, bh = blockIdx.y;
    const int n = a.N >> a.level;
    const int64_t base = (int64_t)bh * a.N + (int64_t)node * n;
    const double *delta = a.delta + base;
    unsigned long long cut = 0;
    int need = 0;
    select_k(S, delta, n, n >> 1, &cut, &need);
    if (last) {
        partition_node(S, delta, n, cut, need, a.order + base, a.order_tmp + base);
    } else {
        uint8_t *side = a.side + base;
        each_side(S, delta, n, cut, need, [&](int i, bool side0) {
            if (i < n) side[i] = side0 ? 0 : 1;
        });
    }
}

// Side sums of kSplitRows consecutive members (all of one node): 64 dims x
// kSplitRows/64 member slices per pass, then one fp64 atomic per (side, dim).
__global__ void __launch_bounds__(kSplitRows) bis_sums_kernel(BisectArgs a, int nodes)
{
    __shared__ double part[2][kSplitRows / 64][64];
    const int bh = blockIdx.y, D = a.D, tid = threadIdx.x;
    const int p0 = blockIdx.x * kSplitRows;
    const int n = a.N >> a.level, node = p0 / n;
    const int32_t *mem = a.order + (int64_t)bh * a.N;
    const uint8_t *side = a.side + (int64_t)bh * a.N;
    const __nv_bfloat16 *X = a.X + (int64_t)bh * a.N * D;
    double *g = a.gsum + ((int64_t)bh * nodes + node) * 2 * D;
    const int dim = tid & 63, slice = tid >> 6;
    for (int d0 = 0; d0 < D; d0 += 64) {
        double s0 = 0.0, s1 = 0.0;
        if (d0 + dim < D)
            for (int i = p0 + slice; i < p0 + kSplitRows; i += kSplitRows / 64) {
                const double xv = (double)__bfloat162float(X[(int64_t)mem[i] * D + d0 + dim]);
                if (side[i] == 0) s0 += xv;
                else s1 += xv;
            }
        part[0][slice][dim] = s0;
        part[1][slice][dim] = s1;
        __syncthreads();
        if (tid < 128) {
            const int which = tid >> 6, dd = tid & 63;
            if (d0 + dd < D) {
                double sum = 0.0;
                for (int q = 0; q < kSplitRows / 64; ++q) sum += part[which][q][dd];
                atomicAdd(g + which * D + d0 + dd, sum);
            }
        }
        __syncthreads();
    }
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
// bisect_aux_bytes(BH, N, D) bytes (256-byte aligned).
void launch_bisect(const __nv_bfloat16 *X, int BH, int N, int D, int leaf, int iters, int32_t *order,
                   int32_t *order_tmp, double *delta, void *aux, int32_t *labels, float *cent, float *cn,
                   int32_t *start, int32_t *sizes, int32_t *perm, cudaStream_t st)
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
                bis_delta_kernel<<<rows, kSplitRows, 0, st>>>(a, nodes);
                bis_select_kernel<<<per_node, kBT, 0, st>>>(a, r == iters ? 1 : 0);
                count_launches(2);
                if (r == iters) break;
                bis_sums_kernel<<<rows, kSplitRows, 0, st>>>(a, nodes);
                bis_means_kernel<<<per_node, 256, 0, st>>>(a);
                count_launches(2);
            }
        } else {
            // a CTA as wide as its node (128..1024 threads): deep levels have many
            // small nodes, and idle threads would only wait at the barriers
            const int threads = n >= kBT ? kBT : (n > 128 ? (n + 63) & ~63 : 128);
            bisect_level_kernel<<<dim3(nodes, BH), threads, 0, st>>>(a);
            count_launches(1);
        }
        int32_t *t = cur;
        cur = nxt;
        nxt = t;
    }
    bisect_leaves_kernel<<<dim3(N / leaf, BH), 256, 0, st>>>(X, cur, N, D, leaf, labels, cent, cn, start, sizes,
                                                             perm);
    count_launches(1);
}

}  // namespace scope
