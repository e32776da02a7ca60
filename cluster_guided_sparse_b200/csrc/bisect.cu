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
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const unsigned long long u = dkey(delta[i]);
            if (hi < 64 && (u >> hi) != (pre >> hi)) continue;
            atomicAdd(&S.hist[(u >> shift) & 255ull], 1);
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

}  // namespace

struct BisectArgs {
    const __nv_bfloat16 *X;   // [BH][N][D]
    int32_t *order;           // [BH][N] members, node by node (in/out)
    int32_t *order_tmp;       // [BH][N]
    double *delta;            // [BH][N]
    int N, D, level, iters;
};

// One CTA per (node, bh) of this level: 2-means split of the node's members.
__global__ void __launch_bounds__(kBT) bisect_level_kernel(BisectArgs a)
{
    __shared__ BisectShared S;
    const int node = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int n = a.N >> a.level, D = a.D, half = n >> 1;
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
        for (int i = tid; i < n; i += blockDim.x) {
            const __nv_bfloat16 *x = X + (int64_t)mem[i] * D;
            double d0 = 0.0, d1 = 0.0;
            for (int k = 0; k < D; ++k) {
                const double xv = (double)__bfloat162float(x[k]);
                const double t0 = xv - S.c[0][k], t1 = xv - S.c[1][k];
                d0 = fma(t0, t0, d0);
                d1 = fma(t1, t1, d1);
            }
            delta[i] = d0 - d1;
        }
        __syncthreads();
        select_k(S, delta, n, half, &cut, &need);
        if (r == a.iters) break;
        // mark sides with one ordered pass (eq keys taken in member order)
        int eq_run = 0;
        for (int b0 = 0; b0 < n; b0 += blockDim.x) {
            const int i = b0 + tid;
            const unsigned long long u = i < n ? dkey(delta[i]) : ~0ull;
            const int eq = (i < n && u == cut) ? 1 : 0;
            int tot;
            const int ex = block_excl_scan(eq, S.tmp, tot);
            if (i < n) {
                const bool side0 = u < cut || (eq && eq_run + ex < need);
                delta[i] = side0 ? 0.0 : 1.0;  // reuse as the side flag for the sums
            }
            eq_run += tot;
        }
        __syncthreads();
        // update: exact fp64 sums of each side (64 dims x 16 member slices per pass)
        for (int d0 = 0; d0 < D; d0 += 64) {
            const int dim = tid & 63, slice = tid >> 6;
            double s0 = 0.0, s1 = 0.0;
            if (d0 + dim < D) {
                for (int i = slice; i < n; i += 16) {
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
                    for (int q = 0; q < 16; ++q) sum += S.part[which][q][dd];
                    S.c[which][d0 + dd] = sum / (double)half;
                }
            }
            __syncthreads();
        }
    }
    // stable partition by the final cut: side 0 (member order), then side 1
    int eq_run = 0, s0_run = 0;
    for (int b0 = 0; b0 < n; b0 += blockDim.x) {
        const int i = b0 + tid;
        const unsigned long long u = i < n ? dkey(delta[i]) : ~0ull;
        const int eq = (i < n && u == cut) ? 1 : 0;
        int tot;
        const int ex = block_excl_scan(eq, S.tmp, tot);
        const bool side0 = i < n && (u < cut || (eq && eq_run + ex < need));
        int tot0;
        const int ex0 = block_excl_scan(side0 ? 1 : 0, S.tmp, tot0);
        if (i < n) {
            const int pos0 = s0_run + ex0;
            const int pos = side0 ? pos0 : half + (i - pos0);
            out[pos] = mem[i];
        }
        eq_run += tot;
        s0_run += tot0;
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

// Bisection of every (bh) row set of X into N/leaf leaves.
void launch_bisect(const __nv_bfloat16 *X, int BH, int N, int D, int leaf, int iters, int32_t *order,
                   int32_t *order_tmp, double *delta, int32_t *labels, float *cent, float *cn, int32_t *start,
                   int32_t *sizes, int32_t *perm, cudaStream_t st)
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
    int32_t *cur = order, *nxt = order_tmp;
    int level = 0;
    for (int n = N; n > leaf; n >>= 1, ++level) {
        a.order = cur;
        a.order_tmp = nxt;
        a.level = level;
        bisect_level_kernel<<<dim3(1u << level, BH), kBT, 0, st>>>(a);
        count_launches(1);
        int32_t *t = cur;
        cur = nxt;
        nxt = t;
    }
    bisect_leaves_kernel<<<dim3(N / leaf, BH), 256, 0, st>>>(X, cur, N, D, leaf, labels, cent, cn, start, sizes,
                                                             perm);
    count_launches(1);
}

}  // namespace scope
