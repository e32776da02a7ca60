// Step 2 of SCOPE (abstract: post-RoPE keys are partitioned into temporal,
// height and width subspaces that are "clustered independently"; queries are
// grouped into query clusters): fixed-iteration Lloyd k-means.
//
// Readings: squared Euclidean distance; strided init at rows
// off + j*floor(N/C) with off = seed mod floor(N/C); argmin ties to the lowest
// index; an empty cluster keeps its centroid; `iters` (assign, update) rounds,
// then a final assign.
//
// Determinism: the update is a stable counting sort of the labels (so every
// cluster's members are listed in ascending token order) followed by one CTA
// per cluster summing its members in 64-bit fixed point.  Integer sums do not
// depend on the order of accumulation, and the shift is chosen so that the
// sum of bf16 inputs is exact; a rerun gives identical centroids, hence
// identical labels.
#include "common.cuh"

namespace scope {

__device__ __forceinline__ int fixed_shift(const uint32_t *maxabs_bits, int N)
{
    // Sum of N values of magnitude <= m must stay below 2^52 (exact in double).
    const float m = __uint_as_float(*maxabs_bits);
    const double bound = (double)m * (double)N + 1.0;
    int S = 52 - (ilogb(bound) + 1);
    return S < 0 ? 0 : (S > 40 ? 40 : S);
}

// -------------------------------------------------------------- init
__global__ void km_init_kernel(KmBatch b, int N, int D, uint32_t seed)
{
    const KmProblem &P = b.p[blockIdx.z];
    const int c = blockIdx.x, bh = blockIdx.y;
    if (c >= P.C) return;
    const int stride = N / P.C;
    const int off = (int)(seed % (uint32_t)stride);
    const __nv_bfloat16 *x = P.X + ((int64_t)bh * N + off + (int64_t)c * stride) * D + P.dim_off;
    float *cent = P.cent + ((int64_t)bh * P.C + c) * P.dim_n;
    for (int k = threadIdx.x; k < P.dim_n; k += blockDim.x) cent[k] = __bfloat162float(x[k]);
    __syncthreads();
    if (threadIdx.x == 0) {
        float s = 0.f;
        for (int k = 0; k < P.dim_n; ++k) s = fmaf(cent[k], cent[k], s);
        P.cn[(int64_t)bh * P.C + c] = s;
    }
}

// Packed f32x2 arithmetic on 64-bit register pairs (lane 0 = low word), IEEE
// round-to-nearest without flushing subnormals: each lane gives the same fp32
// result as the scalar instruction.
__device__ __forceinline__ unsigned long long pack2(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void unpack2(unsigned long long v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b)
{
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// acc + d * d
__device__ __forceinline__ unsigned long long sqacc2(unsigned long long acc, unsigned long long d)
{
    asm("fma.rn.f32x2 %0, %1, %1, %0;" : "+l"(acc) : "l"(d));
    return acc;
}

// -------------------------------------------------------------- assign (direct form)
// Two adjacent rows per thread (256 per CTA).  Their columns are staged in
// shared memory as bf16 pairs (one 32-bit word per column, transposed so
// consecutive threads read consecutive words); the centroids stream through in
// chunks of W, negated and duplicated ((-c, -c) per column), so one packed add
// forms x - c for both rows and one packed FMA adds both squares: the pair
// (x0, x1) is built once per column and every 16-byte broadcast load feeds two
// centroids x two rows.  d = sum_k (x_k - c_k)^2 in fp32 with k ascending: no
// cancellation, relative error <= (dim+2) * 2^-24 of the distance.
constexpr int kDirRows = 256, kDirCH = 32;

template <int W>
__device__ __forceinline__ void direct_chunk(const uint32_t *xs, const unsigned long long *cs, int dn, int c0, int C,
                                             float (&best)[2], int (&arg)[2])
{
    unsigned long long acc[W];
#pragma unroll
    for (int j = 0; j < W; ++j) acc[j] = 0ull;
    for (int k = 0; k < dn; ++k) {
        const uint32_t xp = xs[k * (kDirRows / 2) + threadIdx.x];
        const unsigned long long x = pack2(__uint_as_float(xp << 16), __uint_as_float(xp & 0xffff0000u));
        const ulonglong2 *c2 = reinterpret_cast<const ulonglong2 *>(cs + k * kDirCH);
#pragma unroll
        for (int j2 = 0; j2 < W / 2; ++j2) {
            const ulonglong2 c = c2[j2];
            acc[2 * j2] = sqacc2(acc[2 * j2], add2(x, c.x));
            acc[2 * j2 + 1] = sqacc2(acc[2 * j2 + 1], add2(x, c.y));
        }
    }
#pragma unroll
    for (int j = 0; j < W; ++j) {
        float d0, d1;
        unpack2(acc[j], d0, d1);
        const bool in = c0 + j < C;
        const bool lt0 = in && d0 < best[0], lt1 = in && d1 < best[1];  // first minimum wins
        best[0] = lt0 ? d0 : best[0];
        arg[0] = lt0 ? c0 + j : arg[0];
        best[1] = lt1 ? d1 : best[1];
        arg[1] = lt1 ? c0 + j : arg[1];
    }
}

__global__ void __launch_bounds__(kDirRows / 2) km_assign_direct_kernel(KmBatch b, int N, int D)
{
    extern __shared__ __align__(16) uint32_t smw[];
    const KmProblem &P = b.p[blockIdx.z];
    const int bh = blockIdx.y, T = kDirRows / 2;
    const int n0 = blockIdx.x * kDirRows;
    if (n0 >= N) return;
    const int dn = P.dim_n, C = P.C;
    uint32_t *xs = smw;                                                          // [dn][T]
    unsigned long long *cs = reinterpret_cast<unsigned long long *>(smw + ((dn * T + 3) & ~3));  // [dn][kDirCH]
    const __nv_bfloat16 *Xb = P.X + (int64_t)bh * N * D + P.dim_off;
    // row pair t -> xs[k][t] = bf16(row 2t) | bf16(row 2t+1) << 16
    if (((P.dim_off | dn) & 7) == 0) {
        for (int idx = threadIdx.x; idx < T * (dn >> 3); idx += T) {
            const int t = idx % T, k8 = (idx / T) * 8, n = n0 + 2 * t;
            uint4 u0 = make_uint4(0u, 0u, 0u, 0u), u1 = u0;
            if (n < N) u0 = *reinterpret_cast<const uint4 *>(Xb + (int64_t)n * D + k8);
            if (n + 1 < N) u1 = *reinterpret_cast<const uint4 *>(Xb + (int64_t)(n + 1) * D + k8);
            const uint32_t a[4] = {u0.x, u0.y, u0.z, u0.w}, c[4] = {u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                xs[(k8 + 2 * q) * T + t] = __byte_perm(a[q], c[q], 0x5410);
                xs[(k8 + 2 * q + 1) * T + t] = __byte_perm(a[q], c[q], 0x7632);
            }
        }
    } else {
        const unsigned short *Xs = reinterpret_cast<const unsigned short *>(Xb);
        for (int idx = threadIdx.x; idx < T * dn; idx += T) {
            const int t = idx % T, k = idx / T, n = n0 + 2 * t;
            const uint32_t lo = n < N ? Xs[(int64_t)n * D + k] : 0u;
            const uint32_t hi = n + 1 < N ? Xs[(int64_t)(n + 1) * D + k] : 0u;
            xs[k * T + t] = lo | (hi << 16);
        }
    }
    float best[2] = {INFINITY, INFINITY};
    int arg[2] = {0, 0};
    const float *cent = P.cent + (int64_t)bh * C * dn;
    for (int c0 = 0; c0 < C; c0 += kDirCH) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kDirCH * dn; idx += T) {
            const int j = idx % kDirCH, k = idx / kDirCH;  // consecutive threads: consecutive centroids
            const float v = (c0 + j < C) ? -cent[(int64_t)(c0 + j) * dn + k] : 0.f;
            cs[k * kDirCH + j] = pack2(v, v);
        }
        __syncthreads();
        if (C - c0 <= 16) direct_chunk<16>(xs, cs, dn, c0, C, best, arg);
        else direct_chunk<kDirCH>(xs, cs, dn, c0, C, best, arg);
    }
    const int n = n0 + 2 * threadIdx.x;
    if (n < N) P.labels[(int64_t)bh * N + n] = arg[0];
    if (n + 1 < N) P.labels[(int64_t)bh * N + n + 1] = arg[1];
}

static size_t direct_smem(int dn)
{
    return (size_t)((dn * (kDirRows / 2) + 3) & ~3) * 4 + (size_t)dn * kDirCH * 8;
}

// -------------------------------------------------------------- assign fix-up
// The tensor-core query assignment (kmeans_tc.cu) lists the rows whose best
// and second-best expanded-form scores lie within its fp32 error margin.
// Exact re-decision of the listed rows: fp64 direct-form distance to every
// centroid, lowest index on ties.  One CTA per listed row (grid-strided):
// warp w takes centroids w, w + 8, ..., its lanes split the dims, and eight
// centroids per step keep eight shuffle reductions in flight; the eight
// warps' winners then meet in shared memory.
constexpr int kFixWarps = 8;

__global__ void __launch_bounds__(kFixWarps * 32) km_fixup_kernel(FixBatch fb, int N, int D)
{
    __shared__ double wbest[kFixWarps];
    __shared__ int warg[kFixWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const KmProblem &P = fb.p[blockIdx.y];  // one problem (and its list) per grid row
    const int32_t *fix_list = fb.list[blockIdx.y];
    const int count = *fb.count[blockIdx.y];
    const int C = P.C, dn = P.dim_n;
    for (int w = blockIdx.x; w < count; w += gridDim.x) {
        const int gid = fix_list[w];
        const int bh = gid / N, n = gid % N;
        const __nv_bfloat16 *x = P.X + ((int64_t)bh * N + n) * D + P.dim_off;
        double xv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = lane + 32 * q < dn ? (double)__bfloat162float(x[lane + 32 * q]) : 0.0;
        const float *cent = P.cent + (int64_t)bh * C * dn;
        double best = INFINITY;
        int arg = C;
        constexpr int U = 8;
        for (int j0 = warp; j0 < C; j0 += U * kFixWarps) {
            double d[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                d[u] = 0.0;
                const int j = j0 + u * kFixWarps;
                if (j < C) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (lane + 32 * q < dn) {
                            const double t = xv[q] - (double)cent[(int64_t)j * dn + lane + 32 * q];
                            d[u] = fma(t, t, d[u]);
                        }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int u = 0; u < U; ++u) d[u] += __shfl_xor_sync(0xffffffffu, d[u], o);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + u * kFixWarps;  // ascending within the warp: ties keep the lowest index
                if (j < C && d[u] < best) {
                    best = d[u];
                    arg = j;
                }
            }
        }
        if (lane == 0) {
            wbest[warp] = best;
            warg[warp] = arg;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            double b = wbest[0];
            int a = warg[0];
            for (int i = 1; i < kFixWarps; ++i)
                if (wbest[i] < b || (wbest[i] == b && warg[i] < a)) {
                    b = wbest[i];
                    a = warg[i];
                }
            P.labels[(int64_t)bh * N + n] = a;
        }
        __syncthreads();
    }
}

// -------------------------------------------------------------- stable counting sort
// One warp per block of kSortBlk consecutive rows.
__global__ void km_hist_kernel(KmBatch b, int N, int nblk)
{
    extern __shared__ int hist[];
    const KmProblem &P = b.p[blockIdx.z];
    const int blk = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
    for (int c = lane; c < P.C; c += 32) hist[c] = 0;
    __syncwarp();
    const int32_t *lab = P.labels + (int64_t)bh * N;
    for (int i = lane; i < kSortBlk; i += 32) {
        const int n = blk * kSortBlk + i;
        if (n < N) atomicAdd(&hist[lab[n]], 1);
    }
    __syncwarp();
    int32_t *h = P.blockhist + (int64_t)bh * P.C * nblk;
    for (int c = lane; c < P.C; c += 32) h[(int64_t)c * nblk + blk] = hist[c];
}

// Exclusive scan over (cluster, block) -> stable output bases; cluster starts
// and sizes.  Three parallel steps per (head, problem): the sums of tiles of
// kScanTile counters, then every tile scans its counters from the sum of the
// tiles before it (so no CTA walks C x blocks counters alone), then the
// cluster starts and sizes.
constexpr int kScanThreads = 1024, kScanPer = 4, kScanTile = kScanThreads * kScanPer;
static_assert(kScanTile == kScanTileCounters, "scan tile size");

__global__ void __launch_bounds__(kScanThreads) km_scan_tiles_kernel(KmBatch b, int nblk)
{
    __shared__ int tmp[33];
    const KmProblem &P = b.p[blockIdx.z];
    const int bh = blockIdx.y;
    const int64_t total = (int64_t)P.C * nblk;
    const int64_t t0 = (int64_t)blockIdx.x * kScanTile;
    if (t0 >= total) return;
    const int32_t *h = P.blockhist + (int64_t)bh * total;
    int v = 0;
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
        const int64_t e = t0 + (int64_t)i * kScanThreads + threadIdx.x;
        v += e < total ? h[e] : 0;
    }
    int tot;
    block_excl_scan(v, tmp, tot);
    const int ntiles = (int)((total + kScanTile - 1) / kScanTile);
    if (threadIdx.x == 0) P.tilesum[(int64_t)bh * ntiles + blockIdx.x] = tot;
}

__global__ void __launch_bounds__(kScanThreads) km_scan_apply_kernel(KmBatch b, int nblk)
{
    __shared__ int tmp[33];
    const KmProblem &P = b.p[blockIdx.z];
    const int bh = blockIdx.y;
    const int64_t total = (int64_t)P.C * nblk;
    const int64_t t0 = (int64_t)blockIdx.x * kScanTile;
    if (t0 >= total) return;
    const int ntiles = (int)((total + kScanTile - 1) / kScanTile);
    const int32_t *ts = P.tilesum + (int64_t)bh * ntiles;
    int before = 0;
    for (int i = threadIdx.x; i < (int)blockIdx.x; i += kScanThreads) before += ts[i];
    int carry;
    block_excl_scan(before, tmp, carry);  // carry = sum of the tiles before this one
    int32_t *h = P.blockhist + (int64_t)bh * total;
    // thread-contiguous counters, so a thread's exclusive prefix is local
    const int64_t e0 = t0 + (int64_t)threadIdx.x * kScanPer;
    int v[kScanPer], s = 0;
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
        v[i] = e0 + i < total ? h[e0 + i] : 0;
        s += v[i];
    }
    int tot;
    int ex = carry + block_excl_scan(s, tmp, tot);
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
        if (e0 + i < total) h[e0 + i] = ex;
        ex += v[i];
    }
}

__global__ void km_starts_kernel(KmBatch b, int N, int nblk)
{
    const KmProblem &P = b.p[blockIdx.z];
    const int bh = blockIdx.y;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c > P.C) return;
    const int32_t *h = P.blockhist + (int64_t)bh * P.C * nblk;
    int32_t *start = P.start + (int64_t)bh * (P.C + 1);
    const int s0 = c < P.C ? h[(int64_t)c * nblk] : N;
    start[c] = s0;
    if (c < P.C) {
        const int s1 = c + 1 < P.C ? h[(int64_t)(c + 1) * nblk] : N;
        P.sizes[(int64_t)bh * P.C + c] = s1 - s0;
    }
}

// Rows of a block land at base[c][blk] + (rank among earlier rows of label c
// in the block); lanes see rows in ascending order, so the sort is stable.
__global__ void km_scatter_kernel(KmBatch b, int N, int nblk)
{
    extern __shared__ int run[];
    const KmProblem &P = b.p[blockIdx.z];
    const int blk = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
    const int32_t *h = P.blockhist + (int64_t)bh * P.C * nblk;
    for (int c = lane; c < P.C; c += 32) run[c] = h[(int64_t)c * nblk + blk];
    __syncwarp();
    const int32_t *lab = P.labels + (int64_t)bh * N;
    int32_t *perm = P.perm + (int64_t)bh * N;
    for (int r = 0; r < kSortBlk / 32; ++r) {
        const int n = blk * kSortBlk + r * 32 + lane;
        const bool valid = n < N;
        const int l = valid ? lab[n] : -1;
        const unsigned mask = __match_any_sync(0xffffffffu, l);
        const unsigned lower = mask & lanemask_lt();
        if (valid) perm[run[l] + __popc(lower)] = n;
        __syncwarp();
        if (valid && lower == 0) run[l] += __popc(mask);
        __syncwarp();
    }
}

// -------------------------------------------------------------- update
// One CTA per cluster: exact fixed-point sum of its members, mean in double,
// stored as fp32 with its squared norm.  Empty clusters keep their centroid.
__global__ void __launch_bounds__(1024) km_reduce_kernel(KmBatch b, int N, int D)
{
    __shared__ long long part[1024];
    const KmProblem &P = b.p[blockIdx.z];
    const int c = blockIdx.x, bh = blockIdx.y;
    if (c >= P.C) return;
    const int dn = P.dim_n;
    int colsP = 1;
    while (colsP < dn) colsP <<= 1;
    const int slices = 1024 / colsP;
    const int col = threadIdx.x % colsP, slice = threadIdx.x / colsP;
    const int32_t *start = P.start + (int64_t)bh * (P.C + 1);
    const int st = start[c], sz = start[c + 1] - st;
    const int S = fixed_shift(P.maxabs + bh, N);
    const double scale = ldexp(1.0, S);
    long long acc = 0;
    if (col < dn) {
        const int32_t *perm = P.perm + (int64_t)bh * N + st;
        const __nv_bfloat16 *X = P.X + (int64_t)bh * N * D + P.dim_off + col;
        // four members per step so their (perm -> row) load chains overlap
        int m = slice;
        for (; m + 3 * slices < sz; m += 4 * slices) {
            const int i0 = perm[m], i1 = perm[m + slices], i2 = perm[m + 2 * slices], i3 = perm[m + 3 * slices];
            const float x0 = __bfloat162float(X[(int64_t)i0 * D]), x1 = __bfloat162float(X[(int64_t)i1 * D]);
            const float x2 = __bfloat162float(X[(int64_t)i2 * D]), x3 = __bfloat162float(X[(int64_t)i3 * D]);
            acc += __double2ll_rn((double)x0 * scale) + __double2ll_rn((double)x1 * scale) +
                   __double2ll_rn((double)x2 * scale) + __double2ll_rn((double)x3 * scale);
        }
        for (; m < sz; m += slices) acc += __double2ll_rn((double)__bfloat162float(X[(int64_t)perm[m] * D]) * scale);
    }
    part[threadIdx.x] = acc;
    __syncthreads();
    float *cent = P.cent + ((int64_t)bh * P.C + c) * dn;
    if (slice == 0 && col < dn && sz > 0) {
        long long s = 0;
        for (int k = 0; k < slices; ++k) s += part[k * colsP + col];
        cent[col] = (float)((double)s / scale / (double)sz);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float s = 0.f;
        for (int k = 0; k < dn; ++k) s = fmaf(cent[k], cent[k], s);
        P.cn[(int64_t)bh * P.C + c] = s;
    }
}

// -------------------------------------------------------------- update (segmented)
// The same fixed-point sums, accumulated over the sorted member order in
// equal segments instead of one CTA per cluster, so a cluster of 7000 keys
// no longer runs as one long chain of dependent loads.  Each warp owns 128
// consecutive sorted positions; a row is read by ceil(dim_n/4) lanes with one
// 8-byte load each (several rows per warp step when dim_n is small), and a
// lane keeps int64 sums of its four columns until its rows cross into the next
// cluster, when it adds them to the cluster's sums with integer atomics.
// Integer addition is associative, so the totals (and the means) do not
// depend on the order in which segments arrive.  x * 2^S is exact in fp32
// (bf16 input, S in [0, 40]), so its rounding to an integer equals the fp64
// form of the per-cluster kernel above.
constexpr int kSegWarps = 8, kSegRows = 128, kSegUnroll = 16;

__global__ void __launch_bounds__(kSegWarps * 32, 3) km_accum_kernel(KmBatch b, int N, int D)
{
    __shared__ int32_t rows_sh[kSegWarps][kSegRows];
    const KmProblem &P = b.p[blockIdx.z];
    const int bh = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p0 = (blockIdx.x * kSegWarps + warp) * kSegRows;
    if (p0 >= N) return;
    const int p1 = min(N, p0 + kSegRows);
    const int dn = P.dim_n, C = P.C, quads = (dn + 3) >> 2;
    int lanes = 1;
    while (lanes < quads) lanes <<= 1;
    const int R = 32 / lanes, slot = lane / lanes, d0 = 4 * (lane % lanes);
    const int nv = d0 < dn ? min(4, dn - d0) : 0;
    const bool vec = nv == 4 && ((P.dim_off & 3) == 0);
    const int32_t *start = P.start + (int64_t)bh * (C + 1);
    const int32_t *perm = P.perm + (int64_t)bh * N;
    const __nv_bfloat16 *X = P.X + (int64_t)bh * N * D + P.dim_off + d0;
    unsigned long long *sums = P.sums + (int64_t)bh * C * dn + d0;
    const float scale = ldexpf(1.f, fixed_shift(P.maxabs + bh, N));
    // the warp's member rows, read once and coalesced
    int32_t *rows = rows_sh[warp];
    for (int t = lane; t < kSegRows; t += 32) rows[t] = p0 + t < p1 ? perm[p0 + t] : 0;
    __syncwarp();

    int p = p0 + slot;
    if (p >= p1) return;
    // cluster of position p: the last c with start[c] <= p (skips empty ones)
    int lo = 0, hi = C;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (start[mid] <= p) lo = mid;
        else hi = mid;
    }
    int cur = lo, nxt = start[cur + 1];
    long long acc[4] = {0, 0, 0, 0};
    bool any = false;
    for (; p < p1; p += kSegUnroll * R) {
        uint2 raw[kSegUnroll];
#pragma unroll
        for (int u = 0; u < kSegUnroll; ++u) {
            raw[u] = make_uint2(0u, 0u);
            if (p + u * R < p1) {
                const __nv_bfloat16 *x = X + (int64_t)rows[p + u * R - p0] * D;
                if (vec) {
                    raw[u] = *reinterpret_cast<const uint2 *>(x);
                } else if (nv > 0) {
                    const unsigned short *xs = reinterpret_cast<const unsigned short *>(x);
                    const uint32_t h0 = xs[0], h1 = nv > 1 ? xs[1] : 0u, h2 = nv > 2 ? xs[2] : 0u,
                                   h3 = nv > 3 ? xs[3] : 0u;
                    raw[u] = make_uint2(h0 | (h1 << 16), h2 | (h3 << 16));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kSegUnroll; ++u) {
            const int pu = p + u * R;
            if (pu < p1) {
                while (pu >= nxt) {
                    if (any)
                        for (int i = 0; i < nv; ++i) atomicAdd(sums + (int64_t)cur * dn + i, (unsigned long long)acc[i]);
                    acc[0] = acc[1] = acc[2] = acc[3] = 0;
                    any = false;
                    ++cur;
                    nxt = start[cur + 1];
                }
                const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw[u].x));
                const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw[u].y));
                acc[0] += __float2ll_rn(a.x * scale);
                acc[1] += __float2ll_rn(a.y * scale);
                acc[2] += __float2ll_rn(c.x * scale);
                acc[3] += __float2ll_rn(c.y * scale);
                any = true;
            }
        }
    }
    if (any)
        for (int i = 0; i < nv; ++i) atomicAdd(sums + (int64_t)cur * dn + i, (unsigned long long)acc[i]);
}

// Means from the segmented sums (same rounding as km_reduce_kernel), squared
// norms, and the sums cleared for the next update.
__global__ void __launch_bounds__(128) km_finalize_kernel(KmBatch b, int N)
{
    __shared__ float cs[128];
    const KmProblem &P = b.p[blockIdx.z];
    const int c = blockIdx.x, bh = blockIdx.y, d = threadIdx.x;
    if (c >= P.C) return;
    const int dn = P.dim_n;
    const int sz = P.sizes[(int64_t)bh * P.C + c];
    const double scale = ldexp(1.0, fixed_shift(P.maxabs + bh, N));
    unsigned long long *sums = P.sums + ((int64_t)bh * P.C + c) * dn;
    float *cent = P.cent + ((int64_t)bh * P.C + c) * dn;
    if (d < dn) {
        const long long s = (long long)sums[d];
        sums[d] = 0ull;
        if (sz > 0) cent[d] = (float)((double)s / scale / (double)sz);
        cs[d] = cent[d];
    }
    __syncthreads();
    if (d == 0) {
        float s = 0.f;
        for (int k = 0; k < dn; ++k) s = fmaf(cs[k], cs[k], s);
        P.cn[(int64_t)bh * P.C + c] = s;
    }
}

// -------------------------------------------------------------- launchers
static int max_C(const KmBatch &b)
{
    int m = 0;
    for (int i = 0; i < b.count; ++i) m = b.p[i].C > m ? b.p[i].C : m;
    return m;
}

static int max_dim(const KmBatch &b)
{
    int m = 0;
    for (int i = 0; i < b.count; ++i) m = b.p[i].dim_n > m ? b.p[i].dim_n : m;
    return m;
}

cudaError_t km_configure()
{
    cudaError_t e = cudaFuncSetAttribute(km_assign_direct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)direct_smem(128));
    return e;
}

void launch_km_init(const KmBatch &b, int BH, int N, int D, uint32_t seed, cudaStream_t st)
{
    km_init_kernel<<<dim3(max_C(b), BH, b.count), 128, 0, st>>>(b, N, D, seed);
    count_launches(1);
}

void launch_km_assign_direct(const KmBatch &b, int BH, int N, int D, cudaStream_t st)
{
    km_assign_direct_kernel<<<dim3((N + kDirRows - 1) / kDirRows, BH, b.count), kDirRows / 2,
                              direct_smem(max_dim(b)), st>>>(b, N, D);
    count_launches(1);
}

// One launch re-decides the listed rows of every problem of the batch.
void km_fixup_launch(const FixBatch &fb, int N, int D, cudaStream_t st)
{
    if (fb.n == 0) return;
    km_fixup_kernel<<<dim3(148 * 8 / fb.n, fb.n), kFixWarps * 32, 0, st>>>(fb, N, D);
    count_launches(1);
}

void launch_km_sort(const KmBatch &b, int BH, int N, cudaStream_t st)
{
    const int nblk = (N + kSortBlk - 1) / kSortBlk;
    const size_t smem = (size_t)max_C(b) * sizeof(int);
    km_hist_kernel<<<dim3(nblk, BH, b.count), 32, smem, st>>>(b, N, nblk);
    count_launches(1);
    const int ntiles = (int)(((int64_t)max_C(b) * nblk + kScanTile - 1) / kScanTile);
    km_scan_tiles_kernel<<<dim3(ntiles, BH, b.count), kScanThreads, 0, st>>>(b, nblk);
    km_scan_apply_kernel<<<dim3(ntiles, BH, b.count), kScanThreads, 0, st>>>(b, nblk);
    km_starts_kernel<<<dim3((max_C(b) + 256) / 256, BH, b.count), 256, 0, st>>>(b, N, nblk);
    count_launches(3);
    km_scatter_kernel<<<dim3(nblk, BH, b.count), 32, smem, st>>>(b, N, nblk);
    count_launches(1);
}

// With sums buffers (every problem of the batch has one): segmented
// accumulation + finalize; without: one CTA per cluster.
void launch_km_reduce(const KmBatch &b, int BH, int N, int D, cudaStream_t st)
{
    if (b.p[0].sums) {
        const int per_cta = kSegWarps * kSegRows;
        km_accum_kernel<<<dim3((N + per_cta - 1) / per_cta, BH, b.count), kSegWarps * 32, 0, st>>>(b, N, D);
        km_finalize_kernel<<<dim3(max_C(b), BH, b.count), 128, 0, st>>>(b, N);
        count_launches(2);
        return;
    }
    km_reduce_kernel<<<dim3(max_C(b), BH, b.count), 1024, 0, st>>>(b, N, D);
    count_launches(1);
}

}  // namespace scope
