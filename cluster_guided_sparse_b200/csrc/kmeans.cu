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

// -------------------------------------------------------------- assign (direct form)
// One thread per row; the CTA's rows are staged transposed in shared memory
// and centroids stream through in chunks of CH, transposed so one 16-byte
// broadcast load feeds four centroids.  d = sum_k (x_k - c_k)^2 in fp32: no
// cancellation, relative error <= (dim+2) * 2^-24 of the distance.
template <int CH>
__global__ void __launch_bounds__(128) km_assign_direct_kernel(KmBatch b, int N, int D)
{
    extern __shared__ __align__(16) float sm[];
    const KmProblem &P = b.p[blockIdx.z];
    const int bh = blockIdx.y;
    const int n0 = blockIdx.x * blockDim.x;
    if (n0 >= N) return;
    const int dn = P.dim_n, C = P.C, T = blockDim.x;
    float *xs = sm;            // [dn][T]
    float *cs = sm + dn * T;   // [dn][CH]
    for (int idx = threadIdx.x; idx < T * dn; idx += T) {
        const int r = idx / dn, k = idx % dn, n = n0 + r;
        xs[k * T + r] = n < N ? __bfloat162float(P.X[((int64_t)bh * N + n) * D + P.dim_off + k]) : 0.f;
    }
    float best = INFINITY;
    int arg = 0;
    const float *cent = P.cent + (int64_t)bh * C * dn;
    for (int c0 = 0; c0 < C; c0 += CH) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < CH * dn; idx += T) {
            const int j = idx / dn, k = idx % dn;
            cs[k * CH + j] = (c0 + j < C) ? cent[(int64_t)(c0 + j) * dn + k] : 0.f;
        }
        __syncthreads();
        float acc[CH];
#pragma unroll
        for (int j = 0; j < CH; ++j) acc[j] = 0.f;
        for (int k = 0; k < dn; ++k) {
            const float xv = xs[k * T + threadIdx.x];
            const float4 *c4 = reinterpret_cast<const float4 *>(cs + k * CH);
#pragma unroll
            for (int j4 = 0; j4 < CH / 4; ++j4) {
                const float4 c = c4[j4];
                float d;
                d = xv - c.x; acc[4 * j4 + 0] = fmaf(d, d, acc[4 * j4 + 0]);
                d = xv - c.y; acc[4 * j4 + 1] = fmaf(d, d, acc[4 * j4 + 1]);
                d = xv - c.z; acc[4 * j4 + 2] = fmaf(d, d, acc[4 * j4 + 2]);
                d = xv - c.w; acc[4 * j4 + 3] = fmaf(d, d, acc[4 * j4 + 3]);
            }
        }
#pragma unroll
        for (int j = 0; j < CH; ++j)
            if (c0 + j < C && acc[j] < best) {
                best = acc[j];
                arg = c0 + j;
            }
    }
    const int n = n0 + threadIdx.x;
    if (n < N) P.labels[(int64_t)bh * N + n] = arg;
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

// Exclusive scan over (cluster, block) -> stable output bases; cluster starts.
__global__ void __launch_bounds__(1024) km_scan_kernel(KmBatch b, int N, int nblk)
{
    __shared__ int tmp[33];
    const KmProblem &P = b.p[blockIdx.y];
    const int bh = blockIdx.x;
    const int64_t total = (int64_t)P.C * nblk;
    int32_t *h = P.blockhist + (int64_t)bh * total;
    int carry = 0;
    for (int64_t base = 0; base < total; base += blockDim.x) {
        const int64_t i = base + threadIdx.x;
        const int v = i < total ? h[i] : 0;
        int tot;
        const int ex = block_excl_scan(v, tmp, tot);
        if (i < total) h[i] = carry + ex;
        carry += tot;
    }
    __syncthreads();
    int32_t *start = P.start + (int64_t)bh * (P.C + 1);
    for (int c = threadIdx.x; c <= P.C; c += blockDim.x) start[c] = c < P.C ? h[(int64_t)c * nblk] : N;
    __syncthreads();
    for (int c = threadIdx.x; c < P.C; c += blockDim.x)
        P.sizes[(int64_t)bh * P.C + c] = start[c + 1] - start[c];
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
__global__ void __launch_bounds__(256) km_reduce_kernel(KmBatch b, int N, int D)
{
    __shared__ long long part[256];
    const KmProblem &P = b.p[blockIdx.z];
    const int c = blockIdx.x, bh = blockIdx.y;
    if (c >= P.C) return;
    const int dn = P.dim_n;
    int colsP = 1;
    while (colsP < dn) colsP <<= 1;
    const int slices = 256 / colsP;
    const int col = threadIdx.x % colsP, slice = threadIdx.x / colsP;
    const int32_t *start = P.start + (int64_t)bh * (P.C + 1);
    const int st = start[c], sz = start[c + 1] - st;
    const int S = fixed_shift(P.maxabs, N);
    const double scale = ldexp(1.0, S);
    long long acc = 0;
    if (col < dn) {
        const int32_t *perm = P.perm + (int64_t)bh * N + st;
        const __nv_bfloat16 *X = P.X + (int64_t)bh * N * D + P.dim_off + col;
        for (int m = slice; m < sz; m += slices)
            acc += __double2ll_rn((double)__bfloat162float(X[(int64_t)perm[m] * D]) * scale);
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
    return cudaFuncSetAttribute(km_assign_direct_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (128 + 32) * 128 * 4);
}

void launch_km_init(const KmBatch &b, int BH, int N, int D, uint32_t seed, cudaStream_t st)
{
    km_init_kernel<<<dim3(max_C(b), BH, b.count), 128, 0, st>>>(b, N, D, seed);
    count_launches(1);
}

void launch_km_assign_direct(const KmBatch &b, int BH, int N, int D, cudaStream_t st)
{
    const int dn = max_dim(b);
    const size_t smem = (size_t)(128 + 32) * dn * sizeof(float);
    km_assign_direct_kernel<32><<<dim3((N + 127) / 128, BH, b.count), 128, smem, st>>>(b, N, D);
    count_launches(1);
}

void launch_km_sort(const KmBatch &b, int BH, int N, cudaStream_t st)
{
    const int nblk = (N + kSortBlk - 1) / kSortBlk;
    const size_t smem = (size_t)max_C(b) * sizeof(int);
    km_hist_kernel<<<dim3(nblk, BH, b.count), 32, smem, st>>>(b, N, nblk);
    count_launches(1);
    km_scan_kernel<<<dim3(BH, b.count), 1024, 0, st>>>(b, N, nblk);
    count_launches(1);
    km_scatter_kernel<<<dim3(nblk, BH, b.count), 32, smem, st>>>(b, N, nblk);
    count_launches(1);
}

void launch_km_reduce(const KmBatch &b, int BH, int N, int D, cudaStream_t st)
{
    km_reduce_kernel<<<dim3(max_C(b), BH, b.count), 256, 0, st>>>(b, N, D);
    count_launches(1);
}

}  // namespace scope
