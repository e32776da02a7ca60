// Query k-means assignment on the 5th-generation tensor cores.  The labels
// are certified: they equal the argmin of exact arithmetic on the stored fp32
// centroids and bf16 rows (lowest index on ties).
//
// The assignment score e_j = ||c_j||^2 - 2 x.c_j needs x.c_j for every row
// and centroid: a dense contraction (N x d times d x C per head).  The rows x
// are bf16 (the stored post-RoPE queries, exact); each fp32 centroid is split
// into c = c_hi + c_lo with c_hi = bf16(c), c_lo = bf16(c - c_hi), so two bf16
// MMAs accumulating into the same fp32 TMEM columns give x.c.  Model of the
// accumulation: each bf16 x bf16 product is exact in fp32 (8 + 8 significant
// bits), and every one of the 2d additions into the accumulator (d hi
// products, then d lo products) may lose up to 2^-23 of the running
// magnitude (round to nearest, or truncation), which is bounded by
// sum_k |x_k| (|c_hi,k| + |c_lo,k|) <= |x| |c| (1 + 2^-8).  With the hi/lo
// representation error 2^-16 |x| |c| (c_lo holds c - c_hi to 8 bits), the
// computed x.c is within
//     (2d * 2^-23 * (1 + 2^-8) + 2^-16) * |x| * |c|
// of the exact one.  With R = max_j |c_j| and the fp32 ||c||^2 error
// (d+2) 2^-24 R^2,
//     B = 2 (2d 2^-23 (1 + 2^-8) + 2^-16) |x| R + (d + 2) 2^-24 R^2
// bounds the error of every e_j = ||c_j||^2 - 2 x.c_j; when the runner-up
// beats the best by more than 2B the label is certain, otherwise the row goes
// to the fp64 fix-up pass (km_fixup_kernel).
//
// One CTA = kMT tiles of 128 rows (M = 128 each; kMT = 1 below) sharing
// every centroid chunk the CTA loads.  Warps 0..4*kMT-1: argmin epilogue, one
// row per thread (warps 4t..4t+3 for tile t), reading the 128 x 128 score
// tile of a chunk from TMEM; warp 4*kMT: tcgen05.mma issuer and TMEM owner;
// warp 4*kMT+1: TMA producer (the row tiles once, then hi/lo centroid chunks
// of 128 through one stage).  Each tile's accumulator is double-buffered so
// chunk c+1's MMAs overlap chunk c's epilogue; with one tile, 96 KB of shared
// memory and 256 TMEM columns let two CTAs share an SM.  The epilogue keeps
// eight interleaved (best, arg, second) states so its compare chain is short.
#include "tcgen05.cuh"

namespace scope {

namespace {

using namespace tc;

// Row tiles per CTA.  Tiles of one CTA share every centroid chunk it loads;
// two tiles per CTA (one CTA per SM) halve the chunks' L2 traffic but measured
// slower than one tile per CTA with two CTAs per SM (query assignment 10.9 vs
// 10.0 ms per 720p call, key subspaces 8.0 vs 7.4 ms), so one tile it is.
constexpr int kMT = 1;
constexpr int kMinBlocks = kMT == 1 ? 2 : 1;
constexpr int kKT = 32 * (4 * kMT + 2);  // threads: 4 epilogue warps per tile + MMA warp + producer warp
constexpr int kMmaW = 4 * kMT, kProdW = 4 * kMT + 1;

struct KtArgs {
    KmProblem P;
    const float *xnorm2;
    int32_t *fix_list, *fix_count;
    int32_t *err;
    int N, D;
};

template <int D>
__global__ void __launch_bounds__(kKT, kMinBlocks)
    km_assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmHi,
                        const __grid_constant__ CUtensorMap tmLo, KtArgs a)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int TILE = 128 * D * 2;  // one 128-row bf16 tile
    unsigned char *sX = sm;                  // kMT row tiles
    unsigned char *sC = sm + kMT * TILE;     // [hi, lo]
    __shared__ uint64_t bar_x, bar_c_full[2], bar_c_empty[2], bar_acc_full[2], bar_acc_empty[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ float red[4];
    __shared__ __align__(16) float cn_sh[kMaxClusters];

    const KmProblem &P = a.P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, p0 = blockIdx.x * 128 * kMT;
    const int C = P.C, N = a.N;
    const int nchunks = (C + 127) / 128;
    const float *cn = P.cn + (int64_t)bh * C;

    if (threadIdx.x == 0) {
        mbar_init(&bar_x, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_c_full[i], 1);
            mbar_init(&bar_c_empty[i], 1);
            mbar_init(&bar_acc_full[i], 1);
            mbar_init(&bar_acc_empty[i], 128 * kMT);
        }
        abort_sh = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaW) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "n"(256 * kMT));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // R^2 = max_j ||c_j||^2 (epilogue warps)
    if (warp < 4) {
        float r2 = 0.f;
        for (int j = threadIdx.x; j < (C + 127) / 128 * 128; j += 128) {
            const float v = j < C ? cn[j] : 0.f;
            cn_sh[j] = j < C ? v : __int_as_float(0x7f800000);  // padding never wins
            r2 = fmaxf(r2, v);
        }
        r2 = warp_max(r2);
        if (lane == 0) red[warp] = r2;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int *abort_flag = &abort_sh;

    if (warp == kProdW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_expect_tx(&bar_x, kMT * TILE);
#pragma unroll
            for (int t = 0; t < kMT; ++t)
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_2d(smem_u32(sX) + t * TILE + cb * 128 * 128, &tmX, cb * 64, bh * N + p0 + t * 128, &bar_x);
            for (int c = 0; c < nchunks; ++c) {
                const int s = 0;
                if (c >= 1 && !mbar_wait(&bar_c_empty[0], (c - 1) & 1, abort_flag, a.err, 0x40)) break;
                mbar_expect_tx(&bar_c_full[s], 2 * TILE);
                const uint32_t dst = smem_u32(sC);
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb) {
                    tma_load_2d(dst + cb * 128 * 128, &tmHi, cb * 64, bh * C + c * 128, &bar_c_full[s]);
                    tma_load_2d(dst + TILE + cb * 128 * 128, &tmLo, cb * 64, bh * C + c * 128, &bar_c_full[s]);
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaW) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, false);
            bool ok = mbar_wait(&bar_x, 0, abort_flag, a.err, 0x41);
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c & 1;
                if (!mbar_wait(&bar_c_full[0], c & 1, abort_flag, a.err, 0x42)) break;
                if (c >= 2 && !mbar_wait(&bar_acc_empty[s], ((c >> 1) - 1) & 1, abort_flag, a.err, 0x43)) break;
                tc_fence_after();
                const uint32_t ca = smem_u32(sC);
#pragma unroll
                for (int t = 0; t < kMT; ++t) {
                    const uint32_t xa = smem_u32(sX) + t * TILE;
#pragma unroll
                    for (int half = 0; half < 2; ++half)
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t ko = (k >> 2) * (128 * 128) + (k & 3) * 32;
                            mma_ss(tmem + (t * 2 + s) * 128, sw128_desc(xa + ko, 16, 1024),
                                   sw128_desc(ca + half * TILE + ko, 16, 1024), idesc, (half > 0 || k > 0));
                        }
                }
                mma_commit(&bar_acc_full[s]);
                mma_commit(&bar_c_empty[0]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ argmin epilogue
        const int t = warp >> 2, wq = warp & 3;  // row tile; TMEM lane quarter (= sub-partition)
        const int row = wq * 32 + lane, n = p0 + t * 128 + row;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        float r2 = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        float B1[8], B2[8];
        int A1[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            B1[q] = INFINITY;
            B2[q] = INFINITY;
            A1[q] = 0;
        }
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            if (!mbar_wait(&bar_acc_full[s], (c >> 1) & 1, abort_flag, a.err, 0x44)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t r[128];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld32(tmem + lane_off + (t * 2 + s) * 128 + q * 32, r + q * 32);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bar_acc_empty[s]);
            const int c0 = c * 128;
            const float4 *cnc = reinterpret_cast<const float4 *>(cn_sh + c0);
#pragma unroll
            for (int j = 0; j < 128; ++j) {
                const int q = j & 7;
                const float4 c4 = cnc[j >> 2];
                const float cj = (j & 3) == 0 ? c4.x : (j & 3) == 1 ? c4.y : (j & 3) == 2 ? c4.z : c4.w;
                const float e = fmaf(-2.f, __uint_as_float(r[j]), cj);
                // branch-free best / second-best update; an equal score keeps the
                // earlier (lower) index and collapses the margin to zero
                B2[q] = fminf(B2[q], fmaxf(B1[q], e));
                A1[q] = e < B1[q] ? c0 + j : A1[q];
                B1[q] = fminf(B1[q], e);
            }
        }
        // merge the eight states; equal scores keep the lowest centroid index
        float b1 = B1[0], b2 = B2[0];
        int a1 = A1[0];
#pragma unroll
        for (int q = 1; q < 8; ++q) {
            if (B1[q] < b1 || (B1[q] == b1 && A1[q] < a1)) {
                b2 = fminf(b1, B2[q]);
                b1 = B1[q];
                a1 = A1[q];
            } else {
                b2 = fminf(b2, B1[q]);
            }
            b2 = fminf(b2, B2[q]);
        }
        if (ok && n < N) {
            const float xn = sqrtf(a.xnorm2[(int64_t)bh * N + n]);
            const float R = sqrtf(r2);
            const int dn = D;
            const float B = (2.f * (2.f * (float)dn * 1.1920929e-7f * 1.00390625f + 1.5258789e-5f) * xn * R +
                             (float)(dn + 2) * 5.9604645e-8f * r2) * 1.01f + 1e-30f;
            P.labels[(int64_t)bh * N + n] = a1;
            if (!(b2 - b1 > 2.f * B)) {
                const int slot = atomicAdd(a.fix_count, 1);
                a.fix_list[slot] = bh * N + n;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaW) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(256 * kMT));
    }
}

// c_hi = bf16(c), c_lo = bf16(c - c_hi) for every centroid element.
__global__ void split_hi_lo_kernel(const float *cent, __nv_bfloat16 *hi, __nv_bfloat16 *lo, int64_t n)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float c = cent[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(c);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(c - __bfloat162float(h));
}

// -------------------------------------------------------------- key subspaces
// Key-subspace assignment on the tensor cores.  The three subspaces'
// centroids form one block-diagonal matrix of at most 128 rows: centroid j of
// subspace s (column offset o_s) holds its values in the dims of s and zeros
// elsewhere, so one N = 128 chunk of MMAs over the whole rotated key row
// gives x.c_j for every centroid of every subspace (the zero products are
// exact and leave the accumulator unchanged).  The certificate is the query
// kernel's, per subspace: width d_s, the row's block norm |x_s| (from the
// RoPE pass) and the subspace's centroid radius R_s.  Rows inside a
// subspace's margin go to that subspace's fp64 fix-up list.
struct KkArgs {
    KmProblem P[3];
    const float4 *xsub2;          // [BH][N] squared norms of each row's t, h, w blocks
    int32_t *fix_list[3], *fix_count[3];
    int32_t *err;
    int N, off1, off2, ncols;     // column offsets of the h and w centroids; used columns
};

// A8: the subspace boundaries and the used columns are multiples of 8, so
// only every eighth column can close a subspace or end the row.
template <int D, bool A8>
__global__ void __launch_bounds__(kKT, kMinBlocks)
    km_assign_keys_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmHi,
                             const __grid_constant__ CUtensorMap tmLo, KkArgs a)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int TILE = 128 * D * 2;
    unsigned char *sX = sm;               // kMT row tiles
    unsigned char *sC = sm + kMT * TILE;  // [hi, lo]
    __shared__ uint64_t bar_x, bar_c, bar_acc;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ float red[3][4];
    __shared__ __align__(16) float cn_sh[128];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, p0 = blockIdx.x * 128 * kMT, N = a.N;
    if (threadIdx.x == 0) {
        mbar_init(&bar_x, 1);
        mbar_init(&bar_c, 1);
        mbar_init(&bar_acc, 1);
        abort_sh = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaW) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                     "n"(128 * kMT));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (warp < 4) {
        // column j -> ||c_j||^2 of its subspace's centroid (+inf on padding); R_s^2 per subspace
        const int j = threadIdx.x;
        const int s = j < a.off1 ? 0 : (j < a.off2 ? 1 : 2);
        const int o = s == 0 ? 0 : (s == 1 ? a.off1 : a.off2);
        const bool used = j < a.ncols;
        const float v = used ? a.P[s].cn[(int64_t)bh * a.P[s].C + (j - o)] : 0.f;
        cn_sh[j] = used ? v : __int_as_float(0x7f800000);
        float r[3];
#pragma unroll
        for (int q = 0; q < 3; ++q) r[q] = warp_max(used && s == q ? v : 0.f);
        if (lane == 0)
            for (int q = 0; q < 3; ++q) red[q][warp] = r[q];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int *abort_flag = &abort_sh;

    if (warp == kProdW) {
        if (lane == 0) {
            mbar_expect_tx(&bar_x, kMT * TILE);
#pragma unroll
            for (int t = 0; t < kMT; ++t)
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_2d(smem_u32(sX) + t * TILE + cb * 128 * 128, &tmX, cb * 64, bh * N + p0 + t * 128, &bar_x);
            mbar_expect_tx(&bar_c, 2 * TILE);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
                tma_load_2d(smem_u32(sC) + cb * 128 * 128, &tmHi, cb * 64, bh * 128, &bar_c);
                tma_load_2d(smem_u32(sC) + TILE + cb * 128 * 128, &tmLo, cb * 64, bh * 128, &bar_c);
            }
        }
        __syncwarp();
    } else if (warp == kMmaW) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, false);
            const uint32_t ca = smem_u32(sC);
            if (mbar_wait(&bar_x, 0, abort_flag, a.err, 0x48) && mbar_wait(&bar_c, 0, abort_flag, a.err, 0x49)) {
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < kMT; ++t) {
                    const uint32_t xa = smem_u32(sX) + t * TILE;
#pragma unroll
                    for (int half = 0; half < 2; ++half)
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t ko = (k >> 2) * (128 * 128) + (k & 3) * 32;
                            mma_ss(tmem + t * 128, sw128_desc(xa + ko, 16, 1024),
                                   sw128_desc(ca + half * TILE + ko, 16, 1024), idesc, (half > 0 || k > 0));
                        }
                }
                mma_commit(&bar_acc);
            }
        }
        __syncwarp();
    } else {
        const int t = warp >> 2, wq = warp & 3;  // row tile; TMEM lane quarter (= sub-partition)
        const int row = wq * 32 + lane, n = p0 + t * 128 + row;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        if (mbar_wait(&bar_acc, 0, abort_flag, a.err, 0x4A)) {
            tc_fence_after();
            uint32_t r[128];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld32(tmem + lane_off + t * 128 + q * 32, r + q * 32);
            tmem_wait_ld();
            // one best / second-best tracker, closed at each subspace's first column
            const float INF = __int_as_float(0x7f800000);
            float B1 = INF, B2 = INF, b1[3], b2[3];
            int A1 = 0, a1[3];
            b1[0] = b1[1] = b1[2] = INF;
            b2[0] = b2[1] = b2[2] = INF;
            a1[0] = a1[1] = a1[2] = 0;
#pragma unroll
            for (int j = 0; j < 128; ++j) {
                if (A8 && (j & 7) == 0 && j >= a.ncols) break;  // padding columns: +inf
                if (!A8 || (j & 7) == 0) {
                    if (j == a.off1) {
                        b1[0] = B1; b2[0] = B2; a1[0] = A1;
                        B1 = B2 = INF;
                    }
                    if (j == a.off2) {
                        b1[1] = B1; b2[1] = B2; a1[1] = A1;
                        B1 = B2 = INF;
                    }
                }
                const float e = fmaf(-2.f, __uint_as_float(r[j]), cn_sh[j]);
                B2 = fminf(B2, fmaxf(B1, e));  // an equal score keeps the lower index and a zero margin
                A1 = e < B1 ? j : A1;
                B1 = fminf(B1, e);
            }
            b1[2] = B1; b2[2] = B2; a1[2] = A1;
            if (n < N) {
                const float4 xs = a.xsub2[(int64_t)bh * N + n];
                const float xs2[3] = {xs.x, xs.y, xs.z};
                const int off[3] = {0, a.off1, a.off2};
#pragma unroll
                for (int s = 0; s < 3; ++s) {
                    const KmProblem &P = a.P[s];
                    const float r2 = fmaxf(fmaxf(red[s][0], red[s][1]), fmaxf(red[s][2], red[s][3]));
                    const float xn = sqrtf(xs2[s]), R = sqrtf(r2);
                    const float dn = (float)P.dim_n;
                    const float B = (2.f * (2.f * dn * 1.1920929e-7f * 1.00390625f + 1.5258789e-5f) * xn * R +
                                     (dn + 2.f) * 5.9604645e-8f * r2) * 1.01f + 1e-30f;
                    P.labels[(int64_t)bh * N + n] = a1[s] - off[s];
                    if (P.C > 1 && !(b2[s] - b1[s] > 2.f * B)) {
                        const int slot = atomicAdd(a.fix_count[s], 1);
                        a.fix_list[s][slot] = bh * N + n;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaW) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(128 * kMT));
    }
}

// hi / lo halves of the block-diagonal key-centroid matrix [BH][128][D]
__global__ void keys_split_kernel(KkArgs a, __nv_bfloat16 *hi, __nv_bfloat16 *lo, int D, int64_t total)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= total) return;
    const int d = (int)(i % D), j = (int)((i / D) % 128);
    const int64_t bh = i / ((int64_t)D * 128);
    float c = 0.f;
    if (j < a.ncols) {
        const int s = j < a.off1 ? 0 : (j < a.off2 ? 1 : 2);
        const int o = s == 0 ? 0 : (s == 1 ? a.off1 : a.off2);
        const KmProblem &P = a.P[s];
        if (d >= P.dim_off && d < P.dim_off + P.dim_n)
            c = P.cent[((int64_t)bh * P.C + (j - o)) * P.dim_n + (d - P.dim_off)];
    }
    const __nv_bfloat16 h = __float2bfloat16_rn(c);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(c - __bfloat162float(h));
}

}  // namespace



cudaError_t km_tc_configure()
{
    cudaError_t e = cudaFuncSetAttribute(km_assign_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)((kMT + 2) * 128 * 128 * 2 + 1024));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(km_assign_keys_tc_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (kMT + 2) * 128 * 128 * 2 + 1024);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(km_assign_keys_tc_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (kMT + 2) * 128 * 64 * 2 + 1024);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(km_assign_keys_tc_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)((kMT + 2) * 128 * 128 * 2 + 1024));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(km_assign_keys_tc_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)((kMT + 2) * 128 * 64 * 2 + 1024));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(km_assign_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)((kMT + 2) * 128 * 64 * 2 + 1024));
}

// Tensor maps for the rows and the hi/lo centroid tables; false if encoding
// failed.  The rows inside the margin are left in fix_list for km_fixup_launch.
bool launch_km_assign_tc(const KmProblem &P, __nv_bfloat16 *chi, __nv_bfloat16 *clo, int BH, int N, int D,
                         const float *xnorm2, int32_t *fix_list, int32_t *fix_count, int32_t *err, cudaStream_t st)
{
    const int64_t nc = (int64_t)BH * P.C * D;
    split_hi_lo_kernel<<<(unsigned)((nc + 255) / 256), 256, 0, st>>>(P.cent, chi, clo, nc);
    count_launches(1);
    CUtensorMap tmX, tmHi, tmLo;
    if (!rows_tensor_map(&tmX, P.X, (uint64_t)BH * N, D, 128) ||
        !rows_tensor_map(&tmHi, chi, (uint64_t)BH * P.C, D, 128) ||
        !rows_tensor_map(&tmLo, clo, (uint64_t)BH * P.C, D, 128))
        return false;
    cudaMemsetAsync(fix_count, 0, sizeof(int32_t), st);
    KtArgs a;
    a.P = P;
    a.xnorm2 = xnorm2;
    a.fix_list = fix_list;
    a.fix_count = fix_count;
    a.err = err;
    a.N = N;
    a.D = D;
    const dim3 grid((N + 128 * kMT - 1) / (128 * kMT), BH);
    if (D == 128)
        km_assign_tc_kernel<128><<<grid, kKT, (kMT + 2) * 128 * 128 * 2 + 1024, st>>>(tmX, tmHi, tmLo, a);
    else
        km_assign_tc_kernel<64><<<grid, kKT, (kMT + 2) * 128 * 64 * 2 + 1024, st>>>(tmX, tmHi, tmLo, a);
    count_launches(1);
    return true;
}

}  // namespace scope

namespace scope {

// Key-subspace assignment of the three problems P[0..2] on the tensor cores
// (needs sum of their clusters <= 128); false if a tensor map failed.  The
// rows inside a subspace's margin are left in its list for km_fixup_launch.
bool launch_km_assign_keys_tc(const KmProblem *P, __nv_bfloat16 *chi, __nv_bfloat16 *clo, int BH, int N, int D,
                              const float4 *xsub2, int32_t *fix_base, int32_t *err, cudaStream_t st)
{
    KkArgs a;
    for (int s = 0; s < 3; ++s) a.P[s] = P[s];
    a.xsub2 = xsub2;
    // fix_base: [3][4 + BH*N]: a counter (padded to 16 bytes) then the list, per subspace
    for (int s = 0; s < 3; ++s) {
        a.fix_count[s] = fix_base + (int64_t)s * (4 + (int64_t)BH * N);
        a.fix_list[s] = a.fix_count[s] + 4;
    }
    a.err = err;
    a.N = N;
    a.off1 = P[0].C;
    a.off2 = P[0].C + P[1].C;
    a.ncols = P[0].C + P[1].C + P[2].C;
    const int64_t total = (int64_t)BH * 128 * D;
    keys_split_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(a, chi, clo, D, total);
    count_launches(1);
    CUtensorMap tmX, tmHi, tmLo;
    if (!rows_tensor_map(&tmX, P[0].X, (uint64_t)BH * N, D, 128) || !rows_tensor_map(&tmHi, chi, (uint64_t)BH * 128, D, 128) ||
        !rows_tensor_map(&tmLo, clo, (uint64_t)BH * 128, D, 128))
        return false;
    for (int s = 0; s < 3; ++s) cudaMemsetAsync(a.fix_count[s], 0, sizeof(int32_t), st);
    const dim3 grid((N + 128 * kMT - 1) / (128 * kMT), BH);
    const bool a8 = a.off1 % 8 == 0 && a.off2 % 8 == 0 && a.ncols % 8 == 0;
    const size_t sm = (size_t)(kMT + 2) * 128 * D * 2 + 1024;
    if (D == 128 && a8) km_assign_keys_tc_kernel<128, true><<<grid, kKT, sm, st>>>(tmX, tmHi, tmLo, a);
    else if (D == 128) km_assign_keys_tc_kernel<128, false><<<grid, kKT, sm, st>>>(tmX, tmHi, tmLo, a);
    else if (a8) km_assign_keys_tc_kernel<64, true><<<grid, kKT, sm, st>>>(tmX, tmHi, tmLo, a);
    else km_assign_keys_tc_kernel<64, false><<<grid, kKT, sm, st>>>(tmX, tmHi, tmLo, a);
    count_launches(1);
    return true;
}

}  // namespace scope
