// Query k-means assignment on the 5th-generation tensor cores.  The labels
// are certified: they equal the argmin of exact arithmetic on the stored fp32
// centroids and bf16 rows (lowest index on ties).
//
// The assignment score e_j = ||c_j||^2 - 2 x.c_j needs x.c_j for every row
// and centroid: a dense contraction (N x d times d x C per head).  The rows x
// are bf16 (the stored post-RoPE queries, exact); each fp32 centroid is split
// into c = c_hi + c_lo with c_hi = bf16(c), c_lo = bf16(c - c_hi), so two bf16
// MMAs with fp32 accumulation give x.c to within
//     (d * 2^-23 + 2^-16) * |x| * |c|
// (fp32 accumulation even if it truncates, plus the hi/lo representation
// error).  With R = max_j |c_j| and the fp32 ||c||^2 error (d+2) 2^-24 R^2,
//     B = 2 (d 2^-23 + 2^-16) |x| R + (d + 2) 2^-24 R^2
// bounds the error of every e_j; when the runner-up beats the best by more
// than 2B the label is certain, otherwise the row goes to the fp64 fix-up
// pass (km_fixup_kernel), exactly as for the fp32 kernel.
//
// One CTA = 128 rows (one M=128 tile).  Warps 0-3: argmin epilogue, one row
// per thread, reading the 128 x 128 score tile of a centroid chunk from TMEM;
// warp 4: tcgen05.mma issuer and TMEM owner; warp 5: TMA producer (the row
// tile once, then hi/lo centroid chunks of 128 through one stage).  The TMEM
// accumulator is double-buffered so chunk c+1's MMAs overlap chunk c's
// epilogue; 96 KB of shared memory and 256 TMEM columns let two CTAs share an
// SM and hide each other's load latency.  The epilogue keeps eight
// interleaved (best, arg, second) states so its compare chain is short.
#include "tcgen05.cuh"

namespace scope {

namespace {

using namespace tc;

constexpr int kKT = 192;  // threads: 4 epilogue warps + MMA warp + producer warp

struct KtArgs {
    KmProblem P;
    const float *xnorm2;
    int32_t *fix_list, *fix_count;
    int32_t *err;
    int N, D;
};

template <int D>
__global__ void __launch_bounds__(kKT, 2)
    km_assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmHi,
                        const __grid_constant__ CUtensorMap tmLo, KtArgs a)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int TILE = 128 * D * 2;  // one 128-row bf16 tile
    unsigned char *sX = sm;
    unsigned char *sC = sm + TILE;     // [hi, lo]
    __shared__ uint64_t bar_x, bar_c_full[2], bar_c_empty[2], bar_acc_full[2], bar_acc_empty[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ float red[4];
    __shared__ __align__(16) float cn_sh[kMaxClusters];

    const KmProblem &P = a.P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, p0 = blockIdx.x * 128;
    const int C = P.C, N = a.N;
    const int nchunks = (C + 127) / 128;
    const float *cn = P.cn + (int64_t)bh * C;

    if (threadIdx.x == 0) {
        mbar_init(&bar_x, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_c_full[i], 1);
            mbar_init(&bar_c_empty[i], 1);
            mbar_init(&bar_acc_full[i], 1);
            mbar_init(&bar_acc_empty[i], 128);
        }
        abort_sh = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 4) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(smem_u32(&tmem_base_sh)));
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

    if (warp == 5) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_expect_tx(&bar_x, TILE);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb)
                tma_load_2d(smem_u32(sX) + cb * 128 * 128, &tmX, cb * 64, bh * N + p0, &bar_x);
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
    } else if (warp == 4) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, false);
            const uint32_t xa = smem_u32(sX);
            bool ok = mbar_wait(&bar_x, 0, abort_flag, a.err, 0x41);
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c & 1;
                if (!mbar_wait(&bar_c_full[0], c & 1, abort_flag, a.err, 0x42)) break;
                if (c >= 2 && !mbar_wait(&bar_acc_empty[s], ((c >> 1) - 1) & 1, abort_flag, a.err, 0x43)) break;
                tc_fence_after();
                const uint32_t ca = smem_u32(sC);
#pragma unroll
                for (int half = 0; half < 2; ++half)
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t ko = (k >> 2) * (128 * 128) + (k & 3) * 32;
                        mma_ss(tmem + s * 128, sw128_desc(xa + ko, 16, 1024),
                               sw128_desc(ca + half * TILE + ko, 16, 1024), idesc, (half > 0 || k > 0));
                    }
                mma_commit(&bar_acc_full[s]);
                mma_commit(&bar_c_empty[0]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ argmin epilogue
        const int row = warp * 32 + lane, n = p0 + row;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
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
            for (int q = 0; q < 4; ++q) tmem_ld32(tmem + lane_off + s * 128 + q * 32, r + q * 32);
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
            const float B = (2.f * ((float)dn * 1.1920929e-7f + 1.5258789e-5f) * xn * R +
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
    if (warp == 4) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem));
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

}  // namespace

void km_fixup_launch(const KmProblem &P, int BH, int N, int D, const int32_t *fix_list, const int32_t *fix_count,
                     cudaStream_t st);

cudaError_t km_tc_configure()
{
    cudaError_t e = cudaFuncSetAttribute(km_assign_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(3 * 128 * 128 * 2 + 1024));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(km_assign_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(3 * 128 * 64 * 2 + 1024));
}

// Tensor maps for the rows and the hi/lo centroid tables; false if encoding failed.
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
    const dim3 grid((N + 127) / 128, BH);
    if (D == 128)
        km_assign_tc_kernel<128><<<grid, kKT, 3 * 128 * 128 * 2 + 1024, st>>>(tmX, tmHi, tmLo, a);
    else
        km_assign_tc_kernel<64><<<grid, kKT, 3 * 128 * 64 * 2 + 1024, st>>>(tmX, tmHi, tmLo, a);
    count_launches(1);
    km_fixup_launch(P, BH, N, D, fix_list, fix_count, st);
    return true;
}

}  // namespace scope
