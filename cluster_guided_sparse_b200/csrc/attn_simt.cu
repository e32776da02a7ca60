// Step 5 of SCOPE (abstract: "sparse attention is then computed over the
// selected original keys and values"), plain SIMT form: one warp per query,
// online softmax over the query's cluster list.  It is the simple,
// obviously-correct double of the tensor-core kernel (same tile table, same
// list layout) and serves shapes the tensor-core kernel does not take.
#include "common.cuh"

namespace scope {

// Q-tile table of one head: for every non-empty cluster c, ceil(|c| / kTQ)
// entries (c, tile), clusters in index order.
__global__ void __launch_bounds__(1024) tiles_kernel(const int32_t *sizes, int2 *tiles, int32_t *ntiles, int Cq,
                                                     int max_tiles)
{
    __shared__ int tmp[33];
    const int bh = blockIdx.x;
    int carry = 0;
    for (int base = 0; base < Cq; base += blockDim.x) {
        const int c = base + threadIdx.x;
        const int sz = c < Cq ? sizes[(int64_t)bh * Cq + c] : 0;
        const int nt = (sz + kTQ - 1) / kTQ;
        int tot;
        const int ex = block_excl_scan(nt, tmp, tot);
        for (int t = 0; t < nt; ++t) tiles[(int64_t)bh * max_tiles + carry + ex + t] = make_int2(c, t);
        carry += tot;
    }
    if (threadIdx.x == 0) ntiles[bh] = carry;
}

template <typename TV, int DPL>
__global__ void __launch_bounds__(128) attn_simt_kernel(
    const __nv_bfloat16 *__restrict__ qr, const __nv_bfloat16 *__restrict__ kr, const TV *__restrict__ v,
    __nv_bfloat16 *__restrict__ o, const int2 *__restrict__ tiles, const int32_t *__restrict__ ntiles,
    int max_tiles, const int32_t *__restrict__ perm, const int32_t *__restrict__ start,
    const long long *__restrict__ offsets, const int32_t *__restrict__ indices, const int32_t *__restrict__ n_c,
    int N, int Cq, float scale)
{
    constexpr int D = DPL * 32;
    const int bh = blockIdx.y;
    int c = 0, t = blockIdx.x;
    if (tiles) {
        if (blockIdx.x >= ntiles[bh]) return;
        const int2 e = tiles[(int64_t)bh * max_tiles + blockIdx.x];
        c = e.x;
        t = e.y;
    }
    const int cstart = start ? start[(int64_t)bh * (Cq + 1) + c] : 0;
    const int csize = start ? start[(int64_t)bh * (Cq + 1) + c + 1] - cstart : N;
    const int q0 = t * kTQ;
    if (q0 >= csize) return;
    const int nq = min(kTQ, csize - q0);
    const long long loff = indices ? offsets[(int64_t)bh * Cq + c] : 0;
    const int nk = indices ? n_c[(int64_t)bh * Cq + c] : N;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int64_t base = (int64_t)bh * N;
    for (int i = w; i < nq; i += nw) {
        const int tok = perm ? perm[base + cstart + q0 + i] : cstart + q0 + i;
        float q[DPL], acc[DPL];
#pragma unroll
        for (int d = 0; d < DPL; ++d) {
            q[d] = __bfloat162float(qr[(base + tok) * D + lane * DPL + d]) * scale;
            acc[d] = 0.f;
        }
        float m = -INFINITY, l = 0.f;
        for (int t2 = 0; t2 < nk; ++t2) {
            const int j = indices ? indices[loff + t2] : t2;
            const __nv_bfloat16 *kj = kr + (base + j) * D + lane * DPL;
            float s = 0.f;
#pragma unroll
            for (int d = 0; d < DPL; ++d) s = fmaf(q[d], __bfloat162float(kj[d]), s);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            const float mn = fmaxf(m, s);
            const float alpha = __expf(m - mn), p = __expf(s - mn);
            l = l * alpha + p;
            const TV *vj = v + (base + j) * D + lane * DPL;
#pragma unroll
            for (int d = 0; d < DPL; ++d) acc[d] = acc[d] * alpha + p * (float)vj[d];
            m = mn;
        }
        const float inv = 1.f / l;
#pragma unroll
        for (int d = 0; d < DPL; ++d) o[(base + tok) * D + lane * DPL + d] = __float2bfloat16_rn(acc[d] * inv);
    }
}

void launch_tiles(const int32_t *sizes, int2 *tiles, int32_t *ntiles, int BH, int Cq, int max_tiles,
                  cudaStream_t st)
{
    tiles_kernel<<<BH, 1024, 0, st>>>(sizes, tiles, ntiles, Cq, max_tiles);
    count_launches(1);
}

void launch_attn_simt(const __nv_bfloat16 *qr, const __nv_bfloat16 *kr, const __nv_bfloat16 *v,
                      __nv_bfloat16 *o, const int2 *tiles, const int32_t *ntiles, int max_tiles,
                      const int32_t *perm, const int32_t *start, const long long *offsets, const int32_t *indices,
                      const int32_t *n_c, int BH, int N, int D, int Cq, cudaStream_t st)
{
    const float scale = 1.0f / sqrtf((float)D);
    const int gx = tiles ? max_tiles : (N + kTQ - 1) / kTQ;
    const dim3 grid(gx, BH);
    if (D == 128)
        attn_simt_kernel<__nv_bfloat16, 4><<<grid, 128, 0, st>>>(qr, kr, v, o, tiles, ntiles, max_tiles, perm, start,
                                                                 offsets, indices, n_c, N, Cq, scale);
    else
        attn_simt_kernel<__nv_bfloat16, 2><<<grid, 128, 0, st>>>(qr, kr, v, o, tiles, ntiles, max_tiles, perm, start,
                                                                 offsets, indices, n_c, N, Cq, scale);
    count_launches(1);
}

}  // namespace scope
