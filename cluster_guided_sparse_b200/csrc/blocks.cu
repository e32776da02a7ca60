// VMoBA block-granular key selection ("VMoBA: Mixture-of-Block Attention for
// Video Diffusion Models", abstract: a layer-wise recurrent 1D-2D-3D block
// partition, and threshold selection of blocks by cumulative similarity).
//
// In block mode the key-subspace clustering of SCOPE is replaced by a fixed
// partition of the token grid: every key's "code" is its block, and every
// block's "centroid" is the mean of its rotated keys.  The rest of the plan
// is SCOPE's machinery unchanged: the lookup table then holds q_c . kbar_b,
// the code-triple items are the blocks (weighted by their sizes), and the
// Top-p select keeps whole blocks (every key tied at the cut score).
//
// Readings: kind 1 = runs of bt*bh*bw consecutive tokens in raster order;
// kind 2 = bh x bw tiles inside each frame; kind 3 = bt x bh x bw cubes;
// ragged edge blocks; blocks numbered in raster order of their corners.
#include "common.cuh"

namespace scope {

namespace {

struct BlockGeom {
    int T, Hh, W, kind, bt, bh, bw, nbt, nbh, nbw;
    __device__ __forceinline__ int id_of(int n) const
    {
        if (kind == 1) return n / (bt * bh * bw);
        const int t = n / (Hh * W), y = (n / W) % Hh, x = n % W;
        const int tb = kind == 2 ? t : t / bt;
        return (tb * nbh + y / bh) * nbw + x / bw;
    }
};

// codes[0][bh][n] = block of key n; the other two code planes are zero
__global__ void block_codes_kernel(BlockGeom g, int32_t *codes, int N, int64_t BHN)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= BHN) return;
    codes[i] = g.id_of((int)(i % N));
    codes[BHN + i] = 0;
    codes[2 * BHN + i] = 0;
}

// Mean rotated key of every block, one CTA per (block, head), one thread per
// dim; members are visited in ascending token order, summed in fp32.  Also
// the block sizes and squared norms of the means.
__global__ void block_means_kernel(BlockGeom g, const __nv_bfloat16 *kr, float *cent, float *cn, int32_t *sizes,
                                   int N, int D, int Nb)
{
    __shared__ float part[4];
    const int b = blockIdx.x, bh = blockIdx.y, d = threadIdx.x;
    int t0, t1, y0, y1, x0, x1;
    int64_t n0 = 0, n1 = 0;
    if (g.kind == 1) {
        const int len = g.bt * g.bh * g.bw;
        n0 = (int64_t)b * len;
        n1 = min((int64_t)N, n0 + len);
        t0 = t1 = y0 = y1 = x0 = x1 = 0;
    } else {
        const int bx = b % g.nbw, by = (b / g.nbw) % g.nbh, tb = b / (g.nbw * g.nbh);
        t0 = g.kind == 2 ? tb : tb * g.bt;
        t1 = g.kind == 2 ? tb + 1 : min(g.T, t0 + g.bt);
        y0 = by * g.bh;
        y1 = min(g.Hh, y0 + g.bh);
        x0 = bx * g.bw;
        x1 = min(g.W, x0 + g.bw);
    }
    const __nv_bfloat16 *K = kr + (int64_t)bh * N * D + d;
    float s = 0.f;
    int cnt = 0;
    if (g.kind == 1) {
        for (int64_t n = n0; n < n1; ++n) s += __bfloat162float(K[n * D]);
        cnt = (int)(n1 - n0);
    } else {
        for (int t = t0; t < t1; ++t)
            for (int y = y0; y < y1; ++y)
                for (int x = x0; x < x1; ++x) {
                    s += __bfloat162float(K[((int64_t)(t * g.Hh + y) * g.W + x) * D]);
                    ++cnt;
                }
    }
    const float m = cnt > 0 ? s / (float)cnt : 0.f;
    cent[((int64_t)bh * Nb + b) * D + d] = m;
    float q = m * m;
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if ((d & 31) == 0) part[d >> 5] = q;
    __syncthreads();
    if (d == 0) {
        float tot = 0.f;
        for (int w = 0; w < D / 32; ++w) tot += part[w];
        cn[(int64_t)bh * Nb + b] = tot;
        sizes[(int64_t)bh * Nb + b] = cnt;
    }
}

}  // namespace

int block_count(int T, int Hh, int W, int kind, int bt, int bh, int bw)
{
    if (kind == 1) {
        const int64_t len = (int64_t)bt * bh * bw;
        return (int)(((int64_t)T * Hh * W + len - 1) / len);
    }
    const int nbt = kind == 2 ? T : (T + bt - 1) / bt;
    return nbt * ((Hh + bh - 1) / bh) * ((W + bw - 1) / bw);
}

void launch_blocks(int T, int Hh, int W, int kind, int bt, int bh, int bw, const __nv_bfloat16 *kr, int32_t *codes,
                   float *cent, float *cn, int32_t *sizes, int BH, int N, int D, cudaStream_t st)
{
    BlockGeom g;
    g.T = T;
    g.Hh = Hh;
    g.W = W;
    g.kind = kind;
    g.bt = bt;
    g.bh = bh;
    g.bw = bw;
    g.nbt = kind == 2 ? T : (T + bt - 1) / bt;
    g.nbh = (Hh + bh - 1) / bh;
    g.nbw = (W + bw - 1) / bw;
    const int Nb = block_count(T, Hh, W, kind, bt, bh, bw);
    const int64_t BHN = (int64_t)BH * N;
    block_codes_kernel<<<(unsigned)((BHN + 255) / 256), 256, 0, st>>>(g, codes, N, BHN);
    block_means_kernel<<<dim3(Nb, BH), D, 0, st>>>(g, kr, cent, cn, sizes, N, D, Nb);
    count_launches(2);
}

}  // namespace scope
