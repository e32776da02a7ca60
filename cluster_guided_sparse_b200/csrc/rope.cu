// Step 1 of SCOPE (abstract: "post-RoPE keys", "3D-RoPE-aligned key subspace
// clustering"): rotary embedding on the (t, h, w) latent grid, written once
// as bf16 post-RoPE Q/K that every later stage reads.
//
// Readings: token n sits at (t, y, x) with n = (t*Hh + y)*W + x; the head dim
// is split into contiguous [t | h | w] blocks; pair i of a block of width d_s
// occupies dims (2i, 2i+1) of the block and turns by pos * theta^(-2i/d_s).
//
// HBM-bound: one 16-byte bf16 vector of output per thread, inputs read with
// 16/32-byte vector loads, (cos, sin) from a small per-axis fp64 table that
// stays in L1.  The same pass emits ||x||^2 of every stored (rounded) row and
// the max |x| of every (batch, head), which later stages use for the
// assignment error bound and the fixed-point scale of the centroid sums (per
// head, so a head's results never depend on the other heads of the call).
#include "common.cuh"

namespace scope {

// tab[s][pos][i] = (cos, sin)(pos * theta^(-2i/d_s)), in double.
__global__ void rope_table_kernel(double2 *tab, int T, int Hh, int W, int dt, int dh, int dw,
                                  double theta, int maxL, int maxP)
{
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= 3 * maxL * maxP) return;
    const int s = idx / (maxL * maxP), rem = idx % (maxL * maxP);
    const int pos = rem / maxP, i = rem % maxP;
    const int ds = s == 0 ? dt : (s == 1 ? dh : dw);
    const int len = s == 0 ? T : (s == 1 ? Hh : W);
    double2 v = make_double2(1.0, 0.0);
    if (2 * i < ds && pos < len) {
        const double phi = (double)pos * pow(theta, -2.0 * (double)i / (double)ds);
        double sn, cs;
        sincos(phi, &sn, &cs);
        v = make_double2(cs, sn);
    }
    tab[idx] = v;
}

template <typename TIn>
__device__ __forceinline__ void load8(const TIn *p, float *x);

template <>
__device__ __forceinline__ void load8<float>(const float *p, float *x)
{
    const float4 a = reinterpret_cast<const float4 *>(p)[0];
    const float4 b = reinterpret_cast<const float4 *>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float *x)
{
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

// One thread = 8 consecutive dims of one row; D/8 threads per row (8 or 16).
template <typename TIn>
__global__ void __launch_bounds__(256) rope_apply_kernel(
    const TIn *__restrict__ in, RowStrides rs, __nv_bfloat16 *__restrict__ out, float *__restrict__ norm2,
    float4 *__restrict__ sub2, uint32_t *__restrict__ maxabs, const double2 *__restrict__ tab, int64_t rows, int N,
    int D, int Hh, int W, int dt, int dh, int maxL, int maxP, int use_rope)
{
    __shared__ float bmax[8];
    const int tpr = D >> 3;  // 8 or 16 threads per row (D is 64 or 128)
    const int sh = D == 128 ? 4 : 3;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = gid >> sh;  // < rows < 2^31
    const int c8 = (int)(gid & (tpr - 1));
    const bool valid = row < rows;
    float ss = 0.f, mx = 0.f, nt = 0.f, nh = 0.f, nw = 0.f;  // row sum of squares and its t, h, w parts
    if (valid) {
        float x[8];
        load8<TIn>(in + rs.row(row / N, row % N) + c8 * 8, x);
        // The rotation runs in double and is rounded once to bf16, so every
        // stored element is the correctly rounded rotation of its input (in
        // fp32 a near-zero result of x0*c - x1*s can be off by more than one
        // bf16 ulp).  The kernel stays HBM-bound.
        double y[8];
        if (use_rope) {
            const int n = (int)row % N;
            const int pos3[3] = {n / (Hh * W), (n / W) % Hh, n % W};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int d = c8 * 8 + 2 * p;
                const int s = d < dt ? 0 : (d < dt + dh ? 1 : 2);
                const int off = s == 0 ? 0 : (s == 1 ? dt : dt + dh);
                const int i = (d - off) >> 1;
                const double2 cs = tab[(s * maxL + pos3[s]) * maxP + i];
                const double x0 = x[2 * p], x1 = x[2 * p + 1];
                y[2 * p] = x0 * cs.x - x1 * cs.y;
                y[2 * p + 1] = x0 * cs.y + x1 * cs.x;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = x[i];
        }
        __align__(16) __nv_bfloat162 o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            o[p].x = __double2bfloat16(y[2 * p]);
            o[p].y = __double2bfloat16(y[2 * p + 1]);
            const float2 r = __bfloat1622float2(o[p]);
            const float q2 = fmaf(r.y, r.y, r.x * r.x);  // the pair shares its block (blocks have even widths)
            ss += q2;
            const int d = c8 * 8 + 2 * p;
            nt += d < dt ? q2 : 0.f;
            nh += (d >= dt && d < dt + dh) ? q2 : 0.f;
            nw += d >= dt + dh ? q2 : 0.f;
            mx = fmaxf(mx, fmaxf(fabsf(r.x), fabsf(r.y)));
        }
        *reinterpret_cast<uint4 *>(out + row * D + c8 * 8) = *reinterpret_cast<const uint4 *>(o);
    }
    // Row norm over the tpr lanes that share the row (tpr divides 32).
    for (int o = tpr >> 1; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        nt += __shfl_xor_sync(0xffffffffu, nt, o);
        nh += __shfl_xor_sync(0xffffffffu, nh, o);
        nw += __shfl_xor_sync(0xffffffffu, nw, o);
    }
    if (norm2 && valid && c8 == 0) norm2[row] = ss;
    // squared norms of the (t, h, w) blocks of the stored row, for the key
    // subspaces' assignment error bound
    if (sub2 && valid && c8 == 0) sub2[row] = make_float4(nt, nh, nw, ss);
    // max |x| per (batch, head): the block's rows nearly always belong to one
    // head, whose maximum then takes one atomic (per-warp atomics on one word
    // would serialise); a block that straddles two heads updates per thread.
    const int64_t first = ((int64_t)blockIdx.x * blockDim.x) >> sh;
    const int64_t last = min(rows - 1, first + (int64_t)(blockDim.x >> sh) - 1);
    if (first / N == last / N) {
        mx = warp_max(mx);
        if ((threadIdx.x & 31) == 0) bmax[threadIdx.x >> 5] = mx;
        __syncthreads();
        if (threadIdx.x == 0) {
            for (int w = 1; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, bmax[w]);
            atomicMax(maxabs + first / N, __float_as_uint(mx));
        }
    } else if (valid && mx > 0.f) {
        atomicMax(maxabs + row / N, __float_as_uint(mx));
    }
}

void launch_rope_table(double2 *tab, int T, int Hh, int W, int dt, int dh, int dw, double theta,
                       int maxL, int maxP, cudaStream_t st)
{
    const int total = 3 * maxL * maxP;
    rope_table_kernel<<<(total + 255) / 256, 256, 0, st>>>(tab, T, Hh, W, dt, dh, dw, theta, maxL, maxP);
    count_launches(1);
}

void launch_rope_apply(const void *in, const RowStrides &rs, bool in_f32, __nv_bfloat16 *out, float *norm2,
                       float4 *sub2, uint32_t *maxabs,
                       const double2 *tab, int64_t rows, int N, int D, int Hh, int W, int dt, int dh,
                       int maxL, int maxP, int use_rope, cudaStream_t st)
{
    const int64_t threads = rows * (D / 8);
    const int64_t blocks = (threads + 255) / 256;
    if (in_f32)
        rope_apply_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
            (const float *)in, rs, out, norm2, sub2, maxabs, tab, rows, N, D, Hh, W, dt, dh, maxL, maxP, use_rope);
    else
        rope_apply_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            (const __nv_bfloat16 *)in, rs, out, norm2, sub2, maxabs, tab, rows, N, D, Hh, W, dt, dh, maxL, maxP,
            use_rope);
    count_launches(1);
}

// Contiguous bf16 copy of a (possibly strided) f32 tensor (V of f32 calls; the
// tensor-core path reads bf16).  One thread = 4 elements of one row.
__global__ void to_bf16_kernel(const float *__restrict__ in, RowStrides rs, uint2 *__restrict__ out, int64_t n4,
                               int N, int D)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const int64_t row = i / (D / 4);
    const int c4 = (int)(i % (D / 4));
    const float4 f = *reinterpret_cast<const float4 *>(in + rs.row(row / N, row % N) + 4 * c4);
    __nv_bfloat162 a = __floats2bfloat162_rn(f.x, f.y), b = __floats2bfloat162_rn(f.z, f.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    out[i] = u;
}

void launch_to_bf16(const float *in, const RowStrides &rs, __nv_bfloat16 *out, int64_t n, int N, int D,
                    cudaStream_t st)
{
    const int64_t n4 = n / 4;
    to_bf16_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(in, rs, (uint2 *)out, n4, N, D);
    count_launches(1);
}

}  // namespace scope
