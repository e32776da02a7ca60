// ClusterAttention's compensation of excluded clusters ("ClusterAttention: A
// training-free speedup of bidirectional attention", abstract: the method
// compensates the clusters it leaves out through their mean).
//
// Reading: key cluster k (a bisection leaf) has mean key mu_k -- the plan's
// fp32 leaf centroid, the exact mean of its bf16 member keys -- and mean value
// vbar_k.  For query cluster c with selected keys S_c, m_ck members of k are
// not in S_c, and each enters the softmax through its cluster's mean:
//   o = (sum_{j in S} e^{a_j} v_j + sum_k m_ck e^{b_k} vbar_k)
//     / (sum_{j in S} e^{a_j} + sum_k m_ck e^{b_k}),
// a_j = q.k_j / sqrt(d), b_k = q.mu_k / sqrt(d).  The attention kernel leaves
// the first sums as its (normalised) output row o_S and the row's natural
// log-sum-exp L_S, so this pass forms
//   o = (e^{L_S} o_S + sum_k m_ck e^{b_k} vbar_k) / (e^{L_S} + sum_k m_ck e^{b_k})
// with a running maximum, in fp32, and overwrites the row.
#include "common.cuh"

namespace scope {

namespace {

constexpr int kCompThreads = 128;

// vbar_k: mean of V over the members of key cluster k (fp64 sums), one
// thread per dim.
__global__ void vmean_kernel(const __nv_bfloat16 *V, RowStrides vs, const int32_t *perm, const int32_t *start,
                             float *vmean, int N, int D, int C)
{
    const int k = blockIdx.x, bh = blockIdx.y, d = threadIdx.x;
    if (d >= D) return;
    const int32_t *st = start + (int64_t)bh * (C + 1);
    const int s0 = st[k], s1 = st[k + 1];
    const int32_t *pm = perm + (int64_t)bh * N;
    const __nv_bfloat16 *Vb = V + vs.bh_off(bh);
    double acc = 0.0;
    for (int t = s0; t < s1; ++t) acc += (double)__bfloat162float(Vb[(int64_t)pm[t] * vs.sN + d]);
    vmean[((int64_t)bh * C + k) * D + d] = s1 > s0 ? (float)(acc / (double)(s1 - s0)) : 0.f;
}

struct CompArgs {
    const __nv_bfloat16 *qr;     // [BH][N][D] rotated queries (the attention's)
    const int32_t *q_perm;       // [BH][N] query-cluster members
    const int32_t *q_start;      // [BH][Cq+1]
    const int32_t *klab;         // [BH][N] key cluster of every key
    const int32_t *ksize;        // [BH][Ck]
    const float *kcent;          // [BH][Ck][D] mean keys
    const float *vmean;          // [BH][Ck][D] mean values
    const long long *offsets;    // [BH*Cq]
    const int32_t *indices;      // selected-key lists
    const int32_t *n_c;          // [BH][Cq]
    const float *lse;            // [BH][N] log-sum-exp of the attention rows
    __nv_bfloat16 *o;            // caller's rows (strides os) in: o_S, out: compensated
    RowStrides os;
    int N, Cq, Ck;
    float scale;                 // 1 / sqrt(D)
};

// One CTA per (query cluster, head): count the cluster's selected keys per
// key cluster, list the key clusters with excluded members (with ln m), then
// one thread per query row adds their terms.
template <int D>
__global__ void __launch_bounds__(kCompThreads) comp_kernel(CompArgs a)
{
    extern __shared__ int sh[];
    int *hist = sh;                                         // [Ck]
    int *ex_k = sh + a.Ck;                                  // [Ck]
    float *ex_lm = reinterpret_cast<float *>(ex_k + a.Ck);  // [Ck]
    __shared__ int tmp[33];
    const int c = blockIdx.x, bh = blockIdx.y;
    const int64_t bhc = (int64_t)bh * a.Cq + c;
    const int32_t *qs = a.q_start + (int64_t)bh * (a.Cq + 1);
    const int q0 = qs[c], q1 = qs[c + 1];
    if (q1 <= q0) return;
    for (int k = threadIdx.x; k < a.Ck; k += blockDim.x) hist[k] = 0;
    __syncthreads();
    const int n = a.n_c[bhc];
    const int32_t *lst = a.indices + a.offsets[bhc];
    const int32_t *klab = a.klab + (int64_t)bh * a.N;
    for (int t = threadIdx.x; t < n; t += blockDim.x) atomicAdd(&hist[klab[lst[t]]], 1);
    __syncthreads();
    const int32_t *ksz = a.ksize + (int64_t)bh * a.Ck;
    int carry = 0;
    for (int b0 = 0; b0 < a.Ck; b0 += blockDim.x) {
        const int k = b0 + threadIdx.x;
        const int m = k < a.Ck ? ksz[k] - hist[k] : 0;
        int tot;
        const int ex = block_excl_scan(m > 0 ? 1 : 0, tmp, tot);
        if (m > 0) {
            ex_k[carry + ex] = k;
            ex_lm[carry + ex] = logf((float)m);
        }
        carry += tot;
    }
    __syncthreads();
    const int n_ex = carry;
    if (n_ex == 0) return;
    const float *kc = a.kcent + (int64_t)bh * a.Ck * D;
    const float *vm = a.vmean + (int64_t)bh * a.Ck * D;
    for (int r = q0 + threadIdx.x; r < q1; r += blockDim.x) {
        const int tok = a.q_perm[(int64_t)bh * a.N + r];
        const int64_t row = (int64_t)bh * a.N + tok;
        __nv_bfloat16 *orow = a.o + a.os.row(bh, tok);
        float q[D], acc[D];
#pragma unroll
        for (int d = 0; d < D; ++d) {
            q[d] = __bfloat162float(a.qr[row * D + d]) * a.scale;
            acc[d] = __bfloat162float(orow[d]);
        }
        float mx = a.lse[row], den = 1.f;  // the selected keys: weight e^{L_S}, value o_S
        for (int e = 0; e < n_ex; ++e) {
            const int k = ex_k[e];
            const float *mu = kc + (int64_t)k * D;
            const float *vb = vm + (int64_t)k * D;
            float s = 0.f;
#pragma unroll
            for (int d = 0; d < D; ++d) s = fmaf(q[d], mu[d], s);
            const float b = s + ex_lm[e];
            if (b > mx) {
                const float f = __expf(mx - b);
                den = fmaf(den, f, 1.f);
#pragma unroll
                for (int d = 0; d < D; ++d) acc[d] = fmaf(acc[d], f, vb[d]);
                mx = b;
            } else {
                const float w = __expf(b - mx);
                den += w;
#pragma unroll
                for (int d = 0; d < D; ++d) acc[d] = fmaf(w, vb[d], acc[d]);
            }
        }
        const float inv = 1.f / den;
#pragma unroll
        for (int d = 0; d < D; d += 2) {
            __nv_bfloat162 h = __floats2bfloat162_rn(acc[d] * inv, acc[d + 1] * inv);
            *reinterpret_cast<__nv_bfloat162 *>(orow + d) = h;
        }
    }
}

}  // namespace

// Mean values of the key clusters, then the compensation of every query row.
void launch_compensate(const __nv_bfloat16 *qr, const __nv_bfloat16 *v, const RowStrides &vs, const int32_t *q_perm,
                       const int32_t *q_start, const int32_t *k_perm, const int32_t *k_start, const int32_t *klab,
                       const int32_t *ksize, const float *kcent, float *vmean, const long long *offsets,
                       const int32_t *indices, const int32_t *n_c, const float *lse, __nv_bfloat16 *o,
                       const RowStrides &os, int BH, int N, int D, int Cq, int Ck, cudaStream_t st)
{
    vmean_kernel<<<dim3(Ck, BH), D, 0, st>>>(v, vs, k_perm, k_start, vmean, N, D, Ck);
    count_launches(1);
    CompArgs a;
    a.qr = qr;
    a.q_perm = q_perm;
    a.q_start = q_start;
    a.klab = klab;
    a.ksize = ksize;
    a.kcent = kcent;
    a.vmean = vmean;
    a.offsets = offsets;
    a.indices = indices;
    a.n_c = n_c;
    a.lse = lse;
    a.o = o;
    a.os = os;
    a.N = N;
    a.Cq = Cq;
    a.Ck = Ck;
    a.scale = 1.0f / sqrtf((float)D);
    const size_t smem = (size_t)Ck * 3 * sizeof(int);
    if (D == 128)
        comp_kernel<128><<<dim3(Cq, BH), kCompThreads, smem, st>>>(a);
    else
        comp_kernel<64><<<dim3(Cq, BH), kCompThreads, smem, st>>>(a);
    count_launches(1);
}

}  // namespace scope
