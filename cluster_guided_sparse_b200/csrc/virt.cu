// ClusterAttention's compensation of excluded clusters ("ClusterAttention: A
// training-free speedup of bidirectional attention", abstract: the method
// compensates the clusters it leaves out through their mean), computed on
// the tensor cores inside the sparse attention.
//
// Reading: key cluster k (a bisection leaf) has mean key mu_k -- the plan's
// fp32 leaf centroid, the exact mean of its bf16 member keys -- and mean value
// vbar_k.  For query cluster c with selected keys S_c, m_ck members of k are
// not in S_c, and each enters the softmax through its cluster's mean:
//   o = (sum_{j in S} e^{a_j} v_j + sum_k m_ck e^{b_k} vbar_k)
//     / (sum_{j in S} e^{a_j} + sum_k m_ck e^{b_k}),
// a_j = q.k_j / sqrt(d), b_k = q.mu_k / sqrt(d).  The second sums are an
// attention over "virtual" keys (mu_k, vbar_k) whose logits carry ln m_ck,
// so the attention kernel walks them after the listed keys, in the same
// online softmax: this file builds their lists and operands.
//
//   kbar_split_kernel   mu_k as a bf16 hi + lo pair (plan time)
//   virt_lists_kernel   per virtual group (a grouped work item of Lv leaves,
//                       else one query cluster): the key clusters with an
//                       excluded member for any of its leaves, ascending, in
//                       tiles of 64, and per tile and leaf the 64 logit
//                       offsets ln(m) * sqrt(D) (-inf where the leaf excludes
//                       nothing of that cluster, and on padding slots)
//   vmean_split_kernel  vbar_k (fp64 sums) as a bf16 hi + lo pair (attention
//                       time: V is an argument of scope_attn)
#include "common.cuh"

namespace scope {

namespace {

__device__ __forceinline__ void split_bf16(double x, __nv_bfloat16 &hi, __nv_bfloat16 &lo)
{
    hi = __float2bfloat16_rn((float)x);
    lo = __float2bfloat16_rn((float)(x - (double)__bfloat162float(hi)));
}

__global__ void kbar_split_kernel(const float *kcent, __nv_bfloat16 *hi, __nv_bfloat16 *lo, int64_t total)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < total) split_bf16((double)kcent[i], hi[i], lo[i]);
}

// One CTA per (virtual group, bh).  Shared: per-key-cluster counts of one
// leaf's selected keys, the union flags (bit l: leaf l excludes a member),
// and every flagged cluster's slot.
__global__ void __launch_bounds__(256)
    virt_lists_kernel(const long long *offsets, const int32_t *n_c, const int32_t *indices, const int32_t *klab,
                      const int32_t *ksize, int32_t *vlist, int32_t *vn, float *vbias, int N, int Cq, int Ck, int Lv,
                      int vtiles, float sqrt_d)
{
    __shared__ int hist[kMaxClusters], slot[kMaxClusters];
    __shared__ uint8_t flags[kMaxClusters];
    __shared__ int tmp[33];
    const int g = blockIdx.x, bh = blockIdx.y, NG = gridDim.x, tid = threadIdx.x;
    const int64_t vg = (int64_t)bh * NG + g;
    const int64_t c0 = (int64_t)bh * Cq + (int64_t)g * Lv;
    const int32_t *kl = klab + (int64_t)bh * N;
    const int32_t *ks = ksize + (int64_t)bh * Ck;
    auto count_leaf = [&](int l) {  // hist[k] = selected keys of leaf l in cluster k
        for (int k = tid; k < Ck; k += blockDim.x) hist[k] = 0;
        __syncthreads();
        const int32_t *lst = indices + offsets[c0 + l];
        const int n = n_c[c0 + l];
        for (int t = tid; t < n; t += blockDim.x) atomicAdd(&hist[kl[lst[t]]], 1);
        __syncthreads();
    };
    for (int k = tid; k < Ck; k += blockDim.x) flags[k] = 0;
    for (int l = 0; l < Lv; ++l) {
        count_leaf(l);
        for (int k = tid; k < Ck; k += blockDim.x)
            if (ks[k] - hist[k] > 0) flags[k] |= (uint8_t)(1u << l);
        __syncthreads();
    }
    // slots in ascending cluster order
    int carry = 0;
    for (int b0 = 0; b0 < Ck; b0 += blockDim.x) {
        const int k = b0 + tid;
        const int f = (k < Ck && flags[k]) ? 1 : 0;
        int tot;
        const int ex = block_excl_scan(f, tmp, tot);
        if (f) {
            slot[k] = carry + ex;
            vlist[vg * vtiles * 64 + carry + ex] = k;
        }
        carry += tot;
    }
    const int nv = carry;
    const int padded = (nv + 63) & ~63;
    __syncthreads();
    const int last = nv > 0 ? vlist[vg * vtiles * 64 + nv - 1] : 0;
    for (int p = nv + tid; p < padded; p += blockDim.x) vlist[vg * vtiles * 64 + p] = last;
    float *vb = vbias + vg * vtiles * Lv * 64;
    for (int p = nv + tid; p < padded; p += blockDim.x)
        for (int l = 0; l < Lv; ++l) vb[((p >> 6) * Lv + l) * 64 + (p & 63)] = -INFINITY;
    for (int l = 0; l < Lv; ++l) {
        count_leaf(l);
        for (int k = tid; k < Ck; k += blockDim.x) {
            if (!flags[k]) continue;
            const int m = ks[k] - hist[k], p = slot[k];
            vb[((p >> 6) * Lv + l) * 64 + (p & 63)] = m > 0 ? logf((float)m) * sqrt_d : -INFINITY;
        }
        __syncthreads();
    }
    if (tid == 0) vn[vg] = nv;
}

// vbar_k: mean of V over the members of key cluster k (fp64 sums), one
// thread per dim, stored as a bf16 hi + lo pair.
__global__ void vmean_split_kernel(const __nv_bfloat16 *V, RowStrides vs, const int32_t *perm, const int32_t *start,
                                   __nv_bfloat16 *hi, __nv_bfloat16 *lo, int N, int D, int Ck)
{
    const int k = blockIdx.x, bh = blockIdx.y, d = threadIdx.x;
    if (d >= D) return;
    const int32_t *st = start + (int64_t)bh * (Ck + 1);
    const int s0 = st[k], s1 = st[k + 1];
    const int32_t *pm = perm + (int64_t)bh * N;
    const __nv_bfloat16 *Vb = V + vs.bh_off(bh);
    double acc = 0.0;
    for (int t = s0; t < s1; ++t) acc += (double)__bfloat162float(Vb[(int64_t)pm[t] * vs.sN + d]);
    const int64_t o = ((int64_t)bh * Ck + k) * D + d;
    split_bf16(s1 > s0 ? acc / (double)(s1 - s0) : 0.0, hi[o], lo[o]);
}

}  // namespace

// Tiles of 64 virtual keys a virtual group can need (every key cluster).
int virt_tiles(int Ck) { return (Ck + 63) / 64; }

// Plan time: mean keys as hi/lo pairs, and the virtual lists.
void launch_virt_plan(const float *kcent, __nv_bfloat16 *vk_hi, __nv_bfloat16 *vk_lo, const long long *offsets,
                      const int32_t *n_c, const int32_t *indices, const int32_t *klab, const int32_t *ksize,
                      int32_t *vlist, int32_t *vn, float *vbias, int BH, int N, int D, int Cq, int Ck, int Lv,
                      cudaStream_t st)
{
    const int64_t total = (int64_t)BH * Ck * D;
    kbar_split_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(kcent, vk_hi, vk_lo, total);
    virt_lists_kernel<<<dim3(Cq / Lv, BH), 256, 0, st>>>(offsets, n_c, indices, klab, ksize, vlist, vn, vbias, N, Cq,
                                                         Ck, Lv, virt_tiles(Ck), sqrtf((float)D));
    count_launches(2);
}

// Attention time: mean values as hi/lo pairs.
void launch_vmean(const __nv_bfloat16 *v, const RowStrides &vs, const int32_t *k_perm, const int32_t *k_start,
                  __nv_bfloat16 *vv_hi, __nv_bfloat16 *vv_lo, int BH, int N, int D, int Ck, cudaStream_t st)
{
    vmean_split_kernel<<<dim3(Ck, BH), D, 0, st>>>(v, vs, k_perm, k_start, vv_hi, vv_lo, N, D, Ck);
    count_launches(1);
}

}  // namespace scope
