// Grouped key lists for ClusterAttention leaves smaller than a Q tile
// ("ClusterAttention: A training-free speedup of bidirectional attention",
// abstract: power-of-two clusters, so the sparse attention runs at the
// dense per-pair rate).
//
// A leaf of 32 or 64 queries fills only part of a 128-row Q tile.  Instead,
// L = 256 / leaf consecutive leaves (siblings in the bisection tree, so their
// queries and their selected keys are close) share one attention work item
// of two full Q tiles.  The work item walks the union of the L leaves' lists
// (ascending) and masks, per leaf, the keys outside that leaf's own list, so
// every query still attends over exactly its own cluster's selection.
//
// pack_lists_kernel, one CTA per (group, bh):
//   union[]  the ascending union of the group's lists, stored at the offset
//            of the group's first leaf list (the union is never longer than
//            the lists it merges, so the groups' regions do not overlap);
//   u_n[]    its length;
//   masks    for every 128-key tile of the union and every leaf of the group,
//            the 128-bit membership mask (4 words, bit i = key i of the
//            tile is in the leaf's list), at tile slot
//            floor(loff / 128) + (bh * G + g) + tile, which keeps the
//            groups' slot ranges disjoint.
// The key range is swept in windows of 32 * kPackThreads keys: each leaf's
// entries of the window set bits in a per-leaf bitmap, the OR of the
// bitmaps gives the union's keys in order (one block scan per window), and
// each thread writes its union keys and ORs their membership bits into the
// tile masks (at most two words per leaf per thread and window).
#include "common.cuh"

namespace scope {

namespace {

constexpr int kPackThreads = 256;
constexpr int kPackWin = 32 * kPackThreads;
constexpr int kMaxGroupLeaves = 8;

__global__ void __launch_bounds__(kPackThreads)
    pack_lists_kernel(const long long *offsets, const int32_t *n_c, const int32_t *indices, int32_t *u_idx,
                      int32_t *u_n, uint32_t *masks, int Cq, int L, int G, int N)
{
    __shared__ uint32_t plane[kMaxGroupLeaves][kPackThreads];
    __shared__ int cur[kMaxGroupLeaves], seg_end[kMaxGroupLeaves];
    __shared__ int tmp[33];
    const int g = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int64_t c0 = (int64_t)bh * Cq + (int64_t)g * L;
    const long long loff = offsets[c0];
    long long total = 0;
    for (int l = 0; l < L; ++l) total += n_c[c0 + l];
    const long long slot = loff / 128 + (long long)bh * G + g;
    uint32_t *gm = masks + slot * L * 4;
    const long long words = (total + 127) / 128 * L * 4;
    for (long long i = tid; i < words; i += kPackThreads) gm[i] = 0u;
    if (tid < L) cur[tid] = 0;
    __syncthreads();  // masks zeroed before any OR below
    int out = 0;
    for (int w0 = 0; w0 < N; w0 += kPackWin) {
        if (tid < L) {  // end of this leaf's entries below w0 + kPackWin
            const int32_t *lst = indices + offsets[c0 + tid];
            int lo = cur[tid], hi = n_c[c0 + tid];
            const int lim = w0 + kPackWin;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (lst[mid] < lim) lo = mid + 1;
                else hi = mid;
            }
            seg_end[tid] = lo;
        }
#pragma unroll
        for (int l = 0; l < kMaxGroupLeaves; ++l) plane[l][tid] = 0u;
        __syncthreads();
        for (int l = 0; l < L; ++l) {
            const int32_t *lst = indices + offsets[c0 + l];
            for (int i = cur[l] + tid; i < seg_end[l]; i += kPackThreads) {
                const int kk = lst[i] - w0;
                atomicOr(&plane[l][kk >> 5], 1u << (kk & 31));
            }
        }
        __syncthreads();
        uint32_t bits[kMaxGroupLeaves], u = 0u;
#pragma unroll
        for (int l = 0; l < kMaxGroupLeaves; ++l) {
            bits[l] = plane[l][tid];
            u |= bits[l];
        }
        int tot;
        int p = out + block_excl_scan(__popc(u), tmp, tot);
        // this thread's union keys take positions p .. p + popc(u) - 1, which
        // touch at most two 32-position mask words
        uint32_t acc[kMaxGroupLeaves];
#pragma unroll
        for (int l = 0; l < kMaxGroupLeaves; ++l) acc[l] = 0u;
        int word = p >> 5;
        auto flush = [&]() {
            uint32_t *w = gm + (int64_t)(word >> 2) * L * 4 + (word & 3);
#pragma unroll
            for (int l = 0; l < kMaxGroupLeaves; ++l)
                if (l < L && acc[l]) atomicOr(w + l * 4, acc[l]);
#pragma unroll
            for (int l = 0; l < kMaxGroupLeaves; ++l) acc[l] = 0u;
        };
        while (u) {
            const int b = __ffs(u) - 1;
            u &= u - 1;
            if ((p >> 5) != word) {
                flush();
                word = p >> 5;
            }
            u_idx[loff + p] = w0 + tid * 32 + b;
#pragma unroll
            for (int l = 0; l < kMaxGroupLeaves; ++l) acc[l] |= ((bits[l] >> b) & 1u) << (p & 31);
            ++p;
        }
        flush();
        out += tot;
        __syncthreads();  // cur / seg_end / plane reused by the next window
        if (tid < L) cur[tid] = seg_end[tid];
    }
    if (tid == 0) u_n[(int64_t)bh * G + g] = out;
}

}  // namespace

// Bytes of the tile masks for a list capacity of `cap` entries.
size_t pack_mask_bytes(int64_t cap, int BH, int G, int L)
{
    return (size_t)(cap / 128 + (int64_t)BH * G + 2) * L * 16;
}

void launch_pack_lists(const long long *offsets, const int32_t *n_c, const int32_t *indices, int32_t *u_idx,
                       int32_t *u_n, uint32_t *masks, int BH, int Cq, int L, int N, cudaStream_t st)
{
    const int G = Cq / L;
    pack_lists_kernel<<<dim3(G, BH), kPackThreads, 0, st>>>(offsets, n_c, indices, u_idx, u_n, masks, Cq, L, G, N);
    count_launches(1);
}

}  // namespace scope
