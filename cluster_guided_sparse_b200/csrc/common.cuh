// Internal declarations shared by the libscope.so translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace scope {

constexpr int kSortBlk = 512;   // points per warp-block in the stable label sort
constexpr int kMaxClusters = 1024;
constexpr int kTQ = 128;        // query rows per attention tile
constexpr int kMaxItems = 65536; // c_t * c_h * c_w bound (distinct code triples)
constexpr int kScanTileCounters = 4096;  // block counters per tile of the label-sort scan
constexpr int kMaxBlocks = 16384;        // key blocks of the VMoBA block mode

// Device error word bits (workspace int32[4]).
constexpr int kErrRange = 1;
constexpr int kErrTimeout = 2;

// One clustering problem: rows X[bh][n][dim_off : dim_off + dim_n] into C
// clusters.  Key subspaces and queries of one plan run as one batch.
struct KmProblem {
    const __nv_bfloat16 *X;     // [BH][N][D]
    const uint32_t *maxabs;     // [BH] bits of max |X| per (batch, head) (non-negative float), set by RoPE
    int dim_off, dim_n, C;
    int32_t *labels;            // [BH][N]
    float *cent;                // [BH][C][dim_n]
    float *cn;                  // [BH][C] squared centroid norms
    int32_t *sizes;             // [BH][C]
    int32_t *perm;              // [BH][N]   members cluster by cluster, ascending
    int32_t *start;             // [BH][C+1] cluster starts in perm
    int32_t *blockhist;         // [BH][C][nblk]
    int32_t *tilesum;           // [BH][ceil(C*nblk / 4096)] scan tile sums
    unsigned long long *sums;   // [BH][C][dim_n] fixed-point member sums, zero between updates (or null)
};

// Where the rows of a caller's [B, H, N, D] tensor live: row (b, h, n)
// starts at element b*sB + h*sH + n*sN (D contiguous elements).  Kernels index
// by the flat (batch, head) number bh = b*H + h.
// Grouped attention lists: L consecutive ClusterAttention leaves of 2^leaf_shift
// queries share one work item over the union of their lists (pack.cu).
struct GroupedLists {
    const int32_t *u_idx;    // union lists at their group's first-leaf offset
    const int32_t *u_n;      // [BH][Cq / L] union lengths
    const uint32_t *masks;   // per tile and leaf, 128-bit membership masks
    int L, leaf_shift;
};

// Virtual keys of the ClusterAttention compensation (virt.cu): per virtual
// group (a grouped work item, else a query cluster) up to vtiles tiles of 64
// excluded key clusters, with per-leaf logit biases.
struct CompLists {
    const __nv_bfloat16 *vk_hi, *vk_lo, *vv_hi, *vv_lo;  // [BH][Ck][D] mean key / value, bf16 hi + lo
    const int32_t *vlist;  // [groups][vtiles * 64] key clusters
    const int32_t *vn;     // [groups] virtual keys per group
    const float *vbias;    // [groups][vtiles][Lv][64] ln(m) * sqrt(D), or -inf
    int Ck, Lv, vtiles;
};

// Outputs of a bisection part (bisect.cu): labels, leaf centroids and norms,
// leaf starts and sizes, the leaf-major permutation.
struct BisectOut {
    int32_t *labels;
    float *cent, *cn;
    int32_t *start, *sizes, *perm;
};

struct RowStrides {
    int64_t sB, sH, sN;
    int H;
    __host__ __device__ __forceinline__ int64_t bh_off(int64_t bh) const { return (bh / H) * sB + (bh % H) * sH; }
    __host__ __device__ __forceinline__ int64_t row(int64_t bh, int64_t n) const { return bh_off(bh) + n * sN; }
};

// Rows of up to four problems that a tensor-core assignment left to the
// fp64 re-decision: per problem a device counter and list of bh * N + n.
struct FixBatch {
    KmProblem p[4];
    const int32_t *list[4];
    const int32_t *count[4];
    int n;
};

struct KmBatch {
    KmProblem p[4];
    int count;
};

// Count of kernels launched by the library (see scope_kernel_launches).
void count_launches(int n);

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ uint32_t ordered_key(float s)
{
    // Monotone map float -> uint32: larger float -> larger key (no NaNs here).
    uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

template <typename T>
__device__ __forceinline__ T warp_incl_scan(T v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// Block-wide exclusive scan (blockDim.x a multiple of 32, <= 1024).
// `tmp` needs 33 elements of shared memory.  Returns the exclusive prefix;
// `total` receives the block sum.  Deterministic (fixed combination order).
template <typename T>
__device__ __forceinline__ T block_excl_scan(T v, T *tmp, T &total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    T inc = warp_incl_scan(v);
    __syncthreads();
    if (lane == 31) tmp[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        T w = lane < nw ? tmp[lane] : T(0);
        T wi = warp_incl_scan(w);
        if (lane < nw) tmp[lane] = wi - w;
        if (lane == nw - 1) tmp[32] = wi;
    }
    __syncthreads();
    total = tmp[32];
    return tmp[wid] + inc - v;
}

template <typename T>
__device__ __forceinline__ T warp_max(T v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ void set_error(int32_t *err, int bit, int detail)
{
    if (err) {
        atomicOr(err, bit);
        atomicCAS(err + 1, 0, detail);
    }
}

}  // namespace scope
