// scope_kmeans_noalloc: the k-means stage of scope_plan for callers that
// cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc (or a framework allocator) is
// unavailable or forbidden -- a plain C host program with no allocator of its
// own, an inference server whose device memory plan is frozen after start-up,
// or a plug-in that may only touch the buffers its host hands it.  Such a
// caller can pass its input and output buffers but cannot provide the sort
// and reduction scratch the clustering needs.
//
// How: the scratch lives in one file-scope __device__ array of
// kNoallocScratchBytes, which every GPU that loads the library keeps until the
// process exits.  Host code cannot use the array's name as a device address,
// so the first call on each device resolves the address with
// cudaGetSymbolAddress (with that device current) and caches it; make that
// first call before any stream capture.  All calls share the array and it
// keeps the last call's contents: the one region that must start at zero (the
// per-head max-|x| words) is cleared at the start of every call, everything else is
// fully rewritten.  Calls whose device work overlaps (e.g. on two streams)
// race on the array and must be serialised by the caller.
#include <mutex>

#include "../../include/scope.h"
#include "common.cuh"

namespace scope {
void launch_km_init(const KmBatch &, int, int, int, uint32_t, cudaStream_t);
void launch_km_assign_direct(const KmBatch &, int, int, int, cudaStream_t);
void launch_km_sort(const KmBatch &, int, int, cudaStream_t);
void launch_km_reduce(const KmBatch &, int, int, int, cudaStream_t);
cudaError_t km_configure();
}  // namespace scope

using namespace scope;

scope_status scope_set_error(scope_status s, const char *msg);

static constexpr size_t kNoallocScratchBytes = (size_t)SCOPE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Max |x| over every column of the rows (the fixed-point scale of the
// centroid sums).  scope_plan takes the same maximum over the whole rotated
// key (or query) rows for every subspace, so the two scales, and hence the
// rounding of the centroid sums, agree when x is the plan's rotated tensor.
// One maximum per (batch, head) (grid y), like the plan's.
__global__ void maxabs_kernel(const __nv_bfloat16 *__restrict__ x, int64_t n, uint32_t *out)
{
    float m = 0.f;
    const __nv_bfloat16 *xb = x + (int64_t)blockIdx.y * n;
    out += blockIdx.y;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        m = fmaxf(m, fabsf(__bfloat162float(xb[i])));
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(m));
}

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

}  // namespace

extern "C" size_t scope_kmeans_noalloc_scratch_bytes(int64_t B, int64_t H, int64_t N, int32_t C)
{
    if (B < 1 || H < 1 || N < 1 || C < 1) return 0;
    const int64_t BH = B * H, nblk = (N + kSortBlk - 1) / kSortBlk;
    const int64_t tiles = ((int64_t)C * nblk + kScanTileCounters - 1) / kScanTileCounters;
    return align256((size_t)BH * 4) + align256((size_t)BH * N * 4) + align256((size_t)BH * C * nblk * 4) +
           align256((size_t)BH * tiles * 4) +
           align256((size_t)BH * (C + 1) * 4) + 2 * align256((size_t)BH * C * 4);
}

extern "C" scope_status scope_kmeans_noalloc(const scope_tensor *x, int32_t dim_off, int32_t dim_n, int32_t C,
                                             int32_t iters, uint32_t init_seed, int32_t *labels, float *centroids,
                                             void *stream)
{
    if (!x || !x->ptr || !labels || !centroids) return scope_set_error(SCOPE_EINVAL, "noalloc: null pointer");
    if (((uintptr_t)x->ptr) & 15) return scope_set_error(SCOPE_EALIGN, "noalloc: x not 16-byte aligned");
    if ((((uintptr_t)labels) | ((uintptr_t)centroids)) & 3)
        return scope_set_error(SCOPE_EALIGN, "noalloc: labels and centroids must be 4-byte aligned");
    if (x->dtype != SCOPE_BF16) return scope_set_error(SCOPE_EDTYPE, "noalloc: x must be bf16");
    if (x->B < 1 || x->H < 1 || x->N < 1 || (x->D != 64 && x->D != 128))
        return scope_set_error(SCOPE_ESHAPE, "noalloc: x must be [B,H,N,D] with D in {64, 128}");
    {
        const int64_t *sd = x->strides;
        const bool zero = sd[0] == 0 && sd[1] == 0 && sd[2] == 0 && sd[3] == 0;
        const bool dense = sd[3] == 1 && sd[2] == x->D && sd[1] == x->N * x->D && (x->B == 1 || sd[0] == x->H * x->N * x->D);
        if (!zero && !dense) return scope_set_error(SCOPE_ESHAPE, "noalloc: x must be contiguous");
    }
    if (x->B * x->H > 65535 || x->B * x->H * x->N >= ((int64_t)1 << 31))
        return scope_set_error(SCOPE_ESHAPE, "noalloc: need B*H <= 65535 and B*H*N < 2^31");
    if (dim_off < 0 || dim_n < 1 || dim_off + dim_n > x->D)
        return scope_set_error(SCOPE_ESHAPE, "noalloc: column range outside [0, D)");
    if (C < 1 || C > kMaxClusters || C > x->N)
        return scope_set_error(SCOPE_EINVAL, "noalloc: need 1 <= C <= min(N, 1024)");
    if (iters < 0 || iters > 1000) return scope_set_error(SCOPE_EINVAL, "noalloc: iters must be in [0, 1000]");
    const size_t need = scope_kmeans_noalloc_scratch_bytes(x->B, x->H, x->N, C);
    if (need > kNoallocScratchBytes)
        return scope_set_error(SCOPE_ECAPACITY,
                               "noalloc: this shape needs more than the fixed scratch of "
                               "SCOPE_NOALLOC_SCRATCH_BYTES; use scope_plan with a workspace");

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return scope_set_error(SCOPE_EDEVICE, "noalloc: no usable CUDA device");
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10) return scope_set_error(SCOPE_EDEVICE, "noalloc: libscope.so is built for sm_100a");
    {
        // the scratch address below is the current device's: the stream's
        // kernels must run there too
        int sdev = -1;
        if (cudaStreamGetDevice((cudaStream_t)stream, &sdev) != cudaSuccess || sdev != dev)
            return scope_set_error(SCOPE_EDEVICE, "noalloc: the stream belongs to another device than the current one");
    }
    char *base;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_ptr[dev]) {
            void *p = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess || !p) return scope_set_error(SCOPE_ECUDA, "noalloc: cudaGetSymbolAddress failed");
            if (km_configure() != cudaSuccess) return scope_set_error(SCOPE_ECUDA, "noalloc: kernel setup failed");
            g_scratch_ptr[dev] = p;
        }
        base = (char *)g_scratch_ptr[dev];
    }
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t B = x->B, H = x->H, N = x->N, BH = B * H;
    const int nblk = (int)((N + kSortBlk - 1) / kSortBlk);
    size_t cur = 0;
    auto take = [&](size_t bytes) {
        char *p = base + cur;
        cur += align256(bytes);
        return p;
    };
    uint32_t *stats = (uint32_t *)take((size_t)BH * 4);
    KmProblem P{};
    P.X = (const __nv_bfloat16 *)x->ptr;
    P.maxabs = stats;
    P.dim_off = dim_off;
    P.dim_n = dim_n;
    P.C = C;
    P.labels = labels;
    P.cent = centroids;
    P.perm = (int32_t *)take((size_t)BH * N * 4);
    P.blockhist = (int32_t *)take((size_t)BH * C * nblk * 4);
    P.tilesum = (int32_t *)take((size_t)BH * (((int64_t)C * nblk + kScanTileCounters - 1) / kScanTileCounters) * 4);
    P.start = (int32_t *)take((size_t)BH * (C + 1) * 4);
    P.sizes = (int32_t *)take((size_t)BH * C * 4);
    P.cn = (float *)take((size_t)BH * C * 4);
    KmBatch b{};
    b.p[0] = P;
    b.count = 1;

    cudaMemsetAsync(stats, 0, (size_t)BH * 4, s);
    maxabs_kernel<<<dim3((unsigned)((4 * 148 + BH - 1) / BH), (unsigned)BH), 256, 0, s>>>(P.X, N * x->D, stats);
    count_launches(1);
    launch_km_init(b, (int)BH, (int)N, (int)x->D, init_seed, s);
    for (int it = 0; it < iters; ++it) {
        launch_km_assign_direct(b, (int)BH, (int)N, (int)x->D, s);
        launch_km_sort(b, (int)BH, (int)N, s);
        launch_km_reduce(b, (int)BH, (int)N, (int)x->D, s);
    }
    launch_km_assign_direct(b, (int)BH, (int)N, (int)x->D, s);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return scope_set_error(SCOPE_ECUDA, cudaGetErrorString(e));
    return SCOPE_OK;
}
