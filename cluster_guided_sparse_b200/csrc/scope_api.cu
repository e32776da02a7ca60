// Host side of libscope.so: argument checks, workspace layout, the launch
// sequence of scope_plan / scope_attn / scope_dense_attn, result views.
// Every argument check runs before any CUDA call, so a bad call never
// touches the device.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <string>

#include "../../include/scope.h"
#include "common.cuh"

namespace scope {
// kernels.cu launchers
void launch_rope_table(double2 *, int, int, int, int, int, int, double, int, int, cudaStream_t);
void launch_rope_apply(const void *, const RowStrides &, bool, __nv_bfloat16 *, float *, float4 *, uint32_t *,
                       const double2 *, int64_t, int, int, int, int, int, int, int, int, int, cudaStream_t);
void km_fixup_launch(const FixBatch &, int, int, cudaStream_t);
bool launch_km_assign_keys_tc(const KmProblem *, __nv_bfloat16 *, __nv_bfloat16 *, int, int, int, const float4 *,
                              int32_t *, int32_t *, cudaStream_t);
void launch_to_bf16(const float *, const RowStrides &, __nv_bfloat16 *, int64_t, int, int, cudaStream_t);
cudaError_t km_configure();
void launch_km_init(const KmBatch &, int, int, int, uint32_t, cudaStream_t);
void launch_km_assign_direct(const KmBatch &, int, int, int, cudaStream_t);
void launch_km_sort(const KmBatch &, int, int, cudaStream_t);
void launch_bisect(const __nv_bfloat16 *, int, int, int, int, int, int32_t *, int32_t *, double *, void *,
                   const BisectOut *, int, cudaStream_t);
size_t bisect_aux_bytes(int BH, int N, int D);
cudaError_t km_tc_configure();
bool launch_km_assign_tc(const KmProblem &, __nv_bfloat16 *, __nv_bfloat16 *, int, int, int, const float *, int32_t *,
                         int32_t *, int32_t *, cudaStream_t);
void launch_km_reduce(const KmBatch &, int, int, int, cudaStream_t);

struct SelArgs;
void launch_lut(const float *, const float *, const float *, const float *, float *, int, int, int, int, int, int,
                int, int, int, cudaStream_t);
void launch_items(const int32_t *, int32_t *, int32_t *, int32_t *, int32_t *, uint16_t *, int, int, int, int, int,
                  int, cudaStream_t);
cudaError_t select_configure();
cudaError_t attn_tc_configure();
int attn_tc_max_items(int BH, int N, int Cq);
bool launch_attn_tc(const __nv_bfloat16 *, const __nv_bfloat16 *, const __nv_bfloat16 *, const RowStrides &,
                    __nv_bfloat16 *, const RowStrides &, int4 *, int32_t *, int, const int32_t *, const int32_t *,
                    const int32_t *, const long long *, const int32_t *, const int32_t *, int32_t *, int, int, int, int,
                    cudaStream_t, const GroupedLists *, const CompLists *);
size_t pack_mask_bytes(int64_t cap, int BH, int G, int L);
void launch_pack_lists(const long long *, const int32_t *, const int32_t *, int32_t *, int32_t *, uint32_t *, int, int,
                       int, int, cudaStream_t);
int virt_tiles(int Ck);
void launch_virt_plan(const float *, __nv_bfloat16 *, __nv_bfloat16 *, const long long *, const int32_t *,
                      const int32_t *, const int32_t *, const int32_t *, int32_t *, int32_t *, float *, int, int, int, int,
                      int, int, cudaStream_t);
void launch_vmean(const __nv_bfloat16 *, const RowStrides &, const int32_t *, const int32_t *, __nv_bfloat16 *,
                  __nv_bfloat16 *, int, int, int, int, cudaStream_t);
void launch_wait_timeout(int32_t *err, long long limit, cudaStream_t st);
void run_selection(const float *lut, const int32_t *codes, const int32_t *item_id, const int32_t *item_cnt,
                   const int32_t *item_n, const uint16_t *key_item, int Pcap, int N, int Cq, int Ct, int Ch, int Cw,
                   int BH, float top_p,
                   float inv_sqrt_d, int k_min, int32_t *err, const int32_t *sizes, int32_t *r, int32_t *n,
                   int32_t *kh, long long *offsets, int32_t *indices, int online, void *state, int B, float eg_tau,
                   int eg_group, void *eg_state, int whole_items, cudaStream_t st);
size_t selection_state_bytes(int64_t clusters);
size_t eg_state_bytes(int64_t B, int64_t H, int64_t Cq, int group);
int block_count(int T, int Hh, int W, int kind, int bt, int bh, int bw);
void launch_blocks(int T, int Hh, int W, int kind, int bt, int bh, int bw, const __nv_bfloat16 *kr, int32_t *codes,
                   float *cent, float *cn, int32_t *sizes, int BH, int N, int D, cudaStream_t st);
}  // namespace scope

using namespace scope;

static thread_local std::string g_err;

static scope_status fail(scope_status s, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

extern "C" const char *scope_last_error(void) { return g_err.c_str(); }

// Lets other translation units of the library report an error message.
scope_status scope_set_error(scope_status s, const char *msg) { return fail(s, "%s", msg); }
extern "C" int scope_version(void) { return 1; }

static std::atomic<long long> g_launches{0};
void scope::count_launches(int n) { g_launches += n; }
extern "C" int64_t scope_kernel_launches(void) { return g_launches.load(); }

// ---------------------------------------------------------------- workspace layout
namespace {

struct Layout {
    int64_t B, H, N, D, BH;
    int Cq, C[3], ds[3], off[3], Csum, P, Pcap, nblk, max_work, maxL, maxP;
    bool f32, bisect;
    int64_t cap;
    size_t qr, kr, qnorm, ksub2, kchi, kclo, kfix, tab, stats, maxabs, q_lab, q_cent, q_cn, q_sizes, q_perm, q_start, q_bhist, q_tsum;
    size_t k_codes, k_cent[3], k_cn[3], k_sizes[3], k_perm[3], k_start[3], k_bhist[3], k_tsum[3];
    size_t sel_state, eg_state, lut, item_hist, item_id, item_cnt, item_n, key_item, r, n, kh, offsets, indices, work, nwork, vb, fix;
    size_t bis_order, bis_delta, bis_aux, q_chi, q_clo, q_sums, k_sums[3], sums_bytes;
    size_t vk_hi, vk_lo, vv_hi, vv_lo, vlist, vn, vbias;  // compensation's virtual keys (comp)
    int Lv, vtiles;                                        // leaves per virtual group, tiles per group
    size_t u_idx, u_n, gmask;  // grouped attention lists (gL > 0)
    int gL, gshift, G;         // leaves per group, log2(leaf), groups per head
    bool comp, eg, blocks;
    size_t total;
};

// Tiles of the parallel scan over a problem's C x nblk block counters.
int64_t scan_tiles(int64_t C, int64_t nblk) { return (C * nblk + kScanTileCounters - 1) / kScanTileCounters; }

size_t take(size_t &cur, size_t bytes)
{
    const size_t at = cur;
    cur += (bytes + 255) & ~(size_t)255;
    return at;
}

bool tensor_ok(const scope_tensor *t, const char *name, scope_status *st)
{
    if (!t) {
        *st = fail(SCOPE_EINVAL, "%s: null tensor", name);
        return false;
    }
    if (!t->ptr) {
        *st = fail(SCOPE_EINVAL, "%s: null data pointer", name);
        return false;
    }
    if (((uintptr_t)t->ptr) & 15) {
        *st = fail(SCOPE_EALIGN, "%s: pointer not 16-byte aligned", name);
        return false;
    }
    if (t->B < 1 || t->H < 1 || t->N < 1) {
        *st = fail(SCOPE_ESHAPE, "%s: B, H, N must be >= 1 (got %lld, %lld, %lld)", name, (long long)t->B,
                   (long long)t->H, (long long)t->N);
        return false;
    }
    if (t->D != 64 && t->D != 128) {
        *st = fail(SCOPE_ESHAPE, "%s: head dim must be 64 or 128 (got %lld)", name, (long long)t->D);
        return false;
    }
    if (t->B * t->H * t->N >= (int64_t)1 << 31 || t->B * t->H > 65535) {
        *st = fail(SCOPE_ESHAPE, "%s: B*H*N must be < 2^31 and B*H <= 65535", name);
        return false;
    }
    if (t->N > (1 << 24)) {
        *st = fail(SCOPE_ESHAPE, "%s: N must be <= 2^24 (got %lld)", name, (long long)t->N);
        return false;
    }
    if (t->dtype != SCOPE_F32 && t->dtype != SCOPE_BF16) {
        *st = fail(SCOPE_EDTYPE, "%s: dtype must be f32 or bf16", name);
        return false;
    }
    const int64_t *sd = t->strides;
    if (sd[0] == 0 && sd[1] == 0 && sd[2] == 0 && sd[3] == 0) return true;  // contiguous
    const int64_t elt = t->dtype == SCOPE_F32 ? 4 : 2;
    if (sd[3] != 1 || sd[0] < 0 || sd[1] < 0 || sd[2] < 0) {
        *st = fail(SCOPE_ESHAPE, "%s: strides[3] must be 1 and the others >= 0", name);
        return false;
    }
    for (int i = 0; i < 3; ++i)
        if ((sd[i] * elt) % 16) {
            *st = fail(SCOPE_ESHAPE, "%s: strides[%d] * element size must be a multiple of 16 bytes", name, i);
            return false;
        }
    // distinct (b, h, n) must not share a row: with the dimensions of extent
    // > 1 sorted by stride, each stride must reach past the previous
    // dimension's whole extent (the row itself is D elements wide)
    int64_t st_[4] = {1, sd[2], sd[1], sd[0]}, ex[4] = {t->D, t->N, t->H, t->B};
    int m = 0;
    for (int i = 0; i < 4; ++i)
        if (ex[i] > 1 || i == 0) {
            if (st_[i] == 0) {
                *st = fail(SCOPE_ESHAPE, "%s: strides make distinct rows overlap", name);
                return false;
            }
            st_[m] = st_[i];
            ex[m] = ex[i];
            ++m;
        }
    for (int i = 1; i < m; ++i)
        for (int j = i; j > 0 && st_[j] < st_[j - 1]; --j) {
            int64_t a = st_[j]; st_[j] = st_[j - 1]; st_[j - 1] = a;
            a = ex[j]; ex[j] = ex[j - 1]; ex[j - 1] = a;
        }
    for (int i = 1; i < m; ++i)
        if (st_[i] < st_[i - 1] * ex[i - 1]) {
            *st = fail(SCOPE_ESHAPE, "%s: strides make distinct rows overlap", name);
            return false;
        }
    return true;
}

// Row addressing of a caller tensor (all-zero strides: contiguous).
RowStrides rows_of(const scope_tensor *t)
{
    RowStrides r;
    r.H = (int)t->H;
    if (t->strides[0] == 0 && t->strides[1] == 0 && t->strides[2] == 0 && t->strides[3] == 0) {
        r.sN = t->D;
        r.sH = t->N * t->D;
        r.sB = t->H * t->N * t->D;
    } else {
        r.sB = t->strides[0];
        r.sH = t->strides[1];
        r.sN = t->strides[2];
    }
    return r;
}

RowStrides contiguous_rows(int64_t H, int64_t N, int64_t D)
{
    RowStrides r;
    r.H = (int)H;
    r.sN = D;
    r.sH = N * D;
    r.sB = H * N * D;
    return r;
}

bool same_shape(const scope_tensor *a, const scope_tensor *b)
{
    return a->B == b->B && a->H == b->H && a->N == b->N && a->D == b->D;
}

scope_status check_params(const scope_tensor *q, const scope_grid *g, const scope_params *p)
{
    if (!p) return fail(SCOPE_EINVAL, "params: null");
    const int64_t N = q->N, D = q->D;
    const int ds[3] = {p->d_t, p->d_h, p->d_w};
    const int C[3] = {p->c_t, p->c_h, p->c_w};
    for (int s = 0; s < 3; ++s)
        if (ds[s] < 0 || (ds[s] & 1)) return fail(SCOPE_ESHAPE, "params: d_t/d_h/d_w must be even and >= 0");
    if ((int64_t)ds[0] + ds[1] + ds[2] != D) return fail(SCOPE_ESHAPE, "params: d_t + d_h + d_w must equal D");
    if (!(p->top_p > 0.0f && p->top_p <= 1.0f)) return fail(SCOPE_EINVAL, "params: top_p must be in (0, 1]");
    if (p->k_min < 0) return fail(SCOPE_EINVAL, "params: k_min must be >= 0");
    if (p->iters < 0 || p->iters > 1000) return fail(SCOPE_EINVAL, "params: iters must be in [0, 1000]");
    if (p->online_topk != 0 && p->online_topk != 1) return fail(SCOPE_EINVAL, "params: online_topk must be 0 or 1");
    if (!(p->theta > 0.0)) return fail(SCOPE_EINVAL, "params: theta must be > 0");
    const bool has_grid = g && (g->T != 0 || g->Hh != 0 || g->W != 0);
    if (has_grid) {
        if (g->T < 1 || g->Hh < 1 || g->W < 1) return fail(SCOPE_ESHAPE, "grid: T, Hh, W must all be >= 1 or all 0");
        if ((int64_t)g->T * g->Hh * g->W != N) return fail(SCOPE_ESHAPE, "grid: T*Hh*W must equal N");
    }
    if (p->fixed_cluster_size < 0) return fail(SCOPE_EINVAL, "params: fixed_cluster_size must be >= 0");
    if (p->compensate != 0 && p->compensate != 1) return fail(SCOPE_EINVAL, "params: compensate must be 0 or 1");
    if (!(p->eg_tau >= 0.f && p->eg_tau <= 2.f))
        return fail(SCOPE_EINVAL, "params: eg_tau must be in [0, 2] (0 = no EG-Sparse routing)");
    if (p->eg_tau > 0.f && (p->eg_group < 1 || p->eg_group > 64))
        return fail(SCOPE_EINVAL, "params: eg_group must be in [1, 64] when eg_tau > 0");
    if (p->eg_tau > 0.f && (int64_t)(p->eg_group < q->H ? p->eg_group : q->H) * q->N > ((int64_t)1 << 24))
        return fail(SCOPE_EINVAL, "params: a pool's queries (min(eg_group, H) * N) must be <= 2^24");
    if (p->block_kind < 0 || p->block_kind > 3) return fail(SCOPE_EINVAL, "params: block_kind must be 0..3");
    if (p->block_kind > 0) {
        if (!has_grid) return fail(SCOPE_EINVAL, "block_kind needs a grid");
        if (p->block_t < 1 || p->block_h < 1 || p->block_w < 1)
            return fail(SCOPE_EINVAL, "params: block_t, block_h, block_w must be >= 1");
        if (p->k_min != 0 || p->online_topk != 0 || p->eg_tau > 0.f || p->fixed_cluster_size > 0 || p->compensate)
            return fail(SCOPE_EINVAL, "block_kind needs k_min = 0, online_topk = 0, eg_tau = 0, no "
                                      "fixed_cluster_size and no compensate");
        if ((int64_t)p->block_t * p->block_h * p->block_w > N)
            return fail(SCOPE_EINVAL, "params: a block must not exceed N tokens");
        const int nb = block_count(g->T, g->Hh, g->W, p->block_kind, p->block_t, p->block_h, p->block_w);
        if (nb > kMaxBlocks) return fail(SCOPE_EINVAL, "block_kind: %d blocks > %d", nb, kMaxBlocks);
        if (p->c_q < 1 || p->c_q > N || p->c_q > kMaxClusters)
            return fail(SCOPE_EINVAL, "params: c_q must be in [1, min(N, %d)]", kMaxClusters);
        return SCOPE_OK;
    }
    if (p->compensate && p->fixed_cluster_size == 0)
        return fail(SCOPE_EINVAL, "params: compensate needs the ClusterAttention variant (fixed_cluster_size > 0)");
    if (p->fixed_cluster_size > 0) {
        const int64_t f = p->fixed_cluster_size;
        if (has_grid) return fail(SCOPE_EINVAL, "fixed_cluster_size needs grid {0,0,0} (no RoPE)");
        if (ds[0] != D) return fail(SCOPE_ESHAPE, "fixed_cluster_size needs d_t == D, d_h == d_w == 0");
        if (N % f) return fail(SCOPE_ESHAPE, "fixed_cluster_size must divide N");
        int64_t m = N / f;
        while (m > 1 && !(m & 1)) m >>= 1;
        if (m != 1) return fail(SCOPE_ESHAPE, "N / fixed_cluster_size must be a power of two");
        const int64_t Cn = N / f;
        if (Cn > kMaxClusters) return fail(SCOPE_EINVAL, "N / fixed_cluster_size must be <= %d", kMaxClusters);
        if ((p->c_q != 0 && p->c_q != Cn) || (p->c_t != 0 && p->c_t != Cn))
            return fail(SCOPE_EINVAL, "c_q and c_t must be 0 or N / fixed_cluster_size");
        return SCOPE_OK;
    }
    if (p->c_q < 1 || p->c_q > N || p->c_q > kMaxClusters)
        return fail(SCOPE_EINVAL, "params: c_q must be in [1, min(N, %d)]", kMaxClusters);
    int64_t P = 1;
    for (int s = 0; s < 3; ++s) {
        if (C[s] < 1 || C[s] > N || C[s] > kMaxClusters)
            return fail(SCOPE_EINVAL, "params: c_t/c_h/c_w must be in [1, min(N, %d)]", kMaxClusters);
        if (ds[s] == 0 && C[s] != 1) return fail(SCOPE_EINVAL, "params: a 0-wide subspace needs 1 cluster");
        P *= C[s];
    }
    if (P > kMaxItems) return fail(SCOPE_EINVAL, "params: c_t*c_h*c_w must be <= %d", kMaxItems);
    return SCOPE_OK;
}

Layout make_layout(const scope_tensor *q, const scope_grid *g, const scope_params *p)
{
    Layout L{};
    L.B = q->B; L.H = q->H; L.N = q->N; L.D = q->D; L.BH = L.B * L.H;
    L.f32 = q->dtype == SCOPE_F32;
    L.bisect = p->fixed_cluster_size > 0;
    const int ds[3] = {p->d_t, p->d_h, p->d_w};
    L.blocks = p->block_kind > 0;
    if (L.bisect) {
        const int Cn = (int)(L.N / p->fixed_cluster_size);
        L.Cq = Cn;
        L.C[0] = Cn; L.C[1] = 1; L.C[2] = 1;
    } else if (L.blocks) {
        L.Cq = p->c_q;
        L.C[0] = block_count(g->T, g->Hh, g->W, p->block_kind, p->block_t, p->block_h, p->block_w);
        L.C[1] = 1; L.C[2] = 1;
    } else {
        L.Cq = p->c_q;
        L.C[0] = p->c_t; L.C[1] = p->c_h; L.C[2] = p->c_w;
    }
    for (int s = 0; s < 3; ++s) L.ds[s] = ds[s];
    if (L.blocks) {  // one "subspace": the whole rotated key, one centroid per block
        L.ds[0] = (int)L.D; L.ds[1] = 0; L.ds[2] = 0;
    }
    L.off[0] = 0; L.off[1] = L.ds[0]; L.off[2] = L.ds[0] + L.ds[1];
    L.Csum = L.C[0] + L.C[1] + L.C[2];
    L.P = L.C[0] * L.C[1] * L.C[2];
    L.Pcap = (int)(L.P < L.N ? L.P : L.N);
    L.nblk = (int)((L.N + kSortBlk - 1) / kSortBlk);
    L.max_work = attn_tc_max_items((int)L.BH, (int)L.N, L.Cq);
    const int T = g ? g->T : 0, Hh = g ? g->Hh : 0, W = g ? g->W : 0;
    L.maxL = T > Hh ? T : Hh;
    L.maxL = L.maxL > W ? L.maxL : W;
    if (L.maxL < 1) L.maxL = 1;
    L.maxP = 1;
    for (int s = 0; s < 3; ++s) L.maxP = ds[s] / 2 > L.maxP ? ds[s] / 2 : L.maxP;
    L.cap = L.BH * L.Cq * L.N;
    const int64_t BH = L.BH, N = L.N, D = L.D;
    size_t cur = 0;
    // Qr then Kr with no gap (a whole bisection runs over both as 2*BH row
    // sets); BH*N*D*2 is a multiple of 128 bytes, so Kr stays aligned
    L.qr = take(cur, 2 * BH * N * D * 2);
    L.kr = L.qr + BH * N * D * 2;
    L.qnorm = take(cur, BH * N * 4);
    L.ksub2 = take(cur, BH * N * 16);
    L.kchi = take(cur, BH * 128 * D * 2);
    L.kclo = take(cur, BH * 128 * D * 2);
    L.kfix = take(cur, 3 * (4 + BH * N) * 4);
    L.tab = take(cur, (size_t)3 * L.maxL * L.maxP * 16);
    L.stats = take(cur, 64);
    L.maxabs = take(cur, 2 * BH * 4);
    L.q_lab = take(cur, BH * N * 4);
    L.q_cent = take(cur, BH * L.Cq * D * 4);
    L.q_cn = take(cur, BH * L.Cq * 4);
    L.q_sizes = take(cur, BH * L.Cq * 4);
    L.q_perm = take(cur, BH * N * 4);
    L.q_start = take(cur, BH * (L.Cq + 1) * 4);
    L.q_bhist = take(cur, BH * L.Cq * L.nblk * 4);
    L.q_tsum = take(cur, BH * scan_tiles(L.Cq, L.nblk) * 4);
    L.fix = take(cur, BH * N * 4 + 16);
    L.q_chi = take(cur, BH * L.Cq * D * 2);
    L.q_clo = take(cur, BH * L.Cq * D * 2);
    {
        // fixed-point centroid sums of every k-means problem, one zeroed region
        const size_t s0 = cur;
        L.q_sums = take(cur, BH * L.Cq * D * 8);
        for (int i = 0; i < 3; ++i) L.k_sums[i] = take(cur, BH * L.C[i] * (L.ds[i] > 0 ? L.ds[i] : 1) * 8);
        L.sums_bytes = cur - s0;
    }
    L.bis_order = take(cur, L.bisect ? 4 * BH * N * 4 : 0);  // order + scratch for 2*BH row sets
    L.bis_delta = take(cur, L.bisect ? 2 * BH * N * 8 : 0);
    L.bis_aux = take(cur, L.bisect ? bisect_aux_bytes((int)(2 * BH), (int)N, (int)D) : 0);
    L.comp = p->compensate != 0;
    L.k_codes = take(cur, 3 * BH * N * 4);
    for (int s = 0; s < 3; ++s) {
        L.k_cent[s] = take(cur, BH * L.C[s] * (L.ds[s] > 0 ? L.ds[s] : 1) * 4);
        L.k_cn[s] = take(cur, BH * L.C[s] * 4);
        L.k_sizes[s] = take(cur, BH * L.C[s] * 4);
        L.k_perm[s] = take(cur, BH * N * 4);
        L.k_start[s] = take(cur, BH * (L.C[s] + 1) * 4);
        L.k_bhist[s] = take(cur, BH * L.C[s] * L.nblk * 4);
        L.k_tsum[s] = take(cur, BH * scan_tiles(L.C[s], L.nblk) * 4);
    }
    L.lut = take(cur, BH * L.Cq * L.Csum * 4);
    L.sel_state = take(cur, selection_state_bytes(BH * L.Cq));
    L.eg = p->eg_tau > 0.f;
    L.eg_state = take(cur, L.eg ? eg_state_bytes(L.B, L.H, L.Cq, p->eg_group) : 0);
    L.item_hist = take(cur, BH * L.P * 4);
    L.item_id = take(cur, BH * L.Pcap * 4);
    L.item_cnt = take(cur, BH * L.Pcap * 4);
    L.item_n = take(cur, BH * 4);
    L.key_item = take(cur, BH * N * 2);
    L.r = take(cur, BH * L.Cq * 4);
    L.n = take(cur, BH * L.Cq * 4);
    L.kh = take(cur, BH * 4);
    L.offsets = take(cur, (BH * L.Cq + 1) * 8);
    L.work = take(cur, (size_t)L.max_work * 16);
    L.nwork = take(cur, 16);
    L.vb = take(cur, L.f32 ? BH * N * D * 2 : 0);
    L.indices = take(cur, (size_t)L.cap * 4);
    // ClusterAttention leaves of 32 or 64 queries: 256 / leaf consecutive
    // leaves share one attention work item over the union of their lists
    L.gL = 0;
    if (L.bisect && (p->fixed_cluster_size == 32 || p->fixed_cluster_size == 64)) {
        const int gl = 256 / p->fixed_cluster_size;
        if (L.Cq % gl == 0) {
            L.gL = gl;
            L.gshift = p->fixed_cluster_size == 32 ? 5 : 6;
            L.G = L.Cq / gl;
        }
    }
    L.u_idx = take(cur, L.gL ? (size_t)L.cap * 4 : 0);
    L.u_n = take(cur, L.gL ? (size_t)BH * L.G * 4 : 0);
    L.gmask = take(cur, L.gL ? pack_mask_bytes(L.cap, (int)BH, L.G, L.gL) : 0);
    // compensation: virtual groups follow the attention's work items (a
    // group of leaves when grouped, else one query cluster)
    L.Lv = L.gL ? L.gL : 1;
    L.vtiles = L.comp ? virt_tiles(L.C[0]) : 0;
    {
        const size_t tabs = L.comp ? (size_t)BH * L.C[0] * D * 2 : 0;
        const size_t groups = L.comp ? (size_t)BH * (L.Cq / L.Lv) : 0;
        L.vk_hi = take(cur, tabs);
        L.vk_lo = take(cur, tabs);
        L.vv_hi = take(cur, tabs);
        L.vv_lo = take(cur, tabs);
        L.vlist = take(cur, groups * L.vtiles * 64 * 4);
        L.vn = take(cur, groups * 4);
        L.vbias = take(cur, groups * L.vtiles * L.Lv * 64 * 4);
    }
    L.total = cur;
    return L;
}

scope_status check_device(cudaStream_t)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(SCOPE_EDEVICE, "no CUDA device");
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10)
        return fail(SCOPE_EDEVICE, "libscope.so is built for sm_100a; device has compute capability %d.x", major);
    static bool configured[64] = {false};
    if (dev < 64 && !configured[dev]) {
        if (km_configure() != cudaSuccess || attn_tc_configure() != cudaSuccess || km_tc_configure() != cudaSuccess ||
            select_configure() != cudaSuccess)
            return fail(SCOPE_ECUDA, "kernel attribute setup failed");
        configured[dev] = true;
    }
    return SCOPE_OK;
}

scope_status launch_status(const char *what)
{
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(SCOPE_ECUDA, "%s: %s", what, cudaGetErrorString(e));
    return SCOPE_OK;
}

}  // namespace

struct scope_plan_s {
    Layout L;
    char *ws;
    size_t ws_bytes;
    const void *q_ptr, *k_ptr;
    scope_dtype dtype;
    scope_params p;
    scope_grid g;
};

template <typename T>
static T *at(char *ws, size_t off)
{
    return reinterpret_cast<T *>(ws + off);
}

extern "C" size_t scope_plan_workspace_bytes(const scope_tensor *q, const scope_grid *grid,
                                             const scope_params *p)
{
    scope_status st;
    if (!tensor_ok(q, "q", &st)) return 0;
    if (check_params(q, grid, p) != SCOPE_OK) return 0;
    return make_layout(q, grid, p).total;
}

static void rope_both(const Layout &L, char *ws, const scope_tensor *q, const scope_tensor *k, const scope_grid *g,
                      const scope_params *p, cudaStream_t st)
{
    const bool rope = g && g->T > 0;
    uint32_t *stats = at<uint32_t>(ws, L.stats);
    uint32_t *maxabs = at<uint32_t>(ws, L.maxabs);
    cudaMemsetAsync(stats, 0, 64, st);
    cudaMemsetAsync(maxabs, 0, 2 * L.BH * 4, st);
    if (rope)
        launch_rope_table(at<double2>(ws, L.tab), g->T, g->Hh, g->W, p->d_t, p->d_h, p->d_w, p->theta, L.maxL, L.maxP,
                          st);
    const int Hh = rope ? g->Hh : 1, W = rope ? g->W : 1;
    launch_rope_apply(q->ptr, rows_of(q), L.f32, at<__nv_bfloat16>(ws, L.qr), at<float>(ws, L.qnorm), nullptr, maxabs,
                      at<double2>(ws, L.tab), L.BH * L.N, (int)L.N, (int)L.D, Hh, W, p->d_t, p->d_h, L.maxL, L.maxP,
                      rope ? 1 : 0, st);
    launch_rope_apply(k->ptr, rows_of(k), L.f32, at<__nv_bfloat16>(ws, L.kr), nullptr,
                      L.ksub2 ? at<float4>(ws, L.ksub2) : nullptr, maxabs + L.BH, at<double2>(ws, L.tab),
                      L.BH * L.N, (int)L.N, (int)L.D, Hh, W, p->d_t, p->d_h, L.maxL, L.maxP, rope ? 1 : 0, st);
}

static KmProblem key_problem(const Layout &L, char *ws, int s)
{
    KmProblem P{};
    P.X = at<__nv_bfloat16>(ws, L.kr);
    P.maxabs = at<uint32_t>(ws, L.maxabs) + L.BH;
    P.dim_off = L.off[s];
    P.dim_n = L.ds[s];
    P.C = L.C[s];
    P.labels = at<int32_t>(ws, L.k_codes) + (int64_t)s * L.BH * L.N;
    P.cent = at<float>(ws, L.k_cent[s]);
    P.cn = at<float>(ws, L.k_cn[s]);
    P.sizes = at<int32_t>(ws, L.k_sizes[s]);
    P.perm = at<int32_t>(ws, L.k_perm[s]);
    P.start = at<int32_t>(ws, L.k_start[s]);
    P.blockhist = at<int32_t>(ws, L.k_bhist[s]);
    P.tilesum = at<int32_t>(ws, L.k_tsum[s]);
    P.sums = at<unsigned long long>(ws, L.k_sums[s]);
    return P;
}

static KmProblem query_problem(const Layout &L, char *ws)
{
    KmProblem P{};
    P.X = at<__nv_bfloat16>(ws, L.qr);
    P.maxabs = at<uint32_t>(ws, L.maxabs);
    P.dim_off = 0;
    P.dim_n = (int)L.D;
    P.C = L.Cq;
    P.labels = at<int32_t>(ws, L.q_lab);
    P.cent = at<float>(ws, L.q_cent);
    P.cn = at<float>(ws, L.q_cn);
    P.sizes = at<int32_t>(ws, L.q_sizes);
    P.perm = at<int32_t>(ws, L.q_perm);
    P.start = at<int32_t>(ws, L.q_start);
    P.blockhist = at<int32_t>(ws, L.q_bhist);
    P.tilesum = at<int32_t>(ws, L.q_tsum);
    P.sums = at<unsigned long long>(ws, L.q_sums);
    return P;
}

extern "C" scope_status scope_plan(const scope_tensor *q, const scope_tensor *k, const scope_grid *grid,
                                   const scope_params *p, void *workspace, size_t ws_bytes, void *stream,
                                   scope_plan_t **out)
{
    scope_status st;
    if (!out) return fail(SCOPE_EINVAL, "out: null");
    *out = nullptr;
    if (!tensor_ok(q, "q", &st) || !tensor_ok(k, "k", &st)) return st;
    if (!same_shape(q, k)) return fail(SCOPE_ESHAPE, "q and k shapes differ");
    if (q->dtype != k->dtype) return fail(SCOPE_EDTYPE, "q and k dtypes differ");
    if ((st = check_params(q, grid, p)) != SCOPE_OK) return st;
    const Layout L = make_layout(q, grid, p);
    if (!workspace) return fail(SCOPE_EWORKSPACE, "workspace: null");
    if (((uintptr_t)workspace) & 255) return fail(SCOPE_EALIGN, "workspace must be 256-byte aligned");
    if (ws_bytes < L.total)
        return fail(SCOPE_EWORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, L.total);
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = check_device(s)) != SCOPE_OK) return st;
    char *ws = (char *)workspace;
    const int BH = (int)L.BH, N = (int)L.N, D = (int)L.D;

    rope_both(L, ws, q, k, grid, p, s);

    if (L.bisect) {
        // ClusterAttention variant: balanced bisection of queries and of keys
        // into N / fixed_cluster_size clusters (one subspace = the full head dim).
        const int leaf = p->fixed_cluster_size;
        // Qr and Kr are adjacent in the workspace: one bisection over 2*BH row sets
        int32_t *ord = at<int32_t>(ws, L.bis_order);
        const BisectOut outs[2] = {
            {at<int32_t>(ws, L.q_lab), at<float>(ws, L.q_cent), at<float>(ws, L.q_cn), at<int32_t>(ws, L.q_start),
             at<int32_t>(ws, L.q_sizes), at<int32_t>(ws, L.q_perm)},
            {at<int32_t>(ws, L.k_codes), at<float>(ws, L.k_cent[0]), at<float>(ws, L.k_cn[0]),
             at<int32_t>(ws, L.k_start[0]), at<int32_t>(ws, L.k_sizes[0]), at<int32_t>(ws, L.k_perm[0])}};
        launch_bisect(at<__nv_bfloat16>(ws, L.qr), 2 * BH, N, D, leaf, p->iters, ord, ord + 2 * (int64_t)BH * N,
                      at<double>(ws, L.bis_delta), ws + L.bis_aux, outs, 2, s);
        cudaMemsetAsync(at<int32_t>(ws, L.k_codes) + (int64_t)BH * N, 0, (size_t)2 * BH * N * 4, s);
    } else {
    // Key subspaces always, and the queries when they have few clusters, run
    // as one batch on the direct-form kernel; queries with >= 128 clusters use
    // the certified tensor-core kernel (bf16 hi/lo centroid split, fp64 fix-up
    // of the rows inside its error margin).
    const bool tc_q = L.Cq >= 128;
    KmBatch all{};
    for (int i = 0; i < 3; ++i) all.p[i] = key_problem(L, ws, i);
    all.p[3] = query_problem(L, ws);
    all.count = 4;
    KmBatch keys = all;
    keys.count = 3;
    KmBatch qonly{};
    qonly.p[0] = all.p[3];
    qonly.count = 1;
    if (L.blocks) {
        // VMoBA block mode: only the queries are clustered; the keys' codes and
        // centroids come from the block partition
        all = qonly;
        keys.count = 0;
        launch_blocks(grid->T, grid->Hh, grid->W, p->block_kind, p->block_t, p->block_h, p->block_w,
                      at<__nv_bfloat16>(ws, L.kr), at<int32_t>(ws, L.k_codes), at<float>(ws, L.k_cent[0]),
                      at<float>(ws, L.k_cn[0]), at<int32_t>(ws, L.k_sizes[0]), BH, N, D, s);
    }
    int32_t *fix_count = at<int32_t>(ws, L.fix);
    int32_t *fix_list = fix_count + 4;
    bool tc_ok = true;
    // key subspaces on the tensor cores when their centroids fit one
    // 128-column block-diagonal chunk
    const bool tc_k = keys.count == 3 && L.C[0] + L.C[1] + L.C[2] <= 128;
    auto assign = [&]() {
        if (tc_k)
            tc_ok = tc_ok && launch_km_assign_keys_tc(keys.p, at<__nv_bfloat16>(ws, L.kchi),
                                                      at<__nv_bfloat16>(ws, L.kclo), BH, N, D,
                                                      at<float4>(ws, L.ksub2), at<int32_t>(ws, L.kfix),
                                                      at<int32_t>(ws, L.stats) + 4, s);
        if (tc_q) {
            if (keys.count && !tc_k) launch_km_assign_direct(keys, BH, N, D, s);
            tc_ok = tc_ok && launch_km_assign_tc(qonly.p[0], at<__nv_bfloat16>(ws, L.q_chi),
                                                 at<__nv_bfloat16>(ws, L.q_clo), BH, N, D, at<float>(ws, L.qnorm),
                                                 fix_list, fix_count, at<int32_t>(ws, L.stats) + 4, s);
        } else {
            launch_km_assign_direct(keys.count && !tc_k ? all : qonly, BH, N, D, s);
        }
        // fp64 re-decision of every tensor-core-assigned row inside its margin, one launch
        FixBatch fb{};
        if (tc_q) {
            fb.p[fb.n] = qonly.p[0];
            fb.list[fb.n] = fix_list;
            fb.count[fb.n] = fix_count;
            ++fb.n;
        }
        if (tc_k)
            for (int k = 0; k < 3; ++k)
                if (keys.p[k].C > 1) {
                    int32_t *kc = at<int32_t>(ws, L.kfix) + (int64_t)k * (4 + (int64_t)BH * N);
                    fb.p[fb.n] = keys.p[k];
                    fb.count[fb.n] = kc;
                    fb.list[fb.n] = kc + 4;
                    ++fb.n;
                }
        km_fixup_launch(fb, N, D, s);
    };
    cudaMemsetAsync(ws + L.q_sums, 0, L.sums_bytes, s);
    launch_km_init(all, BH, N, D, p->init_seed, s);
    for (int it = 0; it < p->iters; ++it) {
        assign();
        launch_km_sort(all, BH, N, s);
        launch_km_reduce(all, BH, N, D, s);
    }
    assign();
    launch_km_sort(qonly, BH, N, s);
    if (!tc_ok) return fail(SCOPE_ECUDA, "k-means: tensor map encoding failed");
    }
    if ((st = launch_status("k-means")) != SCOPE_OK) return st;

    launch_lut(at<float>(ws, L.q_cent), at<float>(ws, L.k_cent[0]), at<float>(ws, L.k_cent[1]),
               at<float>(ws, L.k_cent[2]), at<float>(ws, L.lut), BH, L.Cq, D, L.ds[0], L.ds[1], L.ds[2], L.C[0],
               L.C[1], L.C[2], s);
    launch_items(at<int32_t>(ws, L.k_codes), at<int32_t>(ws, L.item_hist), at<int32_t>(ws, L.item_id),
                 at<int32_t>(ws, L.item_cnt), at<int32_t>(ws, L.item_n), at<uint16_t>(ws, L.key_item), BH, N, L.C[1],
                 L.C[2], L.P, L.Pcap, s);
    run_selection(at<float>(ws, L.lut), at<int32_t>(ws, L.k_codes), at<int32_t>(ws, L.item_id),
                  at<int32_t>(ws, L.item_cnt), at<int32_t>(ws, L.item_n), at<uint16_t>(ws, L.key_item), L.Pcap, N,
                  L.Cq, L.C[0], L.C[1], L.C[2], BH, p->top_p, 1.0f / sqrtf((float)D), p->k_min,
                  at<int32_t>(ws, L.stats) + 4,
                  at<int32_t>(ws, L.q_sizes), at<int32_t>(ws, L.r), at<int32_t>(ws, L.n), at<int32_t>(ws, L.kh),
                  at<long long>(ws, L.offsets), at<int32_t>(ws, L.indices), p->online_topk, ws + L.sel_state, (int)L.B,
                  p->eg_tau, p->eg_group, L.eg ? ws + L.eg_state : nullptr, L.blocks ? 1 : 0, s);
    if (L.gL)
        launch_pack_lists(at<long long>(ws, L.offsets), at<int32_t>(ws, L.n), at<int32_t>(ws, L.indices),
                          at<int32_t>(ws, L.u_idx), at<int32_t>(ws, L.u_n), at<uint32_t>(ws, L.gmask), (int)BH, L.Cq,
                          L.gL, (int)N, s);
    if (L.comp)
        launch_virt_plan(at<float>(ws, L.k_cent[0]), at<__nv_bfloat16>(ws, L.vk_hi), at<__nv_bfloat16>(ws, L.vk_lo),
                         at<long long>(ws, L.offsets), at<int32_t>(ws, L.n), at<int32_t>(ws, L.indices),
                         at<int32_t>(ws, L.k_codes), at<int32_t>(ws, L.k_sizes[0]), at<int32_t>(ws, L.vlist),
                         at<int32_t>(ws, L.vn), at<float>(ws, L.vbias), (int)BH, (int)N, (int)D, L.Cq, L.C[0], L.Lv,
                         s);
    if ((st = launch_status("selection")) != SCOPE_OK) return st;

    scope_plan_s *h = (scope_plan_s *)malloc(sizeof(scope_plan_s));
    if (!h) return fail(SCOPE_EINVAL, "host allocation of the plan handle failed");
    h->L = L;
    h->ws = ws;
    h->ws_bytes = ws_bytes;
    h->q_ptr = q->ptr;
    h->k_ptr = k->ptr;
    h->dtype = q->dtype;
    h->p = *p;
    h->g = grid ? *grid : scope_grid{0, 0, 0};
    *out = h;
    return SCOPE_OK;
}

static scope_status check_vo(const scope_tensor *q, const scope_tensor *v, const scope_tensor *o)
{
    scope_status st;
    if (!tensor_ok(v, "v", &st) || !tensor_ok(o, "o", &st)) return st;
    if (!same_shape(q, v) || !same_shape(q, o)) return fail(SCOPE_ESHAPE, "v and o must have q's shape");
    if (o->dtype != SCOPE_BF16) return fail(SCOPE_EDTYPE, "o must be bf16");
    return SCOPE_OK;
}

// bf16 V for the attention: the caller's rows, or a contiguous bf16 copy of
// f32 ones in the workspace (`vs` receives the row addressing of either).
static const __nv_bfloat16 *v_bf16(const Layout &L, char *ws, const scope_tensor *v, RowStrides *vs, cudaStream_t s)
{
    if (v->dtype == SCOPE_BF16) {
        *vs = rows_of(v);
        return (const __nv_bfloat16 *)v->ptr;
    }
    __nv_bfloat16 *vb = at<__nv_bfloat16>(ws, L.vb);
    launch_to_bf16((const float *)v->ptr, rows_of(v), vb, L.BH * L.N * L.D, (int)L.N, (int)L.D, s);
    *vs = contiguous_rows(L.H, L.N, L.D);
    return vb;
}

extern "C" scope_status scope_attn(const scope_tensor *q, const scope_tensor *k, const scope_tensor *v,
                                   const scope_plan_t *plan, scope_tensor *o, void *stream)
{
    scope_status st;
    if (!plan) return fail(SCOPE_EINVAL, "plan: null");
    if (!tensor_ok(q, "q", &st) || !tensor_ok(k, "k", &st)) return st;
    const Layout &L = plan->L;
    if (q->ptr != plan->q_ptr || k->ptr != plan->k_ptr)
        return fail(SCOPE_EINVAL, "q and k must be the tensors the plan was made from");
    if (q->B != L.B || q->H != L.H || q->N != L.N || q->D != L.D || !same_shape(q, k))
        return fail(SCOPE_ESHAPE, "q/k shape differs from the plan's");
    if ((st = check_vo(q, v, o)) != SCOPE_OK) return st;
    if (v->dtype == SCOPE_F32 && !L.f32) return fail(SCOPE_EDTYPE, "f32 v needs a plan made from f32 q/k");
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = check_device(s)) != SCOPE_OK) return st;
    char *ws = plan->ws;
    RowStrides vs;
    const __nv_bfloat16 *vb = v_bf16(L, ws, v, &vs, s);
    const RowStrides os = rows_of(o);
    const GroupedLists grouped{at<int32_t>(ws, L.u_idx), at<int32_t>(ws, L.u_n), at<uint32_t>(ws, L.gmask), L.gL,
                               L.gshift};
    const CompLists comp{at<__nv_bfloat16>(ws, L.vk_hi), at<__nv_bfloat16>(ws, L.vk_lo),
                         at<__nv_bfloat16>(ws, L.vv_hi), at<__nv_bfloat16>(ws, L.vv_lo),
                         at<int32_t>(ws, L.vlist), at<int32_t>(ws, L.vn), at<float>(ws, L.vbias),
                         L.C[0], L.Lv, L.vtiles};
    if (L.comp)  // mean values of the key clusters: the compensation's virtual values
        launch_vmean(vb, vs, at<int32_t>(ws, L.k_perm[0]), at<int32_t>(ws, L.k_start[0]),
                     at<__nv_bfloat16>(ws, L.vv_hi), at<__nv_bfloat16>(ws, L.vv_lo), (int)L.BH, (int)L.N, (int)L.D,
                     L.C[0], s);
    if (!launch_attn_tc(at<__nv_bfloat16>(ws, L.qr), at<__nv_bfloat16>(ws, L.kr), vb, vs, (__nv_bfloat16 *)o->ptr, os,
                   at<int4>(ws, L.work), at<int32_t>(ws, L.nwork), L.max_work, at<int32_t>(ws, L.q_sizes),
                   at<int32_t>(ws, L.q_perm), at<int32_t>(ws, L.q_start), at<long long>(ws, L.offsets),
                   at<int32_t>(ws, L.indices), at<int32_t>(ws, L.n), at<int32_t>(ws, L.stats) + 4,
                   (int)L.BH, (int)L.N, (int)L.D, L.Cq, s, L.gL ? &grouped : nullptr, L.comp ? &comp : nullptr))
        return fail(SCOPE_ECUDA, "scope_attn: tensor map encoding failed");
    return launch_status("scope_attn");
}

// ---------------------------------------------------------------- dense baseline
static Layout dense_layout(const scope_tensor *q, const scope_grid *g, const scope_params *p)
{
    Layout L{};
    L.B = q->B; L.H = q->H; L.N = q->N; L.D = q->D; L.BH = L.B * L.H;
    L.f32 = q->dtype == SCOPE_F32;
    const int T = g ? g->T : 0, Hh = g ? g->Hh : 0, W = g ? g->W : 0;
    L.maxL = T > Hh ? T : Hh;
    L.maxL = L.maxL > W ? L.maxL : W;
    if (L.maxL < 1) L.maxL = 1;
    L.maxP = 1;
    const int ds[3] = {p ? p->d_t : 0, p ? p->d_h : 0, p ? p->d_w : 0};
    for (int s = 0; s < 3; ++s) L.maxP = ds[s] / 2 > L.maxP ? ds[s] / 2 : L.maxP;
    size_t cur = 0;
    L.qr = take(cur, L.BH * L.N * L.D * 2);
    L.kr = take(cur, L.BH * L.N * L.D * 2);
    L.qnorm = take(cur, L.BH * L.N * 4);
    L.tab = take(cur, (size_t)3 * L.maxL * L.maxP * 16);
    L.stats = take(cur, 64);
    L.maxabs = take(cur, 2 * L.BH * 4);
    L.vb = take(cur, L.f32 ? L.BH * L.N * L.D * 2 : 0);
    L.max_work = attn_tc_max_items((int)L.BH, (int)L.N, 0);
    L.work = take(cur, (size_t)L.max_work * 16);
    L.nwork = take(cur, 16);
    L.total = cur;
    return L;
}

extern "C" size_t scope_dense_workspace_bytes(const scope_tensor *q, const scope_grid *grid,
                                              const scope_params *p)
{
    scope_status st;
    if (!tensor_ok(q, "q", &st)) return 0;
    if (!p) {
        fail(SCOPE_EINVAL, "params: null");
        return 0;
    }
    const bool has_grid = grid && (grid->T || grid->Hh || grid->W);
    return dense_layout(q, has_grid ? grid : nullptr, p).total;
}

extern "C" scope_status scope_dense_attn(const scope_tensor *q, const scope_tensor *k, const scope_tensor *v,
                                         const scope_grid *grid, const scope_params *p, scope_tensor *o,
                                         void *workspace, size_t ws_bytes, void *stream)
{
    scope_status st;
    if (!tensor_ok(q, "q", &st) || !tensor_ok(k, "k", &st)) return st;
    if (!same_shape(q, k)) return fail(SCOPE_ESHAPE, "q and k shapes differ");
    if (q->dtype != k->dtype) return fail(SCOPE_EDTYPE, "q and k dtypes differ");
    if ((st = check_vo(q, v, o)) != SCOPE_OK) return st;
    if (v->dtype != q->dtype) return fail(SCOPE_EDTYPE, "v dtype must match q");
    if (!p) return fail(SCOPE_EINVAL, "params: null");
    const bool has_grid = grid && (grid->T || grid->Hh || grid->W);
    if (has_grid) {
        if (grid->T < 1 || grid->Hh < 1 || grid->W < 1 || (int64_t)grid->T * grid->Hh * grid->W != q->N)
            return fail(SCOPE_ESHAPE, "grid: T*Hh*W must equal N");
        if (p->d_t < 0 || p->d_h < 0 || p->d_w < 0 || (p->d_t | p->d_h | p->d_w) & 1 ||
            (int64_t)p->d_t + p->d_h + p->d_w != q->D)
            return fail(SCOPE_ESHAPE, "params: d_t/d_h/d_w must be even and sum to D");
        if (!(p->theta > 0.0)) return fail(SCOPE_EINVAL, "params: theta must be > 0");
    }
    const Layout L = dense_layout(q, has_grid ? grid : nullptr, p);
    if (!workspace) return fail(SCOPE_EWORKSPACE, "workspace: null");
    if (((uintptr_t)workspace) & 255) return fail(SCOPE_EALIGN, "workspace must be 256-byte aligned");
    if (ws_bytes < L.total) return fail(SCOPE_EWORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, L.total);
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = check_device(s)) != SCOPE_OK) return st;
    char *ws = (char *)workspace;
    rope_both(L, ws, q, k, has_grid ? grid : nullptr, p, s);
    RowStrides vs;
    const __nv_bfloat16 *vb = v_bf16(L, ws, v, &vs, s);
    if (!launch_attn_tc(at<__nv_bfloat16>(ws, L.qr), at<__nv_bfloat16>(ws, L.kr), vb, vs, (__nv_bfloat16 *)o->ptr,
                        rows_of(o), at<int4>(ws, L.work), at<int32_t>(ws, L.nwork), L.max_work, nullptr, nullptr, nullptr,
                        nullptr, nullptr, nullptr, at<int32_t>(ws, L.stats) + 4, (int)L.BH, (int)L.N,
                        (int)L.D, 1, s, nullptr, nullptr))
        return fail(SCOPE_ECUDA, "scope_dense_attn: tensor map encoding failed");
    return launch_status("scope_dense_attn");
}

// ---------------------------------------------------------------- views / status
extern "C" scope_status scope_plan_view(const scope_plan_t *plan, int which, scope_view *out)
{
    if (!plan || !out) return fail(SCOPE_EINVAL, "plan/out: null");
    const Layout &L = plan->L;
    char *ws = plan->ws;
    const int64_t B = L.B, H = L.H, N = L.N, D = L.D;
    scope_view v{};
    auto set = [&](size_t off, scope_dtype dt, int nd, int64_t a, int64_t b, int64_t c, int64_t d) {
        v.ptr = ws + off;
        v.dtype = dt;
        v.ndim = nd;
        v.shape[0] = a; v.shape[1] = b; v.shape[2] = c; v.shape[3] = d;
    };
    switch (which) {
    case SCOPE_VIEW_QR: set(L.qr, SCOPE_BF16, 4, B, H, N, D); break;
    case SCOPE_VIEW_KR: set(L.kr, SCOPE_BF16, 4, B, H, N, D); break;
    case SCOPE_VIEW_Q_LABELS: set(L.q_lab, SCOPE_I32, 3, B, H, N, 0); break;
    case SCOPE_VIEW_Q_CENTROIDS: set(L.q_cent, SCOPE_F32, 4, B, H, L.Cq, D); break;
    case SCOPE_VIEW_Q_SIZES: set(L.q_sizes, SCOPE_I32, 3, B, H, L.Cq, 0); break;
    case SCOPE_VIEW_Q_PERM: set(L.q_perm, SCOPE_I32, 3, B, H, N, 0); break;
    case SCOPE_VIEW_Q_START: set(L.q_start, SCOPE_I32, 3, B, H, L.Cq + 1, 0); break;
    case SCOPE_VIEW_K_CODES: set(L.k_codes, SCOPE_I32, 4, 3, B, H, N); break;
    case SCOPE_VIEW_K_CENT_T: set(L.k_cent[0], SCOPE_F32, 4, B, H, L.C[0], L.ds[0]); break;
    case SCOPE_VIEW_K_CENT_H: set(L.k_cent[1], SCOPE_F32, 4, B, H, L.C[1], L.ds[1]); break;
    case SCOPE_VIEW_K_CENT_W: set(L.k_cent[2], SCOPE_F32, 4, B, H, L.C[2], L.ds[2]); break;
    case SCOPE_VIEW_LUT: set(L.lut, SCOPE_F32, 4, B, H, L.Cq, L.Csum); break;
    case SCOPE_VIEW_R: set(L.r, SCOPE_I32, 3, B, H, L.Cq, 0); break;
    case SCOPE_VIEW_KH: set(L.kh, SCOPE_I32, 2, B, H, 0, 0); break;
    case SCOPE_VIEW_N: set(L.n, SCOPE_I32, 3, B, H, L.Cq, 0); break;
    case SCOPE_VIEW_OFFSETS: set(L.offsets, SCOPE_I64, 1, L.BH * L.Cq + 1, 0, 0, 0); break;
    case SCOPE_VIEW_INDICES: set(L.indices, SCOPE_I32, 1, L.cap, 0, 0, 0); break;
    case SCOPE_VIEW_ERROR: set(L.stats + 16, SCOPE_I32, 1, 4, 0, 0, 0); break;
    case SCOPE_VIEW_FIXUP: set(L.fix, SCOPE_I32, 1, 1, 0, 0, 0); break;
    case SCOPE_VIEW_GROUP_INDICES:
        if (!L.gL) return fail(SCOPE_EINVAL, "view: the plan has no grouped lists");
        set(L.u_idx, SCOPE_I32, 1, L.cap, 0, 0, 0);
        break;
    case SCOPE_VIEW_GROUP_N:
        if (!L.gL) return fail(SCOPE_EINVAL, "view: the plan has no grouped lists");
        set(L.u_n, SCOPE_I32, 3, B, H, L.G, 0);
        break;
    case SCOPE_VIEW_GROUP_MASKS:
        if (!L.gL) return fail(SCOPE_EINVAL, "view: the plan has no grouped lists");
        set(L.gmask, SCOPE_I32, 1, (int64_t)(pack_mask_bytes(L.cap, (int)L.BH, L.G, L.gL) / 4), 0, 0, 0);
        break;
    case SCOPE_VIEW_EG_ENTROPY:
        if (!L.eg) return fail(SCOPE_EINVAL, "no EG-Sparse routing in this plan (eg_tau = 0)");
        set(L.eg_state, SCOPE_F32, 2, B, H, 0, 0);
        break;
    case SCOPE_VIEW_EG_POOL:
        if (!L.eg) return fail(SCOPE_EINVAL, "no EG-Sparse routing in this plan (eg_tau = 0)");
        set(L.eg_state + L.BH * 4, SCOPE_I32, 2, B, H, 0, 0);
        break;
    default: return fail(SCOPE_EINVAL, "view id %d out of range", which);
    }
    *out = v;
    return SCOPE_OK;
}

extern "C" scope_status scope_sync_status(const scope_plan_t *plan, void *stream)
{
    if (!plan) return fail(SCOPE_EINVAL, "plan: null");
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return fail(SCOPE_ECUDA, "stream: %s", cudaGetErrorString(e));
    int32_t err[4] = {0, 0, 0, 0};
    e = cudaMemcpy(err, plan->ws + plan->L.stats + 16, sizeof err, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(SCOPE_ECUDA, "reading the error word: %s", cudaGetErrorString(e));
    if (err[0] & kErrTimeout) return fail(SCOPE_ETIMEOUT, "a bounded device wait gave up (detail 0x%x)", err[1]);
    if (err[0]) return fail(SCOPE_EDEVICE, "device range check fired (flags 0x%x, detail 0x%x)", err[0], err[1]);
    return SCOPE_OK;
}

extern "C" scope_status scope_selftest_wait_timeout(const scope_plan_t *plan, int64_t wait_cycles, void *stream)
{
    if (!plan) return fail(SCOPE_EINVAL, "plan: null");
    if (wait_cycles < 1000 || wait_cycles > 4000000000ll)
        return fail(SCOPE_EINVAL, "wait_cycles must be in [1e3, 4e9]");
    scope_status st;
    if ((st = check_device((cudaStream_t)stream)) != SCOPE_OK) return st;
    launch_wait_timeout((int32_t *)(plan->ws + plan->L.stats + 16), (long long)wait_cycles, (cudaStream_t)stream);
    return launch_status("scope_selftest_wait_timeout");
}

extern "C" void scope_plan_destroy(scope_plan_t *plan) { free(plan); }
