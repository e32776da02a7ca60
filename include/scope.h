/*
 * scope.h -- C ABI of libscope.so: centroid-guided sparse attention over
 * spatiotemporal tokens, in the formulation of
 *   "SCOPE: Subspace Clustering with Online Per-Head Top-K Estimation for
 *    Sparse Video Attention" (abstract)
 * with the fixed-size-cluster variant of
 *   "ClusterAttention: A training-free speedup of bidirectional attention"
 *    (abstract: power-of-two cluster sizes, block-sparse attention).
 *
 * Conventions for every entry point
 *   - Tensors are DEVICE memory owned by the caller, logical shape
 *     [B, H, N, D] (D is 64 or 128) with element strides (see scope_tensor);
 *     every row of D elements is contiguous and starts on a 16-byte boundary.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All device work is enqueued on it; no call synchronises the
 *     host except scope_sync_status.
 *   - The library never allocates device memory: scratch comes from the
 *     caller's workspace, sized by the matching *_workspace_bytes call.
 *   - Argument errors are detected on the host before any launch and return
 *     a non-zero scope_status; scope_last_error() then holds a message
 *     (thread-local, valid until the next call on the same thread).
 *   - Device-side anomalies (an index out of range, a bounded wait that ran
 *     out) set an error word inside the workspace; scope_sync_status reads it.
 */
#ifndef SCOPE_H
#define SCOPE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SCOPE_OK = 0,
    SCOPE_EINVAL = 1,     /* bad parameter value (p, counts, null pointer) */
    SCOPE_ESHAPE = 2,     /* inconsistent shapes (grid vs N, split vs D)    */
    SCOPE_EDTYPE = 3,     /* unsupported or mismatched dtypes               */
    SCOPE_EALIGN = 4,     /* pointer not 16-byte aligned                    */
    SCOPE_EWORKSPACE = 5, /* workspace missing or smaller than required     */
    SCOPE_ECAPACITY = 6,  /* a device-side capacity was exceeded            */
    SCOPE_ECUDA = 7,      /* a CUDA runtime call or launch failed           */
    SCOPE_ETIMEOUT = 8,   /* a bounded device wait gave up                  */
    SCOPE_EDEVICE = 9     /* no sm_100 device, or a device-side range check */
} scope_status;

typedef enum {
    SCOPE_F32 = 0,
    SCOPE_BF16 = 1,
    SCOPE_I32 = 2,
    SCOPE_I64 = 3
} scope_dtype;

/* A caller-owned device tensor of logical shape [B, H, N, D].
 *   strides  element strides of the B, H, N and D dimensions.  strides[3]
 *            must be 1 (a row of D elements is contiguous); strides[0..2]
 *            must be >= 0 and keep every row start 16-byte aligned
 *            (multiples of 8 elements for bf16, of 4 for f32), and distinct
 *            (b, h, n) must not share a row.  All four zero means the
 *            contiguous layout {H*N*D, N*D, D, 1}.  Any other layout (for
 *            example [B, N, H, D] memory seen as [B, H, N, D], or every
 *            second head of a larger tensor) is read and written in place.
 *            scope_kmeans_noalloc takes contiguous x only.
 *   A layout outside these rules returns SCOPE_ESHAPE before any launch. */
typedef struct {
    void *ptr;
    scope_dtype dtype;
    int64_t B, H, N, D;
    int64_t strides[4];
} scope_tensor;

/* Latent grid of the tokens: token n sits at (t, y, x) with
 * n = (t*Hh + y)*W + x.  {0,0,0} = no grid (no RoPE). */
typedef struct {
    int32_t T, Hh, W;
} scope_grid;

/* Parameters of one call (SCOPE abstract; the readings of what it leaves
 * open are listed per field).
 *   d_t, d_h, d_w  head-dim split into the temporal / height / width RoPE
 *                  blocks and key subspaces, contiguous in that order; each
 *                  even; d_t + d_h + d_w == D.  A block may be 0 wide.
 *   theta          RoPE base: pair i of a block of width d_s turns by
 *                  pos * theta^(-2i/d_s).
 *   c_q            query clusters (1 <= c_q <= min(N, 1024)).
 *   c_t, c_h, c_w  key-subspace clusters (1 <= c_s <= N; 1 for a 0-wide
 *                  block); c_t*c_h*c_w <= 65536.
 *   iters          Lloyd rounds (assign, update) before the final assign.
 *   init_seed      strided init offset: centroid j starts at row
 *                  (seed mod floor(N/C)) + j*floor(N/C).
 *   top_p          0 < top_p <= 1: keep the shortest score-ordered key
 *                  prefix holding top_p of the softmax(score/sqrt(D)) mass.
 *   k_min          fixed Top-k floor of the hybrid rule (>= 0).
 *   online_topk    1: per-head Top-k K_h = ceil(size-weighted mean of the
 *                  retained counts); clusters below it are topped up.
 *   fixed_cluster_size  > 0: ClusterAttention variant.  Requires no grid,
 *                  d_t == D, d_h == d_w == 0, N == fixed_cluster_size * 2^L;
 *                  queries and keys are each split by balanced recursive
 *                  2-means bisection into N / fixed_cluster_size clusters
 *                  (c_q and c_t are then taken as that count; pass 0 or it).
 *   compensate     0 or 1.  1 (ClusterAttention variant only, and at most
 *                  1024 key clusters): scope_attn adds every excluded key
 *                  through its key cluster's mean key and mean value
 *                  ("ClusterAttention: A training-free speedup of
 *                  bidirectional attention", abstract: compensation of
 *                  excluded clusters through their mean).  Reading: the
 *                  m_ck members of key cluster k missing from query cluster
 *                  c's list add m_ck * e^{q.mu_k/sqrt(D)} to the softmax
 *                  denominator and that times the mean value to the
 *                  numerator.  The attention computes these terms in the
 *                  same online softmax, as extra keys (mu_k, vbar_k) whose
 *                  logits carry ln m_ck.
 *   eg_tau, eg_group  EG-Sparse routing ("EG-Sparse", abstract: low-entropy
 *                  heads go to a grouped cross-head pool, high-entropy heads
 *                  keep per-row selection).  eg_tau <= 0: off (plain SCOPE
 *                  selection).  Otherwise a head's entropy E_h is the
 *                  query-weighted mean entropy of its clusters' proxy
 *                  softmax rows over ln N (0..1); heads with E_h < eg_tau
 *                  are grouped eg_group at a time in index order (per batch
 *                  entry, 1 <= eg_group <= 64), and a group's low-entropy
 *                  heads take their Top-p counts from one pool: every (head,
 *                  cluster, key) entry competes by its row's proxy
 *                  probability and the shortest prefix reaching top_p of
 *                  the pool's mass (each entry weighing its cluster's query
 *                  count) is kept.  k_min, the online Top-k and the lists
 *                  then follow as for the other heads.
 *   block_kind     VMoBA block-granular selection ("VMoBA: Mixture-of-Block
 *                  Attention for Video Diffusion Models", abstract: a
 *                  layer-wise recurrent 1D-2D-3D block partition, and blocks
 *                  chosen by a threshold on their cumulative similarity).
 *                  0: off (per-key SCOPE selection).  1, 2, 3: keys are
 *                  grouped into blocks -- 1: runs of block_t*block_h*block_w
 *                  tokens in raster order; 2: block_h x block_w tiles inside
 *                  each frame; 3: block_t x block_h x block_w cubes (ragged
 *                  edges; the caller cycles the kind with the layer index) --
 *                  in place of the key-subspace clustering.  Each block is
 *                  scored for query cluster c by q_c . (mean of its rotated
 *                  keys); blocks are kept by descending score until their
 *                  size-weighted softmax(score/sqrt(D)) mass reaches top_p,
 *                  whole blocks only (blocks tied with the last kept one are
 *                  kept too).  Needs a grid, at most 16384 blocks, k_min = 0,
 *                  online_topk = 0, eg_tau = 0 and no fixed_cluster_size;
 *                  c_t, c_h, c_w are not used. */
typedef struct {
    int32_t d_t, d_h, d_w;
    double theta;
    int32_t c_q, c_t, c_h, c_w;
    int32_t iters;
    uint32_t init_seed;
    float top_p;
    int32_t k_min;
    int32_t online_topk;
    int32_t fixed_cluster_size;
    int32_t compensate;
    float eg_tau;
    int32_t eg_group;
    int32_t block_kind;
    int32_t block_t, block_h, block_w;
} scope_params;

typedef struct scope_plan_s scope_plan_t; /* opaque host handle */

/* Bytes of device workspace scope_plan needs for this shape, grid and
 * parameters (worst case: the selected-key lists are sized for every key
 * of every cluster, so no call ever waits on the device for a size).
 * Returns 0 if the arguments are invalid (see scope_last_error). */
size_t scope_plan_workspace_bytes(const scope_tensor *q, const scope_grid *grid,
                                  const scope_params *p);

/* Steps 1-4 of SCOPE (abstract): 3D-RoPE of q and k; k-means of each key
 * subspace (codes, centroids) and of the queries (labels, centroids, sizes);
 * centroid-dot lookup tables; per-key proxy scores; hybrid Top-p / k_min
 * counts; online per-head Top-k; per-cluster selected-key index lists.
 *   q, k       [B,H,N,D] f32 or bf16 (same dtype), device.
 *   grid       token grid (T*Hh*W == N) or {0,0,0}.
 *   workspace  device, >= scope_plan_workspace_bytes bytes, 256-B aligned;
 *              owned by the caller, must outlive the plan; every result
 *              lives in it (read them with scope_plan_view).
 *   out        receives a host handle (malloc'd; free with
 *              scope_plan_destroy).  Returned before the device finishes. */
scope_status scope_plan(const scope_tensor *q, const scope_tensor *k,
                        const scope_grid *grid, const scope_params *p,
                        void *workspace, size_t ws_bytes, void *stream,
                        scope_plan_t **out);

/* Step 5 of SCOPE (abstract): "sparse attention is then computed over the
 * selected original keys and values".  Each query attends, with softmax
 * scale 1/sqrt(D), over the selected keys of its cluster, using the plan's
 * post-RoPE q and k (bf16) and the caller's v.
 *   q, k   the tensors given to scope_plan (checked by pointer and shape).
 *   v      [B,H,N,D] f32 or bf16, device.
 *   o      [B,H,N,D] bf16, device, written in full. */
scope_status scope_attn(const scope_tensor *q, const scope_tensor *k,
                        const scope_tensor *v, const scope_plan_t *plan,
                        scope_tensor *o, void *stream);

/* Dense baseline: 3D-RoPE of q and k, then softmax attention of every query
 * over every key, on the same tensor-core pipeline as scope_attn.
 *   workspace  >= scope_dense_workspace_bytes(q) bytes. */
size_t scope_dense_workspace_bytes(const scope_tensor *q, const scope_grid *grid,
                                   const scope_params *p);
scope_status scope_dense_attn(const scope_tensor *q, const scope_tensor *k,
                              const scope_tensor *v, const scope_grid *grid,
                              const scope_params *p, scope_tensor *o,
                              void *workspace, size_t ws_bytes, void *stream);

/* Results of a plan, as views into its workspace (no copy). */
typedef enum {
    SCOPE_VIEW_QR = 0,          /* bf16 [B,H,N,D] post-RoPE queries        */
    SCOPE_VIEW_KR = 1,          /* bf16 [B,H,N,D] post-RoPE keys           */
    SCOPE_VIEW_Q_LABELS = 2,    /* i32  [B,H,N]   query cluster of a token */
    SCOPE_VIEW_Q_CENTROIDS = 3, /* f32  [B,H,c_q,D]                        */
    SCOPE_VIEW_Q_SIZES = 4,     /* i32  [B,H,c_q] queries per cluster      */
    SCOPE_VIEW_Q_PERM = 5,      /* i32  [B,H,N]   tokens, cluster by cluster, ascending inside */
    SCOPE_VIEW_Q_START = 6,     /* i32  [B,H,c_q+1] cluster starts in Q_PERM */
    SCOPE_VIEW_K_CODES = 7,     /* i32  [3,B,H,N] key code per subspace t,h,w */
    SCOPE_VIEW_K_CENT_T = 8,    /* f32  [B,H,c_t,d_t]                      */
    SCOPE_VIEW_K_CENT_H = 9,    /* f32  [B,H,c_h,d_h]                      */
    SCOPE_VIEW_K_CENT_W = 10,   /* f32  [B,H,c_w,d_w]                      */
    SCOPE_VIEW_LUT = 11,        /* f32  [B,H,c_q,c_t+c_h+c_w]              */
    SCOPE_VIEW_R = 12,          /* i32  [B,H,c_q] initial retained counts  */
    SCOPE_VIEW_KH = 13,         /* i32  [B,H]     per-head online Top-k    */
    SCOPE_VIEW_N = 14,          /* i32  [B,H,c_q] final key counts         */
    SCOPE_VIEW_OFFSETS = 15,    /* i64  [B*H*c_q+1] list starts in INDICES */
    SCOPE_VIEW_INDICES = 16,    /* i32  [capacity] selected keys, ascending per cluster */
    SCOPE_VIEW_ERROR = 17,      /* i32  [4] device error word              */
    SCOPE_VIEW_EG_ENTROPY = 18, /* f32  [B,H] EG-Sparse head entropy (eg_tau > 0) */
    SCOPE_VIEW_EG_POOL = 19,    /* i32  [B,H] pool of a routed head (b * ceil(H/eg_group) + h/eg_group), -1 if not routed */
    SCOPE_VIEW_FIXUP = 20,      /* i32  [1] rows the last tensor-core query assignment sent to the fp64 re-check */
    /* ClusterAttention leaves of 32 or 64 queries: L = 256 / leaf consecutive
     * leaves form a group that the attention serves as one work item. */
    SCOPE_VIEW_GROUP_INDICES = 21, /* i32 [capacity] ascending union of a group's lists, at the
                                      OFFSETS entry of its first leaf */
    SCOPE_VIEW_GROUP_N = 22,    /* i32  [B,H,c_q/L] union lengths          */
    SCOPE_VIEW_GROUP_MASKS = 23, /* u32 words: for union tile t (128 keys) of group g of flat
                                    head bh and leaf l of the group, 4 words at
                                    ((OFFSETS[first leaf] / 128 + bh*c_q/L + g + t) * L + l) * 4;
                                    bit i = key i of the tile is in leaf l's list */
    SCOPE_VIEW_COUNT = 24
} scope_view_id;

typedef struct {
    void *ptr;         /* device pointer into the workspace */
    scope_dtype dtype;
    int32_t ndim;
    int64_t shape[4];
} scope_view;

scope_status scope_plan_view(const scope_plan_t *plan, int which, scope_view *out);

/* Synchronises `stream` and reports the plan's device error word:
 * SCOPE_OK, SCOPE_EDEVICE (a range check fired), SCOPE_ETIMEOUT or
 * SCOPE_ECUDA (an asynchronous CUDA error). */
scope_status scope_sync_status(const scope_plan_t *plan, void *stream);

/* Failure-handling self-test (no counterpart on the pages).  Enqueues one
 * CTA that waits, with the same bounded mbarrier wait every tensor-core
 * kernel of the library uses, on a barrier nothing ever arrives on; after
 * `wait_cycles` SM clock cycles (1e3 .. 4e9; 2e6 is about a millisecond) the
 * wait gives up and sets the timeout bit of the plan's device error word,
 * as a stalled kernel would.  scope_sync_status(plan) then returns
 * SCOPE_ETIMEOUT.  Nothing faults or hangs and the CUDA context stays
 * usable; the plan's error word stays set (make a new plan to clear it). */
scope_status scope_selftest_wait_timeout(const scope_plan_t *plan, int64_t wait_cycles, void *stream);

/* Frees the host handle only; the workspace stays the caller's. */
void scope_plan_destroy(scope_plan_t *plan);

/* Message for the last non-OK status on this thread ("" if none). */
const char *scope_last_error(void);

/* Library version, for the binding's load check. */
int scope_version(void);

/* ---------------------------------------------------------------------- */
/* Clustering without device allocation.  The pages have no counterpart of  */
/* this entry point; it exists for callers that cannot allocate device      */
/* memory (a plain C program without an allocator, a server whose device    */
/* memory plan is fixed after start-up, a plug-in that may only touch the   */
/* buffers its host passes in).                                             */
/*                                                                          */
/* scope_kmeans_noalloc runs Lloyd k-means on columns                      */
/* [dim_off, dim_off + dim_n) of x with scope_plan's strided init, tie      */
/* rule, empty-cluster rule, final assign and per-head fixed-point centroid */
/* sums, assigning by the fp32 direct-form distance.  Given the plan's      */
/* rotated queries and C < 128 its labels and centroids equal the plan's    */
/* query clustering.  Where the plan assigns on the tensor cores (queries   */
/* at C >= 128; key subspaces whose clusters fit one 128-column chunk) it   */
/* decides labels exactly (certified margin, fp64 re-decision of near-ties) */
/* while this entry point keeps the fp32 direct form: a label can then      */
/* differ where a row's two nearest centroids lie within fp32 rounding of   */
/* each other, and later rounds follow from it.                             */
/*   x          bf16 [B,H,N,D] device, D in {64, 128} (e.g. post-RoPE rows). */
/*   labels     int32 [B,H,N] device, written (final assign).               */
/*   centroids  f32 [B,H,C,dim_n] device, written (after the last update).  */
/* Scratch: a fixed SCOPE_NOALLOC_SCRATCH_BYTES array inside the library,   */
/* held on every GPU that loads it until the process exits.  The first call */
/* on a device looks up that array's device address (make it before any    */
/* stream capture).  All calls share the array: calls whose device work     */
/* overlaps race and must be serialised by the caller.  A shape needing     */
/* more than the array (scope_kmeans_noalloc_scratch_bytes) returns         */
/* SCOPE_ECAPACITY before any launch.  Allocates nothing.                   */
/* ---------------------------------------------------------------------- */
#define SCOPE_NOALLOC_SCRATCH_BYTES (32u << 20)

size_t scope_kmeans_noalloc_scratch_bytes(int64_t B, int64_t H, int64_t N, int32_t C);
scope_status scope_kmeans_noalloc(const scope_tensor *x, int32_t dim_off, int32_t dim_n,
                                  int32_t C, int32_t iters, uint32_t init_seed,
                                  int32_t *labels, float *centroids, void *stream);

/* Number of kernels this library has launched in this process so far (all
 * devices, all threads); a diagnostic for launch accounting. */
int64_t scope_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* SCOPE_H */
