// Step 5 of SCOPE (abstract: "sparse attention is then computed over the
// selected original keys and values") on the 5th-generation tensor cores.
//
// One CTA = one work item = up to 256 queries of one query cluster (two
// 128-row Q tiles) against that cluster's selected-key list, walked in tiles
// of 128 keys.  Both Q tiles share every gathered K/V tile, which halves the
// K/V bytes per flop (the tiles come from L2: a head's K/V is 61 MB at 720p).
//
// Warp roles (384 threads; warp w runs on SM sub-partition w % 4, so each
// sub-partition hosts two softmax warps and at most one other busy warp):
//   warps 0-3  softmax / epilogue of Q tile 0 (one thread per query row)
//   warps 4-7  softmax / epilogue of Q tile 1
//   warp 8     idle (keeps the issuer off sub-partition 0)
//   warp 11    tcgen05.mma issuer (one lane), owns the TMEM allocation
//   warps 9-10 producer: Q rows and the listed K and V rows by coalesced
//              16-byte cp.async (16 lanes per 256-byte row) into 128B-swizzled
//              shared-memory tiles, 2 stages each; K and V have their own
//              full/empty barriers so K(j+1) can land while V(j) is in use.
//              (A tile::gather4 TMA producer measured ~7 B/clk per SM here,
//              which made the loads the bottleneck; the LSU gather does not.)
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D).
// S = Q K^T lands in TMEM (fp32); the softmax rows read it with tcgen05.ld,
// write P as packed bf16 over the first 64 columns of their S, and the
// issuer runs O += P V with P taken from TMEM and V from shared memory.
// Online softmax in base 2 with a lazy rescale: O and l are rescaled only
// when a row's max grows by more than 2^8, so P never exceeds 256.
//
// The softmax loads its 128-wide S row with four back-to-back tcgen05.ld
// (one wait) and keeps it in registers: a three-input max for the row max,
// then the scale/subtract and the row sum as packed f32x2 instructions on
// 64-bit registers.  (Moving a third of the exponentials to a cubic on the
// FMA pipe, and handing P to the issuer in two 64-key halves, were both
// slower here.)
//
// Every mbarrier wait is bounded (about two seconds of clock64); on timeout
// the thread records SCOPE's timeout bit in the device error word, the CTA
// abandons its work item, and all threads still meet at the final barrier
// so the TMEM is released.
#include "tcgen05.cuh"

namespace scope {

namespace tc {

constexpr int kThreads = 384;
constexpr int kMmaWarp = 11;
constexpr int BN = 128;       // keys per K/V tile
constexpr int BM = 128;       // rows per Q tile

// Byte offset of 16-byte chunk `c` (0 .. D/8-1) of row `r` in a [rows][D] bf16
// tile stored as D/64 column blocks of rows x 128 B, 128B-swizzled.
__device__ __forceinline__ uint32_t sw_off(int r, int c, int rows)
{
    return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

struct Args {
    const __nv_bfloat16 *qr, *kr, *v;
    __nv_bfloat16 *o;
    RowStrides vs, os;         // caller's V and O rows
    const int4 *items;         // (bh, cluster, first query, query count) per work item
    const int32_t *n_items;    // total work items
    const int32_t *perm;       // [BH][N] or null (dense: identity)
    const int32_t *start;      // [BH][Cq+1] or null
    const long long *offsets;  // [BH*Cq] or null (dense: all keys)
    const int32_t *indices;
    const int32_t *n_c;        // [BH][Cq] or null
    int32_t *err;
    // Grouped work items (ClusterAttention leaves of 32 or 64 queries): item =
    // (bh, group of L consecutive leaves), `indices` holds the groups' union
    // lists at their first leaf's offset, u_n their lengths, and gmask the
    // per-tile, per-leaf 128-bit membership masks (null: one cluster per item).
    const uint32_t *gmask;
    const int32_t *u_n;
    int L, leaf_shift, G;
    // Compensation of excluded key clusters (ClusterAttention, compensate = 1):
    // after its listed keys a work item walks "virtual" keys, one per key
    // cluster k with members outside a leaf's list, whose key and value are
    // the cluster's mean key mu_k and mean value vbar_k (each as a bf16
    // hi + lo pair, summed by two MMAs) and whose logit carries log2(m_k),
    // m_k the leaf's excluded members of k (-inf where m_k = 0).  Virtual
    // tiles hold 64 keys: rows 0-63 of a K/V stage the hi halves, 64-127 the
    // lo halves.  Per virtual group vg (the work item's group, or its cluster
    // when ungrouped): vn[vg] keys in tiles vg*vtiles .. of vlist (key
    // cluster ids, 64 per tile) and vbias ([tile][leaf][64]).
    const __nv_bfloat16 *vk_hi, *vk_lo, *vv_hi, *vv_lo;  // [BH][Ck][D]
    const int32_t *vlist, *vn;
    const float *vbias;
    int Ck, Lv, vtiles;
    int N, Cq;
    float scale_log2;          // log2(e) / sqrt(D)
};

template <int D, bool GROUPED, bool COMP>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(Args a)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzle atoms.
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int QT_BYTES = BM * D * 2;
    constexpr int KV_BYTES = BN * D * 2;
    unsigned char *sQ = sm;                      // 2 Q tiles
    unsigned char *sK = sm + 2 * QT_BYTES;       // 2 stages
    unsigned char *sV = sK + 2 * KV_BYTES;       // 2 stages

    __shared__ uint64_t bar_q, bar_k_full[2], bar_k_empty[2], bar_v_full[2], bar_v_empty[2], bar_s_full[2],
        bar_p_full[2], bar_o_final[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int item = blockIdx.x;
    int bh, c, q0, nq, grp = 0;
    if constexpr (GROUPED) {  // grid = BH * G: one item per (bh, group), all 256 rows
        bh = item / a.G;
        grp = item % a.G;
        c = grp * a.L;
        q0 = 0;
        nq = a.L << a.leaf_shift;
    } else {
        if (item >= *a.n_items) return;  // uniform for the CTA
        const int4 it = a.items[item];
        bh = it.x;
        c = it.y;
        q0 = it.z;
        nq = it.w;
    }
    const bool two = nq > BM;
    const int64_t base = (int64_t)bh * a.N;
    const __nv_bfloat16 *vbh = a.v + a.vs.bh_off(bh);
    const int64_t vsn = a.vs.sN;
    const int cstart = a.start ? a.start[(int64_t)bh * (a.Cq + 1) + c] : 0;
    const long long loff = a.indices ? a.offsets[(int64_t)bh * a.Cq + c] : 0;
    const int nk = GROUPED ? a.u_n[(int64_t)bh * a.G + grp] : a.indices ? a.n_c[(int64_t)bh * a.Cq + c] : a.N;
    // first mask slot of the group (kept disjoint across groups by the +item)
    const long long mslot = GROUPED ? loff / 128 + item : 0;
    if (GROUPED && nk <= 0) return;  // uniform; a group's leaves always hold keys
    const int ntiles = (nk + BN - 1) / BN;
    // virtual tiles (compensation) follow the listed keys' tiles
    const int64_t vg = GROUPED ? (int64_t)item : (int64_t)bh * a.Cq + c;
    const int64_t vt0 = COMP ? vg * a.vtiles : 0;
    const int ttot = ntiles + (COMP ? (a.vn[vg] + 63) / 64 : 0);

    if (threadIdx.x == 0) {
        // producer and softmax barriers take one arrival per warp (lane 0,
        // after the warp's own waits, fences and a __syncwarp)
        mbar_init(&bar_q, 2);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_k_full[i], 2);
            mbar_init(&bar_k_empty[i], 1);
            mbar_init(&bar_v_full[i], 2);
            mbar_init(&bar_v_empty[i], 1);
            mbar_init(&bar_s_full[i], 1);
            mbar_init(&bar_p_full[i], 4);
            mbar_init(&bar_o_final[i], 1);
        }
        abort_sh = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&tmem_base_sh)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int *abort_flag = &abort_sh;

    if (warp == 9 || warp == 10) {
        // ------------------------------------------------------------ producer
        // 64 threads; a warp instruction covers 32 / (D/8) whole rows, so
        // every 16-byte chunk request is part of a fully used 128-byte line.
        constexpr int CH = D / 8;           // 16-byte chunks per row
        constexpr int RPI = 64 / CH;         // rows per producer-wide pass
        const int pt = threadIdx.x - 9 * 32;
        const int ch = pt % CH, r0 = pt / CH;
        for (int qi0 = 0; qi0 < 2 * BM; qi0 += RPI) {
            const int qi = qi0 + r0, t = qi / BM, r = qi % BM;
            const bool ok = qi < nq;
            const int tok = ok ? (a.perm ? a.perm[base + cstart + q0 + qi] : q0 + qi) : 0;
            cp_async16(smem_u32(sQ + t * QT_BYTES) + sw_off(r, ch, BM), a.qr + (base + tok) * D + ch * 8, ok);
        }
        cp_async_commit();
        cp_async_wait_all();
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_q);
        // Rows past the list repeat the last listed key (finite V, masked P).
        // A tile's keys are read once, up front (independent loads), and
        // serve both its K and its V rows.
        constexpr int NR = BN / RPI;
        int keys[NR];
        auto load_keys = [&](int j) {
            if (COMP && j >= ntiles) {
                // virtual tile: rows r and r + 64 take slot r & 63 (padding
                // slots repeat a real cluster and carry a -inf bias)
#pragma unroll
                for (int i = 0; i < NR; ++i) keys[i] = a.vlist[(vt0 + j - ntiles) * 64 + ((i * RPI + r0) & 63)];
                return;
            }
            // the lists are read once: streaming loads (evict first from L2),
            // so they do not push the head's K/V rows out of L2
#pragma unroll
            for (int i = 0; i < NR; ++i) {
                const int kj = min(j * BN + i * RPI + r0, nk - 1);
                keys[i] = a.indices ? __ldcs(a.indices + loff + kj) : kj;
            }
        };
        auto issue = [&](unsigned char *dst_base, const __nv_bfloat16 *src, int64_t sn, int j) {
            const uint32_t dst = smem_u32(dst_base + (j & 1) * KV_BYTES);
#pragma unroll
            for (int i = 0; i < NR; ++i)
                cp_async16(dst + sw_off(i * RPI + r0, ch, BN), src + keys[i] * sn + ch * 8, true);
            cp_async_commit();
        };
        // virtual tiles: rows 0-63 the bf16 hi halves, rows 64-127 the lo halves
        auto issue_virtual = [&](unsigned char *dst_base, const __nv_bfloat16 *hi, const __nv_bfloat16 *lo, int j) {
            const uint32_t dst = smem_u32(dst_base + (j & 1) * KV_BYTES);
            const int64_t tb = (int64_t)bh * a.Ck * D;
#pragma unroll
            for (int i = 0; i < NR; ++i)
                cp_async16(dst + sw_off(i * RPI + r0, ch, BN), (i * RPI < 64 ? hi : lo) + tb + (int64_t)keys[i] * D + ch * 8,
                           true);
            cp_async_commit();
        };
        const __nv_bfloat16 *kbh = a.kr + base * D;
        auto issue_k = [&](int j) {
            if (COMP && j >= ntiles) issue_virtual(sK, a.vk_hi, a.vk_lo, j);
            else issue(sK, kbh, D, j);
        };
        auto issue_v = [&](int j) {
            if (COMP && j >= ntiles) issue_virtual(sV, a.vv_hi, a.vv_lo, j);
            else issue(sV, vbh, vsn, j);
        };
        load_keys(0);
        issue_k(0);
        issue_v(0);
        for (int j = 0; j < ttot; ++j) {
            const bool more = j + 1 < ttot;
            // in flight: K(j), V(j)
            cp_async_wait1();
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_k_full[j & 1]);
            if (more) {
                load_keys(j + 1);
                if (j + 1 >= 2 && !mbar_wait(&bar_k_empty[(j + 1) & 1], (((j + 1) >> 1) - 1) & 1, abort_flag, a.err,
                                             0x10))
                    break;
                issue_k(j + 1);
                cp_async_wait1();  // in flight: V(j), K(j+1)
            } else {
                cp_async_wait_all();
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_v_full[j & 1]);
            if (more) {
                if (j + 1 >= 2 && !mbar_wait(&bar_v_empty[(j + 1) & 1], (((j + 1) >> 1) - 1) & 1, abort_flag, a.err,
                                             0x11))
                    break;
                issue_v(j + 1);
            }
        }
        cp_async_wait_all();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(BN, false);
            const uint32_t id_qk64 = idesc_bf16(64, false);
            const uint32_t id_pv = idesc_bf16(D, true);
            const int nt = two ? 2 : 1;
            // descriptors of the first tile / stage; the start-address field
            // (bits 0-13, 16-byte units) takes the offsets as plain adds
            const uint64_t dq = sw128_desc(smem_u32(sQ), 16, 1024);
            const uint64_t dk = sw128_desc(smem_u32(sK), 16, 1024);
            const uint64_t dv = sw128_desc(smem_u32(sV), BN * 128, 1024);
            auto issue_qk = [&](int t, int j) {
                const uint64_t aq = dq + (uint64_t)((t * QT_BYTES) >> 4);
                const uint64_t bk = dk + (uint64_t)(((j & 1) * KV_BYTES) >> 4);
                if (COMP && j >= ntiles) {
                    // S[:, 0:64] = Q (K_hi + K_lo)^T: N = 64 over rows 0-63, then rows 64-127
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int k = 0; k < D / 16; ++k)
                            mma_ss(tmem + t * 128, aq + (uint64_t)(((k >> 2) * (BM * 128) + (k & 3) * 32) >> 4),
                                   bk + (uint64_t)(((k >> 2) * (BN * 128) + h * 64 * 128 + (k & 3) * 32) >> 4),
                                   id_qk64, h > 0 || k > 0);
                } else {
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        mma_ss(tmem + t * 128, aq + (uint64_t)(((k >> 2) * (BM * 128) + (k & 3) * 32) >> 4),
                               bk + (uint64_t)(((k >> 2) * (BN * 128) + (k & 3) * 32) >> 4), id_qk, k > 0);
                }
                mma_commit(&bar_s_full[t]);
                if (t == nt - 1) mma_commit(&bar_k_empty[j & 1]);
            };
            bool ok = mbar_wait(&bar_q, 0, abort_flag, a.err, 0x20) &&
                      mbar_wait(&bar_k_full[0], 0, abort_flag, a.err, 0x21);
            if (ok) {
                tc_fence_after();
                for (int t = 0; t < nt; ++t) issue_qk(t, 0);
            }
            for (int j = 0; ok && j < ttot; ++j) {
                const int s = j & 1;
                if (!mbar_wait(&bar_v_full[s], (j >> 1) & 1, abort_flag, a.err, 0x24)) break;
                const uint64_t bv = dv + (uint64_t)((s * KV_BYTES) >> 4);
                for (int t = 0; t < nt; ++t) {
                    if (!mbar_wait(&bar_p_full[t], j & 1, abort_flag, a.err, 0x22)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (COMP && j >= ntiles) {
                        // O += P[:, 0:64] (V_hi + V_lo): P's first 64 keys against rows 0-63, then 64-127
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ts(tmem + 256 + t * 128, tmem + t * 128 + (k & 3) * 8, bv + (uint64_t)((k * 2048) >> 4),
                                   id_pv, true);
                    } else {
#pragma unroll
                        for (int k = 0; k < BN / 16; ++k)
                            mma_ts(tmem + 256 + t * 128, tmem + t * 128 + k * 8, bv + (uint64_t)((k * 2048) >> 4),
                                   id_pv, (j > 0 || k > 0));
                    }
                    if (t == nt - 1) mma_commit(&bar_v_empty[s]);
                    if (j + 1 < ttot) {
                        if (t == 0 && !mbar_wait(&bar_k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, abort_flag, a.err,
                                                 0x23)) {
                            ok = false;
                            break;
                        }
                        issue_qk(t, j + 1);
                    } else {
                        mma_commit(&bar_o_final[t]);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax + epilogue
        const int t = warp >> 2;           // Q tile of this warpgroup
        const int wq = warp & 3;           // TMEM lane quarter
        const int row = wq * 32 + lane;    // row of the Q tile
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_off + t * 128;
        const uint32_t tO = tmem + lane_off + 256 + t * 128;
        const bool active = t == 0 || two;
        float m_run = -INFINITY, l = 0.f;
        bool ok = active;
        // grouped items: this row's leaf inside the group and its mask words
        const uint4 *gm = GROUPED ? reinterpret_cast<const uint4 *>(a.gmask) + mslot * a.L +
                                        ((t * BM + row) >> a.leaf_shift)
                                  : nullptr;
        // compensation: this row's leaf among the virtual group's bias rows
        const int leaf_v = GROUPED ? ((t * BM + row) >> a.leaf_shift) : 0;
        for (int j = 0; ok && j < ttot; ++j) {
            const bool virt = COMP && j >= ntiles;
            uint4 mw = make_uint4(~0u, ~0u, ~0u, ~0u);
            if (GROUPED && !virt) mw = __ldg(gm + (int64_t)j * a.L);  // in flight during the wait
            if (!mbar_wait(&bar_s_full[t], j & 1, abort_flag, a.err, 0x30 + t)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t r[BN];
#pragma unroll
            for (int c4 = 0; c4 < BN / 32; ++c4) tmem_ld32(tS + c4 * 32, r + c4 * 32);
            tmem_wait_ld();
            if (virt) {
                // 64 virtual keys: the raw logit plus ln(m) * sqrt(D) (so that
                // the scaled exponent gains log2 m), -inf for m = 0, padding
                // slots and the unused columns 64-127
                const float4 *bq =
                    reinterpret_cast<const float4 *>(a.vbias + ((vt0 + j - ntiles) * a.Lv + leaf_v) * 64);
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const float4 b = __ldg(bq + c4);
                    r[4 * c4 + 0] = __float_as_uint(__uint_as_float(r[4 * c4 + 0]) + b.x);
                    r[4 * c4 + 1] = __float_as_uint(__uint_as_float(r[4 * c4 + 1]) + b.y);
                    r[4 * c4 + 2] = __float_as_uint(__uint_as_float(r[4 * c4 + 2]) + b.z);
                    r[4 * c4 + 3] = __float_as_uint(__uint_as_float(r[4 * c4 + 3]) + b.w);
                }
#pragma unroll
                for (int i = 64; i < BN; ++i) r[i] = __float_as_uint(-INFINITY);
            } else {
                const int valid = min(BN, nk - j * BN);
                if (valid < BN) {
#pragma unroll
                    for (int i = 0; i < BN; ++i)
                        if (i >= valid) r[i] = __float_as_uint(-INFINITY);
                }
            }
            if constexpr (GROUPED) {
                if ((mw.x & mw.y & mw.z & mw.w) != ~0u) {  // warp-uniform: a warp's rows share a leaf
                    const uint32_t m4[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
                    for (int i = 0; i < BN; ++i)
                        if (!((m4[i >> 5] >> (i & 31)) & 1u)) r[i] = __float_as_uint(-INFINITY);
                }
            }
            // row max: three-input max, two new values per instruction, four chains
            float m4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) m4[i] = __uint_as_float(r[i]);
#pragma unroll
            for (int i = 4; i < BN; i += 2)
                m4[(i >> 1) & 3] = fmax3(m4[(i >> 1) & 3], __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
            const float mraw = fmax3(fmax3(m4[0], m4[1], m4[2]), m4[3], m4[3]);
            const float mt = mraw * a.scale_log2;
            // Lazy rescale: move the reference max only when it grew by > 8
            // (log2 units); O and l are scaled after P is written, so the S
            // row and the O chunk never need registers at the same time.
            bool rescale = false;
            float alpha = 1.f;
            if (j == 0) {
                m_run = mt;
            } else if (__any_sync(0xffffffffu, mt > m_run + 8.f)) {
                const float mn = fmaxf(m_run, mt);
                // grouped: a row with no key yet (m = -inf: every key so far
                // masked) has l = 0 and O = 0, and takes alpha = 0
                alpha = (GROUPED && m_run == -INFINITY) ? 0.f : ex2(m_run - mn);
                m_run = mn;
                l *= alpha;
                rescale = true;
            }
            // p = 2^(s*scale - m) on pairs straight from the loaded row; row sum
            // in four partial lanes; bf16 pairs written over S.  (Grouped: while
            // m is still -inf every p is 0; a finite reference keeps it so.)
            const float m_ref = (GROUPED && m_run == -INFINITY) ? 0.f : m_run;
            const uint64_t scp = f2pack(a.scale_log2, a.scale_log2), nmp = f2pack(-m_ref, -m_ref);
            uint64_t sA = 0ull, sB = 0ull;  // (0.f, 0.f)
#pragma unroll
            for (int c4 = 0; c4 < BN / 32; ++c4) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint64_t x2 = ffma2(
                        f2pack(__uint_as_float(r[c4 * 32 + 2 * i]), __uint_as_float(r[c4 * 32 + 2 * i + 1])), scp, nmp);
                    float x0, x1;
                    f2unpack(x2, x0, x1);
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    if (i & 1) sB = fadd2(sB, f2pack(p0, p1));
                    else sA = fadd2(sA, f2pack(p0, p1));
                    pk[i] = pack_bf16(p0, p1);
                }
                tmem_st16(tS + c4 * 16, pk);
            }
            float la, lb, lc, ld;
            f2unpack(sA, la, lb);
            f2unpack(sB, lc, ld);
            la += lc;
            lb += ld;
            l += la + lb;
            if (rescale) {
#pragma unroll
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(tO + c4 * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tO + c4 * 32, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_p_full[t]);
        }
        if (ok && mbar_wait(&bar_o_final[t], 0, abort_flag, a.err, 0x38 + t)) {
            tc_fence_after();
            const int qi = t * BM + row;
            const bool store = qi < nq;
            const int tok = store ? (a.perm ? a.perm[base + cstart + q0 + qi] : q0 + qi) : 0;
            const float inv = 1.f / l;
            __nv_bfloat16 *dst = a.o + a.os.row(bh, tok);
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t o[32];
                tmem_ld32(tO + ch * 32, o);
                tmem_wait_ld();
                if (store) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 u;
                        u.x = pack_bf16(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
                        u.y = pack_bf16(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                        u.z = pack_bf16(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
                        u.w = pack_bf16(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
                        *reinterpret_cast<uint4 *>(dst + ch * 32 + i) = u;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

// Work items: per (bh, cluster) ceil(|c| / 256) items of up to 256 queries
// (dense: per bh, ceil(N / 256) contiguous items).
__global__ void __launch_bounds__(1024) tc_items_kernel(const int32_t *sizes, int4 *items, int32_t *n_items, int BH,
                                                        int Cq, int N)
{
    __shared__ int tmp[33];
    int carry = 0;
    for (int bh = 0; bh < BH; ++bh) {
        for (int b0 = 0; b0 < Cq; b0 += blockDim.x) {
            const int c = b0 + threadIdx.x;
            const int sz = c < Cq ? (sizes ? sizes[(int64_t)bh * Cq + c] : N) : 0;
            const int nt = (sz + 2 * BM - 1) / (2 * BM);
            int tot;
            const int ex = block_excl_scan(nt, tmp, tot);
            for (int t = 0; t < nt; ++t) {
                const int q0 = t * 2 * BM;
                items[carry + ex + t] = make_int4(bh, c, q0, min(2 * BM, sz - q0));
            }
            carry += tot;
        }
    }
    if (threadIdx.x == 0) *n_items = carry;
}

}  // namespace tc

// Dynamic shared memory per CTA.  Every CTA allocates all 512 TMEM columns,
// so a second CTA on the same SM would only wait inside tcgen05.alloc: the
// D = 64 tiles (97 KB) are padded past half of the SM's 228 KB so that the
// scheduler places one CTA per SM, as for D = 128.
constexpr size_t tc_smem_bytes(int D)
{
    const size_t need = (size_t)(2 * tc::BM * D * 2 + 4 * tc::BN * D * 2) + 1024;
    return need > 120 * 1024 ? need : 120 * 1024;
}

template <int D, bool G, bool C>
static cudaError_t attn_attr()
{
    return cudaFuncSetAttribute(tc::attn_tc_kernel<D, G, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)tc_smem_bytes(D));
}

cudaError_t attn_tc_configure()
{
    const cudaError_t e[8] = {attn_attr<128, false, false>(), attn_attr<64, false, false>(),
                              attn_attr<128, true, false>(),  attn_attr<64, true, false>(),
                              attn_attr<128, false, true>(),  attn_attr<64, false, true>(),
                              attn_attr<128, true, true>(),   attn_attr<64, true, true>()};
    for (cudaError_t x : e)
        if (x != cudaSuccess) return x;
    return cudaSuccess;
}

template <int D>
static void attn_launch(const tc::Args &a, bool grouped, bool comp, int grid, cudaStream_t st)
{
    const size_t sm = tc_smem_bytes(D);
    if (grouped && comp) tc::attn_tc_kernel<D, true, true><<<grid, tc::kThreads, sm, st>>>(a);
    else if (grouped) tc::attn_tc_kernel<D, true, false><<<grid, tc::kThreads, sm, st>>>(a);
    else if (comp) tc::attn_tc_kernel<D, false, true><<<grid, tc::kThreads, sm, st>>>(a);
    else tc::attn_tc_kernel<D, false, false><<<grid, tc::kThreads, sm, st>>>(a);
}

int attn_tc_max_items(int BH, int N, int Cq) { return BH * ((N + 2 * tc::BM - 1) / (2 * tc::BM) + Cq); }

bool rows_tensor_map(CUtensorMap *m, const void *base, uint64_t rows, int D, int box_rows)
{
    using Encode = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static Encode encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return false;
        encode = (Encode)fn;
    }
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool launch_attn_tc(const __nv_bfloat16 *qr, const __nv_bfloat16 *kr, const __nv_bfloat16 *v, const RowStrides &vs,
                    __nv_bfloat16 *o, const RowStrides &os, int4 *items, int32_t *n_items, int max_items, const int32_t *sizes, const int32_t *perm,
                    const int32_t *start, const long long *offsets, const int32_t *indices, const int32_t *n_c,
                    int32_t *err, int BH, int N, int D, int Cq, cudaStream_t st,
                    const GroupedLists *grouped, const CompLists *comp)
{
    if (grouped) {
        max_items = BH * (Cq / grouped->L);
    } else {
        tc::tc_items_kernel<<<1, 1024, 0, st>>>(sizes, items, n_items, BH, sizes ? Cq : 1, N);
        count_launches(1);
    }
    tc::Args a{};
    a.qr = qr;
    a.kr = kr;
    a.v = v;
    a.o = o;
    a.vs = vs;
    a.os = os;
    a.items = items;
    a.n_items = n_items;
    a.perm = perm;
    a.start = start;
    a.offsets = offsets;
    a.indices = indices;
    a.n_c = n_c;
    a.err = err;
    a.gmask = grouped ? grouped->masks : nullptr;
    a.u_n = grouped ? grouped->u_n : nullptr;
    a.L = grouped ? grouped->L : 0;
    a.leaf_shift = grouped ? grouped->leaf_shift : 0;
    a.G = grouped ? Cq / grouped->L : 0;
    if (grouped) a.indices = grouped->u_idx;
    if (comp) {
        a.vk_hi = comp->vk_hi;
        a.vk_lo = comp->vk_lo;
        a.vv_hi = comp->vv_hi;
        a.vv_lo = comp->vv_lo;
        a.vlist = comp->vlist;
        a.vn = comp->vn;
        a.vbias = comp->vbias;
        a.Ck = comp->Ck;
        a.Lv = comp->Lv;
        a.vtiles = comp->vtiles;
    }
    a.N = N;
    a.Cq = Cq;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    if (D == 128) attn_launch<128>(a, grouped != nullptr, comp != nullptr, max_items, st);
    else attn_launch<64>(a, grouped != nullptr, comp != nullptr, max_items, st);
    count_launches(1);
    return true;
}

}  // namespace scope
