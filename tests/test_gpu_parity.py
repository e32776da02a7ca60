"""CUDA path vs the fp64 oracle, stage by stage, through the C ABI.

Small workloads are checked in full; the Wan-480p and HunyuanVideo-720p sized
workloads at their full sizes on sampled heads, rows, clusters and queries.
Tolerances and the near-tie rule are in parity.py.
"""
import numpy as np
import pytest
import torch

import cluster_guided_sparse_b200 as scope
import oracle
import parity as P
from cluster_guided_sparse_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def to_dev(*ts):
    return [t.to(DEV).contiguous() for t in ts]


def plan_of(w, q, k, **kw):
    params, grid = scope.make_params(w, **kw)
    return scope.plan(q, k, params, grid)


def pull(pl, w, heads):
    """Host copies of one plan's per-head results."""
    out = {}
    B = 0
    lab = pl.view("q_labels")
    cent = pl.view("q_centroids")
    codes = pl.view("k_codes")
    kc = [pl.view("k_cent_t"), pl.view("k_cent_h"), pl.view("k_cent_w")]
    for h in heads:
        out[h] = dict(
            q_labels=lab[B, h].cpu().numpy(),
            q_cent=P.np64(cent[B, h]),
            codes=[codes[s, B, h].cpu().numpy() for s in range(3)],
            k_cent=[P.np64(kc[s][B, h]) for s in range(3)],
        )
    return out


def lists_fn(pl, w, h, B=0):
    off = pl.view("offsets").cpu().numpy()
    n = pl.view("n").cpu().numpy()
    idx = pl.view("indices")

    def get(c):
        i = (B * w.H + h) * w.c_q + c if w.fixed_cluster_size == 0 else (B * w.H + h) * (w.N // w.fixed_cluster_size) + c
        return idx[int(off[i]):int(off[i]) + int(n[B, h, c])].cpu().numpy()
    return get


def stagefed(w, heads, iters_list, row_sample=None, cl_sample=None, q_sample=None, seed=0):
    rng = np.random.default_rng(seed)
    q, k, v = synth.make_inputs(w)
    qd, kd, vd = to_dev(q, k, v)
    N, D = w.N, w.D
    rows = np.sort(rng.choice(N, row_sample, replace=False)) if row_sample else np.arange(N)
    states = {}
    for it in iters_list:
        pl = plan_of(w, qd, kd, iters=it)
        states[it] = pull(pl, w, heads)
        if it == iters_list[-1]:
            final = pl
        else:
            del pl
    torch.cuda.synchronize()
    final.sync_status()
    qr_all, kr_all = final.view("qr"), final.view("kr")
    o = scope.attn(qd, kd, vd, final)
    torch.cuda.synchronize()
    tc_q, tc_k, tc_sel = P.TieCounter(), P.TieCounter(), P.TieCounter()
    offs = np.cumsum((0,) + tuple(w.d_split))
    report = {}
    for h in heads:
        qr, kr = P.np64(qr_all[0, h]), P.np64(kr_all[0, h])
        P.check_rope(qr[rows], q[0, h].double().numpy(), w, rows)
        P.check_rope(kr[rows], k[0, h].double().numpy(), w, rows)
        for i, it in enumerate(iters_list):
            st = states[it][h]
            if it == 0:  # strided init: exact rows
                stride = N // w.c_q
                np.testing.assert_array_equal(st["q_cent"], qr[np.arange(w.c_q) * stride])
            P.check_assign(qr[rows], st["q_cent"], st["q_labels"][rows], tc_q, f"h{h} it{it} queries")
            for s in range(3):
                a, b = int(offs[s]), int(offs[s + 1])
                P.check_assign(kr[rows, a:b], st["k_cent"][s], st["codes"][s][rows], tc_k, f"h{h} it{it} keys s{s}")
            if i > 0 and iters_list[i - 1] == it - 1:
                prev = states[it - 1][h]
                P.check_update(qr, prev["q_labels"], prev["q_cent"], st["q_cent"], f"h{h} it{it} query update")
                for s in range(3):
                    a, b = int(offs[s]), int(offs[s + 1])
                    P.check_update(kr[:, a:b], prev["codes"][s], prev["k_cent"][s], st["k_cent"][s],
                                   f"h{h} it{it} key update s{s}")
        st = states[iters_list[-1]][h]
        lut = final.view("lut")[0, h].cpu().numpy()
        P.check_lut(st["q_cent"], st["k_cent"], w.d_split, lut.astype(np.float64))
        sizes = final.view("q_sizes")[0, h].cpu().numpy()
        assert (sizes == np.bincount(st["q_labels"], minlength=w.c_q)).all()
        perm = final.view("q_perm")[0, h].cpu().numpy()
        qstart = final.view("q_start")[0, h].cpu().numpy()
        assert (perm == np.argsort(st["q_labels"], kind="stable")).all()
        assert (np.diff(qstart) == sizes).all()
        clusters = np.arange(w.c_q) if cl_sample is None else rng.choice(w.c_q, cl_sample, replace=False)
        get = lists_fn(final, w, h)
        P.check_selection(lut, st["codes"], sizes, final.view("r")[0, h].cpu().numpy(),
                          final.view("kh")[0, h].item(), final.view("n")[0, h].cpu().numpy(), get, w, N, D,
                          clusters, tc_sel)
        qrows = np.arange(N) if q_sample is None else np.sort(rng.choice(N, q_sample, replace=False))
        report[h] = P.check_attention(qr, kr, v[0, h].double().numpy(), st["q_labels"], get,
                                      P.np64(o[0, h]), qrows)
    tc_q.assert_ok("query assign")
    tc_k.assert_ok("key assign")
    tc_sel.assert_ok("Top-p counts")
    return report


def test_tiny_config_full_parity():
    w = synth.WORKLOADS["tiny"]
    stagefed(w, range(w.H), list(range(w.iters + 1)))


def test_small_config_full_parity():
    w = synth.WORKLOADS["small"]
    stagefed(w, range(w.H), list(range(w.iters + 1)))


@pytest.mark.parametrize("top_p", [0.8, 0.9, 0.95])
def test_wan480p_sampled_parity(top_p):
    w = synth.WORKLOADS["wan480p"].with_(top_p=top_p)
    iters = [0, 1, 2, 9, 10] if top_p == 0.9 else [10]
    stagefed(w, [0, w.H // 2, w.H - 1], iters, row_sample=3000, cl_sample=6, q_sample=48)


def test_hunyuan720p_sampled_parity():
    w = synth.WORKLOADS["hunyuan720p"]
    stagefed(w, [0, w.H - 1], [0, 1, 9, 10], row_sample=2000, cl_sample=4, q_sample=32)


def test_plan_is_deterministic():
    w = synth.WORKLOADS["small"]
    qd, kd, _ = to_dev(*synth.make_inputs(w))
    a, b = plan_of(w, qd, kd), plan_of(w, qd, kd)
    torch.cuda.synchronize()
    for name in ("q_labels", "k_codes", "q_centroids", "r", "kh", "n", "offsets"):
        assert torch.equal(a.view(name), b.view(name)), name
    tot = int(a.view("offsets")[-1])
    assert torch.equal(a.view("indices")[:tot], b.view("indices")[:tot])


@pytest.mark.parametrize("name", ["tiny", "small", "wan480p"])
def test_dense_attention_parity(name):
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_inputs(w, heads=[0, 1]) if w.H > 2 else synth.make_inputs(w)
    qd, kd, vd = to_dev(q, k, v)
    params, grid = scope.make_params(w)
    o = scope.dense_attn(qd, kd, vd, params, grid)
    torch.cuda.synchronize()
    rows = np.arange(w.N) if w.N <= 2048 else np.sort(np.random.default_rng(1).choice(w.N, 64, replace=False))
    for h in range(q.shape[1]):
        qr = oracle.rope3d(q[0, h].double().numpy(), w.grid, w.d_split, w.theta)
        kr = oracle.rope3d(k[0, h].double().numpy(), w.grid, w.d_split, w.theta)
        qr, kr = oracle._round_bf16(qr), oracle._round_bf16(kr)
        ref = oracle.attention_rows(qr[rows], kr, v[0, h].double().numpy(), np.arange(w.N, dtype=np.int32),
                                    1.0 / np.sqrt(w.D))
        max_abs, rel = P.attn_error(P.np64(o[0, h])[rows], ref)
        assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, (max_abs, rel)


def test_top_p_one_equals_dense():
    w = synth.WORKLOADS["small"].with_(top_p=1.0)
    qd, kd, vd = to_dev(*synth.make_inputs(w))
    pl = plan_of(w, qd, kd)
    o = scope.attn(qd, kd, vd, pl)
    params, grid = scope.make_params(w)
    od = scope.dense_attn(qd, kd, vd, params, grid)
    torch.cuda.synchronize()
    assert (pl.view("n") == w.N).all()
    max_abs, rel = P.attn_error(P.np64(o), P.np64(od))
    assert max_abs <= 1e-2 and rel <= 2e-3, (max_abs, rel)


@pytest.mark.parametrize("case", [
    dict(N=105, D=64, grid=(3, 5, 7), d_split=(16, 24, 24), c_q=5, c_sub=(3, 4, 5)),   # ragged everything
    dict(N=64, D=64, grid=(1, 8, 8), d_split=(0, 32, 32), c_q=1, c_sub=(1, 8, 8)),     # one cluster, empty t block
    dict(N=300, D=128, grid=(3, 10, 10), d_split=(16, 56, 56), c_q=7, c_sub=(4, 4, 4), top_p=1.0),
    dict(N=200, D=64, grid=(2, 10, 10), d_split=(16, 24, 24), c_q=6, c_sub=(2, 2, 2), k_min=500),
    dict(N=200, D=64, grid=(2, 10, 10), d_split=(16, 24, 24), c_q=6, c_sub=(3, 3, 3), online_topk=0, iters=0),
    dict(N=256, D=64, grid=(0, 0, 0), d_split=(16, 24, 24), c_q=8, c_sub=(4, 4, 4), top_p=0.5),  # no grid
    dict(N=512, D=128, grid=(2, 16, 16), d_split=(16, 56, 56), c_q=16, c_sub=(8, 8, 8), H=3, B=2),
])
def test_edge_cases(case):
    case = dict(case)
    B = case.pop("B", 1)
    w, (q, k, v) = synth.tiny_case(**case)
    if B > 1:
        w = w.with_(B=B)
        q, k, v = synth.make_inputs(w)
    qd, kd, vd = to_dev(q, k, v)
    pl = plan_of(w, qd, kd)
    o = scope.attn(qd, kd, vd, pl)
    torch.cuda.synchronize()
    pl.sync_status()
    N, D = w.N, w.D
    tc = P.TieCounter()
    for b in range(w.B):
        for h in range(w.H):
            qr, kr = P.np64(pl.view("qr")[b, h]), P.np64(pl.view("kr")[b, h])
            if w.grid[0]:
                P.check_rope(qr, q[b, h].double().numpy(), w)
            lab = pl.view("q_labels")[b, h].cpu().numpy()
            cent = P.np64(pl.view("q_centroids")[b, h])
            P.check_assign(qr, cent, lab, tc)
            codes = [pl.view("k_codes")[s, b, h].cpu().numpy() for s in range(3)]
            lut = pl.view("lut")[b, h].cpu().numpy()
            sizes = pl.view("q_sizes")[b, h].cpu().numpy()
            get = lists_fn(pl, w, h, B=b)
            P.check_selection(lut, codes, sizes, pl.view("r")[b, h].cpu().numpy(), pl.view("kh")[b, h].item(),
                              pl.view("n")[b, h].cpu().numpy(), get, w, N, D, range(w.c_q), tc)
            P.check_attention(qr, kr, v[b, h].double().numpy(), lab, get, P.np64(o[b, h]), np.arange(N))
    tc.assert_ok("edge")


def test_degenerate_identical_tokens_leave_clusters_empty():
    w, _ = synth.tiny_case(N=128, D=64, grid=(2, 8, 8), d_split=(16, 24, 24), c_q=4, c_sub=(2, 2, 2))
    q = torch.ones((1, 1, 128, 64))
    k = torch.ones((1, 1, 128, 64))
    v = torch.randn((1, 1, 128, 64), generator=torch.Generator().manual_seed(0))
    w = w.with_(grid=(0, 0, 0))
    qd, kd, vd = to_dev(q, k, v)
    pl = plan_of(w, qd, kd)
    o = scope.attn(qd, kd, vd, pl)
    torch.cuda.synchronize()
    sizes = pl.view("q_sizes")[0, 0].cpu().numpy()
    assert sizes.tolist() == [128, 0, 0, 0]  # all equal -> lowest index wins, others stay empty
    n = pl.view("n")[0, 0].cpu().numpy()
    assert n[1:].tolist() == [0, 0, 0]
    # equal logits: attention is the mean of V over the selected keys
    get = lists_fn(pl, w, 0)
    sel = get(0)
    np.testing.assert_allclose(P.np64(o[0, 0]), np.broadcast_to(v[0, 0].double().numpy()[sel].mean(0), (128, 64)),
                               atol=2e-2)


def check_groups(pl, w, h, get, groups=None):
    """Grouped attention lists (leaves of 32 or 64 queries): every group's
    union is the ascending union of its leaves' lists, stored at its first
    leaf's offset, and its tile masks mark exactly each leaf's own keys."""
    leaf, C = w.fixed_cluster_size, w.N // w.fixed_cluster_size
    Lg = 256 // leaf if leaf in (32, 64) else 0
    if not Lg or C % Lg:
        with pytest.raises(scope.ScopeError):
            pl.view("group_n")
        return 0
    G = C // Lg
    off = pl.view("offsets").cpu().numpy()
    gidx = pl.view("group_indices")
    gn = pl.view("group_n")[0, h].cpu().numpy()
    gm = pl.view("group_masks")
    for g in (range(G) if groups is None else groups):
        lists = [get(c) for c in range(g * Lg, (g + 1) * Lg)]
        u = np.unique(np.concatenate(lists))
        start = int(off[h * C + g * Lg])
        assert int(gn[g]) == len(u), (h, g)
        assert (gidx[start:start + len(u)].cpu().numpy() == u).all(), (h, g)
        T = (len(u) + 127) // 128
        slot = start // 128 + h * G + g
        words = gm[slot * Lg * 4:(slot + T) * Lg * 4].cpu().numpy().view(np.uint32).reshape(T, Lg, 4)
        for li, lst in enumerate(lists):
            bits = np.zeros(T * 128, dtype=np.uint8)
            bits[:len(u)] = np.isin(u, lst)
            want = np.packbits(bits.reshape(T * 4, 32), axis=1, bitorder="little").view("<u4").reshape(T, 4)
            assert (words[:, li, :] == want).all(), (h, g, li)
    return G


def bisect_parity(w, heads, cl_sample=None, q_sample=None, seed=0, tie_groups=0):
    rng = np.random.default_rng(seed)
    q, k, v = synth.make_inputs(w)
    if tie_groups:
        # 90% of the rows become copies of `tie_groups` rows, so the median
        # cuts fall among equal deltas (member-order tie rule)
        idx = torch.from_numpy(np.nonzero(rng.random(w.N) < 0.9)[0])
        src = torch.from_numpy(rng.integers(0, w.N, tie_groups))[idx % tie_groups]
        for t in (q, k):
            t[:, :, idx] = t[:, :, src]
    qd, kd, vd = to_dev(q, k, v)
    pl = plan_of(w, qd, kd)
    o = scope.attn(qd, kd, vd, pl)
    torch.cuda.synchronize()
    pl.sync_status()
    N, D, leaf = w.N, w.D, w.fixed_cluster_size
    C = N // leaf
    wq = w.with_(c_q=C, c_sub=(C, 1, 1))
    tc = P.TieCounter()
    for h in heads:
        qr, kr = P.np64(pl.view("qr")[0, h]), P.np64(pl.view("kr")[0, h])
        np.testing.assert_array_equal(qr, q[0, h].double().numpy())  # no grid: identity
        np.testing.assert_array_equal(kr, k[0, h].double().numpy())
        qlab = pl.view("q_labels")[0, h].cpu().numpy()
        codes = [pl.view("k_codes")[s, 0, h].cpu().numpy() for s in range(3)]
        qcent, kcent = P.np64(pl.view("q_centroids")[0, h]), P.np64(pl.view("k_cent_t")[0, h])
        for X, lab_gpu, cent_gpu in ((qr, qlab, qcent), (kr, codes[0], kcent)):
            lab, cent, perm = oracle.bisect(X, leaf, w.iters)
            assert (lab == lab_gpu).all(), f"bisection labels differ on {(lab != lab_gpu).sum()} rows"
            np.testing.assert_allclose(cent_gpu, cent, rtol=0, atol=1e-6 * max(1.0, np.abs(cent).max()))
        assert (codes[1] == 0).all() and (codes[2] == 0).all()
        sizes = pl.view("q_sizes")[0, h].cpu().numpy()
        assert (sizes == leaf).all()
        assert (pl.view("q_perm")[0, h].cpu().numpy() == np.argsort(qlab, kind="stable")).all()
        lut = pl.view("lut")[0, h].cpu().numpy()
        P.check_lut(qcent, [kcent, np.zeros((1, 0)), np.zeros((1, 0))], (D, 0, 0), lut.astype(np.float64))
        clusters = np.arange(C) if cl_sample is None else rng.choice(C, cl_sample, replace=False)
        get = lists_fn(pl, w, h)
        P.check_selection(lut, codes, sizes, pl.view("r")[0, h].cpu().numpy(), pl.view("kh")[0, h].item(),
                          pl.view("n")[0, h].cpu().numpy(), get, wq, N, D, clusters, tc)
        rows = np.arange(N) if q_sample is None else np.sort(rng.choice(N, q_sample, replace=False))
        P.check_attention(qr, kr, v[0, h].double().numpy(), qlab, get, P.np64(o[0, h]), rows)
        ng = C // (256 // leaf) if leaf in (32, 64) and C % (256 // leaf) == 0 else 0
        check_groups(pl, w, h, get, None if cl_sample is None or ng == 0 else rng.choice(ng, 16, replace=False))
    tc.assert_ok("bisection Top-p counts")


def test_unstructured_bisection_parity():
    w = synth.WORKLOADS["unstructured"]
    bisect_parity(w, [0, w.H - 1], cl_sample=8, q_sample=48)


@pytest.mark.parametrize("N,D,H,leaf", [(128, 64, 1, 64), (512, 128, 2, 64), (4096, 64, 1, 64), (2048, 128, 2, 32),
                                         (1024, 64, 1, 128)])
def test_bisection_small_shapes(N, D, H, leaf):
    w = synth.WORKLOADS["unstructured"].with_(N=N, D=D, H=H, d_split=(D, 0, 0), components=16, k_min=32,
                                               config_id=150 + N, c_q=N // leaf, c_sub=(N // leaf, 1, 1),
                                               fixed_cluster_size=leaf)
    bisect_parity(w, range(H))


@pytest.mark.parametrize("groups", [1, 3, 24])
def test_bisection_tied_rows(groups):
    w = synth.WORKLOADS["unstructured"].with_(N=4096, D=64, H=1, d_split=(64, 0, 0), components=16, k_min=32,
                                               config_id=170 + groups, c_q=64, c_sub=(64, 1, 1))
    bisect_parity(w, [0], tie_groups=groups)


# ClusterAttention compensation: every excluded key enters through its key
# cluster's mean key and value (the oracle's attention_rows_comp, reading R16),
# fed the device's own rotated rows, key-cluster labels and lists.
@pytest.mark.parametrize("N,D,H,p,leaf", [(4096, 64, 2, 0.9, 64), (4096, 64, 1, 0.5, 64), (512, 128, 1, 0.9, 64),
                                          (65536, 64, 1, 0.9, 64),  # the benchmarked shape: 1024 key leaves
                                          (2048, 128, 1, 0.7, 32),  # eight leaves per work item
                                          (4096, 64, 1, 0.7, 128),  # one leaf per work item (ungrouped)
                                          (8192, 64, 1, 0.7, 512)])  # two work items per leaf
def test_compensation_parity(N, D, H, p, leaf):
    w = synth.WORKLOADS["unstructured"].with_(N=N, D=D, H=H, d_split=(D, 0, 0), components=16, k_min=32,
                                               config_id=170 + N + D, c_q=N // leaf, c_sub=(N // leaf, 1, 1),
                                               top_p=p, compensate=1, fixed_cluster_size=leaf)
    q, k, v = synth.make_inputs(w)
    qd, kd, vd = to_dev(q, k, v)
    pl = plan_of(w, qd, kd)
    o = scope.attn(qd, kd, vd, pl)
    pl_plain = plan_of(w.with_(compensate=0), qd, kd)
    o_plain = scope.attn(qd, kd, vd, pl_plain)
    torch.cuda.synchronize()
    pl.sync_status()
    rng = np.random.default_rng(5)
    for h in range(H):
        qr, kr = P.np64(pl.view("qr")[0, h]), P.np64(pl.view("kr")[0, h])
        vv = v[0, h].double().numpy()
        qlab = pl.view("q_labels")[0, h].cpu().numpy()
        klab = pl.view("k_codes")[0, 0, h].cpu().numpy()
        get = lists_fn(pl, w, h)
        rows = np.sort(rng.choice(N, 96, replace=False))
        ref = np.stack([oracle.attention_rows_comp(qr[n:n + 1], kr, vv, get(qlab[n]), klab, 1.0 / np.sqrt(D))[0]
                        for n in rows])
        max_abs, rel = P.attn_error(P.np64(o[0, h])[rows], ref)
        assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, f"compensated: max-abs {max_abs:.3g}, rel {rel:.3g}"
        # rows whose cluster kept every key are untouched by the compensation
        full = [n for n in rows if len(get(qlab[n])) == N]
        if full:
            np.testing.assert_array_equal(o[0, h, full].cpu().numpy(), o_plain[0, h, full].cpu().numpy())


# B > 1: (batch, head) pairs run through the same kernels; batch 1's selection
# and attention are checked against the oracle on the device's own stage inputs.
def test_second_batch_entry_stage_fed():
    w = synth.WORKLOADS["small"].with_(B=2, config_id=190)
    q, k, v = synth.make_inputs(w)
    qd, kd, vd = to_dev(q, k, v)
    pl = plan_of(w, qd, kd)
    o = scope.attn(qd, kd, vd, pl)
    torch.cuda.synchronize()
    pl.sync_status()
    b, N, D = 1, w.N, w.D
    tc = P.TieCounter()
    for h in (0, w.H - 1):
        qr, kr = P.np64(pl.view("qr")[b, h]), P.np64(pl.view("kr")[b, h])
        qlab = pl.view("q_labels")[b, h].cpu().numpy()
        codes = [pl.view("k_codes")[s, b, h].cpu().numpy() for s in range(3)]
        kc = [P.np64(pl.view(n)[b, h]) for n in ("k_cent_t", "k_cent_h", "k_cent_w")]
        lut = pl.view("lut")[b, h].cpu().numpy()
        P.check_lut(P.np64(pl.view("q_centroids")[b, h]), kc, w.d_split, lut.astype(np.float64))
        get = lists_fn(pl, w, h, B=b)
        P.check_selection(lut, codes, pl.view("q_sizes")[b, h].cpu().numpy(), pl.view("r")[b, h].cpu().numpy(),
                          pl.view("kh")[b, h].item(), pl.view("n")[b, h].cpu().numpy(), get, w, N, D,
                          np.arange(w.c_q), tc)
        P.check_attention(qr, kr, v[b, h].double().numpy(), qlab, get, P.np64(o[b, h]), np.arange(0, N, 7))
    tc.assert_ok("batch 1 Top-p counts")


# B > 1 through the ClusterAttention path: the bisection's 2*B*H row sets,
# the grouped work items (unions and masks per (batch, head)) and the
# compensation's virtual lists, checked on batch entry 1 against the oracle.
def test_second_batch_entry_cluster_attention_compensated():
    N, D, H, leaf = 4096, 64, 2, 64
    w = synth.WORKLOADS["unstructured"].with_(B=2, N=N, D=D, H=H, d_split=(D, 0, 0), components=16, k_min=32,
                                               config_id=195, c_q=N // leaf, c_sub=(N // leaf, 1, 1), top_p=0.8,
                                               compensate=1, fixed_cluster_size=leaf)
    q, k, v = synth.make_inputs(w)
    qd, kd, vd = to_dev(q, k, v)
    pl = plan_of(w, qd, kd)
    o = scope.attn(qd, kd, vd, pl)
    torch.cuda.synchronize()
    pl.sync_status()
    b, C = 1, N // leaf
    rng = np.random.default_rng(11)
    for h in range(H):
        qr, kr = P.np64(pl.view("qr")[b, h]), P.np64(pl.view("kr")[b, h])
        qlab = pl.view("q_labels")[b, h].cpu().numpy()
        klab = pl.view("k_codes")[0, b, h].cpu().numpy()
        for X, lab_gpu in ((qr, qlab), (kr, klab)):
            lab, _, _ = oracle.bisect(X, leaf, w.iters)
            assert (lab == lab_gpu).all(), f"bisection labels differ on {(lab != lab_gpu).sum()} rows"
        get = lists_fn(pl, w, h, B=b)
        # the grouped lists of flat head (b, h)
        off = pl.view("offsets").cpu().numpy()
        gn = pl.view("group_n")[b, h].cpu().numpy()
        gidx = pl.view("group_indices")
        bh, Lg = b * H + h, 256 // leaf
        for g in range(C // Lg):
            u = np.unique(np.concatenate([get(c) for c in range(g * Lg, (g + 1) * Lg)]))
            start = int(off[bh * C + g * Lg])
            assert int(gn[g]) == len(u) and (gidx[start:start + len(u)].cpu().numpy() == u).all(), (h, g)
        rows = np.sort(rng.choice(N, 64, replace=False))
        ref = np.stack([oracle.attention_rows_comp(qr[n:n + 1], kr, v[b, h].double().numpy(), get(qlab[n]), klab,
                                                   1.0 / np.sqrt(D))[0] for n in rows])
        max_abs, rel = P.attn_error(P.np64(o[b, h])[rows], ref)
        assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, f"compensated: max-abs {max_abs:.3g}, rel {rel:.3g}"
