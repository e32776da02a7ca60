"""Pins of the fp64 oracle against what the pages and mathematics fix.

No page prints a worked value, so each step is pinned by closed forms,
invariants, special cases that reduce to a textbook routine, and brute force on
tiny inputs -- chosen so that a dropped term, a wrong sign or index or a
transposed operand in the oracle fails at least one of them.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle
from cluster_guided_sparse_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- RoPE
def test_rope_hand_examples():
    g = _gold("rope_pairs.json")
    T, Hh, W = g["grid"]
    N, D = T * Hh * W, sum(g["d_split"])
    for case in g["cases"]:
        x = np.zeros((N, D))
        x[case["token"]] = case["x"]
        y = oracle.rope3d(x, g["grid"], g["d_split"], g["theta"])
        np.testing.assert_allclose(y[case["token"]], case["expect"], rtol=0, atol=1e-15, err_msg=case["note"])


def test_rope_norm_and_identity_at_origin():
    rng = np.random.default_rng(1)
    grid, ds = (3, 4, 5), (8, 12, 12)
    x = rng.standard_normal((60, 32))
    y = oracle.rope3d(x, grid, ds, 10000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_array_equal(y[0], x[0])
    # per-pair norms are kept too (each pair is a plane rotation)
    np.testing.assert_allclose(np.hypot(y[:, 0::2], y[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]), rtol=1e-12)


def test_rope_relative_position_invariance():
    """<R_{m+s} q, R_{n+s} k> = <R_m q, R_n k> for any per-axis shift s."""
    rng = np.random.default_rng(2)
    grid, ds = (6, 7, 9), (8, 12, 12)
    T, Hh, W = grid
    D = sum(ds)
    q, k = rng.standard_normal(D), rng.standard_normal(D)

    def tok(t, y, x):
        return (t * Hh + y) * W + x

    for (m, n, s) in [((0, 1, 2), (3, 4, 5), (1, 2, 3)), ((2, 0, 8), (0, 6, 0), (3, 0, 0)),
                      ((1, 1, 1), (1, 1, 1), (4, 5, 7))]:
        X = np.zeros((T * Hh * W, D))
        a, b = tok(*m), tok(*n)
        a2 = tok(*(mi + si for mi, si in zip(m, s)))
        b2 = tok(*(ni + si for ni, si in zip(n, s)))
        X[a], X[a2] = q, q
        Y = oracle.rope3d(X, grid, ds, 10000.0)
        Xk = np.zeros_like(X)
        Xk[b], Xk[b2] = k, k
        Yk = oracle.rope3d(Xk, grid, ds, 10000.0)
        assert abs(Y[a] @ Yk[b] - Y[a2] @ Yk[b2]) < 1e-12 * (np.linalg.norm(q) * np.linalg.norm(k))


def test_rope_no_grid_is_identity():
    x = np.random.default_rng(3).standard_normal((16, 8))
    np.testing.assert_array_equal(oracle.rope3d(x, (0, 0, 0), (8, 0, 0), 10000.0), x)


# ----------------------------------------------------------------------------- k-means
def test_kmeans_brute_force_assign_and_ties():
    rng = np.random.default_rng(4)
    x = rng.integers(-3, 4, size=(200, 3)).astype(float)
    c = rng.integers(-3, 4, size=(7, 3)).astype(float)
    lab = oracle.kmeans_assign(x, c)
    for n in range(x.shape[0]):
        d = [sum((x[n, t] - c[j, t]) ** 2 for t in range(3)) for j in range(7)]
        best = min(d)
        assert lab[n] == d.index(best)  # first (lowest) index among the minima
    # an equidistant point goes to the lower index
    assert oracle.kmeans_assign(np.array([[0.0, 0.0]]), np.array([[1.0, 0.0], [-1.0, 0.0]]))[0] == 0
    assert oracle.kmeans_assign(np.array([[0.0, 0.0]]), np.array([[5.0, 0.0], [0.0, 1.0], [1.0, 0.0]]))[0] == 1


def test_kmeans_objective_never_increases():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((500, 6)) + rng.integers(0, 4, size=(500, 1)) * 3.0
    C = 9
    cent = x[np.arange(C) * (500 // C)].copy()
    prev = np.inf
    for _ in range(8):
        lab = oracle.kmeans_assign(x, cent)
        J_assign = oracle.kmeans_objective(x, lab, cent)
        assert J_assign <= prev + 1e-9
        cent, _ = oracle.kmeans_update(x, lab, cent)
        J_update = oracle.kmeans_objective(x, lab, cent)
        assert J_update <= J_assign + 1e-9
        prev = J_update


def test_kmeans_separated_blobs_recover_means():
    """Strided init picks one point per blob -> blob means after one update."""
    rng = np.random.default_rng(6)
    C, per, D = 4, 25, 5
    centers = np.eye(C, D) * 100.0
    x = np.concatenate([centers[j] + rng.standard_normal((per, D)) for j in range(C)])
    lab, cent, sizes = oracle.kmeans(x, C, iters=1)
    for j in range(C):
        np.testing.assert_allclose(cent[j], x[j * per:(j + 1) * per].mean(0), rtol=0, atol=1e-12)
        assert (lab[j * per:(j + 1) * per] == j).all()
    assert sizes.tolist() == [per] * C


def test_kmeans_init_offset_and_empty_cluster():
    x = np.array([[0.0], [1.0], [2.0], [3.0], [100.0], [101.0]])
    # strided init with stride 3 and seed 1 -> offset 1: centroids x[1], x[4]
    lab, cent, _ = oracle.kmeans(x, 2, iters=0, seed=1)
    np.testing.assert_array_equal(cent[:, 0], [1.0, 100.0])
    assert lab.tolist() == [0, 0, 0, 0, 1, 1]
    # a centroid far from every point gets no member and keeps its place
    c0 = np.array([[0.0], [1000.0], [101.0]])
    l0 = oracle.kmeans_assign(x, c0)
    c1, sizes = oracle.kmeans_update(x, l0, c0)
    assert sizes[1] == 0 and c1[1, 0] == 1000.0
    np.testing.assert_allclose(c1[:, 0], [1.5, 1000.0, 100.5])


# ----------------------------------------------------------------------------- LUT / proxy
def test_lut_sum_is_product_quantised_dot():
    """s_c(j) = qbar_c . concat(mu_t[a_t(j)], mu_h[a_h(j)], mu_w[a_w(j)])."""
    rng = np.random.default_rng(7)
    ds, Cs, Cq, N = (4, 6, 6), (3, 5, 4), 6, 40
    qc = rng.standard_normal((Cq, sum(ds)))
    offs = np.cumsum((0,) + ds)
    kcs = [rng.standard_normal((Cs[s], ds[s])) for s in range(3)]
    codes = [rng.integers(0, Cs[s], N).astype(np.int32) for s in range(3)]
    luts = [oracle.lut(qc[:, offs[s]:offs[s + 1]], kcs[s]) for s in range(3)]
    for c in range(Cq):
        s = oracle.proxy_scores([L[c] for L in luts], codes)
        full = np.stack([np.concatenate([kcs[t][codes[t][j]] for t in range(3)]) for j in range(N)])
        np.testing.assert_allclose(s, full @ qc[c], rtol=1e-13, atol=1e-13)


def test_each_key_its_own_centroid_gives_exact_per_query_topp():
    """C_q = C_t = C_h = C_w = N: proxy = exact q.k, so selection = exact Top-p per query."""
    w, (q, k, v) = synth.tiny_case(N=32, D=8, grid=(2, 4, 4), d_split=(2, 2, 4), c_q=32, c_sub=(32, 32, 32), k_min=0)
    p = oracle.Params.of(w)
    q0, k0 = q[0, 0].double().numpy(), k[0, 0].double().numpy()
    out = oracle.scope_plan_head(q0, k0, p)
    assert (out["q_labels"] == np.arange(32)).all()
    assert all((c == np.arange(32)).all() for c in out["codes"])
    logits = out["qr"] @ out["kr"].T / np.sqrt(8)
    for i in range(32):
        o = np.lexsort((np.arange(32), -logits[i]))
        wgt = np.exp(logits[i] - logits[i].max())
        cum = np.cumsum(wgt[o]) / wgt.sum()
        m = int(np.argmax(cum >= p.top_p - 1e-15)) + 1
        assert out["r"][i] == min(32, max(m, p.k_min))


# ----------------------------------------------------------------------------- Top-p
def test_order_matches_library_sort_with_ties():
    # score descending, then key index ascending (ties by the lower index)
    rng = np.random.default_rng(21)
    for N in (1, 7, 40):
        sc = rng.integers(0, 5, N).astype(np.float64)  # many exact ties
        want = sorted(range(N), key=lambda j: (-sc[j], j))
        assert oracle.order(sc).tolist() == want


def test_prefix_mass_closed_forms():
    N = 12
    # equal scores: the first m keys hold exactly m/N of the mass
    for m in (0, 1, 5, N):
        assert oracle.prefix_mass(np.zeros(N), m, 0.7) == pytest.approx(m / N, abs=1e-15)
    rng = np.random.default_rng(22)
    sc = rng.standard_normal(N)
    masses = [oracle.prefix_mass(sc, m, 0.5) for m in range(N + 1)]
    assert masses[0] == 0.0 and masses[-1] == pytest.approx(1.0, abs=1e-15)
    assert all(b >= a for a, b in zip(masses, masses[1:]))  # prefixes of the order only add mass
    # the top key alone: its softmax weight, the largest single weight
    w = np.exp(0.5 * (sc - sc.max()))
    assert masses[1] == pytest.approx(w.max() / w.sum(), rel=1e-12)


def test_topp_brute_force_minimal_set():
    rng = np.random.default_rng(8)
    for trial in range(60):
        N = int(rng.integers(1, 11))
        s = rng.integers(-3, 4, N).astype(float) * rng.choice([0.5, 1.0, 3.0])
        p = float(rng.choice([0.3, 0.5, 0.8, 0.9, 0.99]))
        scale = 1.0
        w = np.exp(s - s.max())
        m = oracle.topp_count(s, p, scale)
        sel = set(oracle.emit(s, m).tolist())
        assert len(sel) == m
        # the chosen set reaches p, no smaller set does
        assert w[list(sel)].sum() >= p * w.sum() - 1e-12
        for size in range(m):
            for sub in itertools.combinations(range(N), size):
                assert w[list(sub)].sum() < p * w.sum() + 1e-12
        # among equal scores the lower index wins: the set is the lexicographic
        # first of the best-mass sets of size m
        best = max(itertools.combinations(range(N), m), key=lambda sub: (round(w[list(sub)].sum(), 12), [-i for i in sub]))
        assert sel == set(best)


def test_topp_uniform_closed_form():
    for N, p, m in [(256, 0.9, 231), (256, 0.5, 128), (128, 0.25, 32), (64, 0.999, 64)]:
        assert oracle.topp_count(np.zeros(N), p, 1.0) == m
    assert oracle.topp_count(np.arange(10.0), 1.0, 1.0) == 10


def test_topp_dominant_key():
    s = np.array([0.0, 0.0, 50.0, 0.0])
    assert oracle.topp_count(s, 0.9, 1.0) == 1
    assert oracle.emit(s, 1).tolist() == [2]
    assert oracle.retained_count(s, 0.9, 3, 1.0) == 3
    assert oracle.emit(s, 3).tolist() == [0, 1, 2]  # ties at 0.0 go to the lowest indices


# ----------------------------------------------------------------------------- online Top-k
def test_online_topk_hand_examples():
    g = _gold("online_topk.json")
    for case in g["cases"]:
        K, n = oracle.online_topk(case["sizes"], case["r"], case["N"], online=True)
        assert K == case["K_h"], case["work"]
        assert n.tolist() == case["n"], case["work"]
    K, n = oracle.online_topk([5, 2, 1], [10, 4, 3], 1000, online=False)
    assert n.tolist() == [10, 4, 3]


# ----------------------------------------------------------------------------- attention
def test_full_selection_equals_dense_attention():
    rng = np.random.default_rng(9)
    N, D = 40, 16
    qr, kr, v = (rng.standard_normal((N, D)) * 2 for _ in range(3))
    lab = np.zeros(N, np.int32)
    o = oracle.scope_attn_head(qr, kr, v, lab, [np.arange(N, dtype=np.int32)])
    # independent dense reference: explicit softmax rows
    ref = np.empty_like(o)
    for i in range(N):
        lg = np.array([qr[i] @ kr[j] for j in range(N)]) / 4.0
        e = np.exp(lg - lg.max())
        ref[i] = (e / e.sum()) @ v
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.dense_attention(qr, kr, v), ref, rtol=0, atol=1e-12)


def test_attention_equal_logits_and_single_key():
    rng = np.random.default_rng(10)
    K, V = rng.standard_normal((10, 4)), rng.standard_normal((10, 4))
    sel = np.array([1, 4, 7], np.int32)
    o = oracle.attention_rows(np.zeros((1, 4)), K, V, sel, 0.5)
    np.testing.assert_allclose(o[0], V[sel].mean(0), atol=1e-15)
    o = oracle.attention_rows(rng.standard_normal((2, 4)), K, V, np.array([6], np.int32), 0.5)
    np.testing.assert_allclose(o, V[[6, 6]], atol=1e-15)


# ----------------------------------------------------------------------------- bisection
def test_bisect_balanced_leaves_and_first_split():
    rng = np.random.default_rng(11)
    N, D, leaf = 512, 8, 64
    blob = np.where(rng.permutation(N) < N // 2, 1.0, -1.0)
    x = rng.standard_normal((N, D)) + blob[:, None] * 50.0
    lab, cent, perm = oracle.bisect(x, leaf, 10)
    assert np.bincount(lab).tolist() == [leaf] * (N // leaf)
    assert sorted(perm.tolist()) == list(range(N))
    for c in range(N // leaf):
        members = perm[c * leaf:(c + 1) * leaf]
        assert (lab[members] == c).all()
        assert (np.diff(members) > 0).all()  # token order within a leaf
        np.testing.assert_allclose(cent[c], x[members].mean(0), atol=1e-12)
    first = lab < (N // leaf) // 2
    assert (blob[first] == blob[first][0]).all() and (blob[~first] == -blob[first][0]).all()
    with pytest.raises(ValueError):
        oracle.bisect(x[:448], leaf, 10)  # 7 leaves: not a power of two


def test_bisect_median_split_ties_by_token():
    # points on a line: the lower half of delta (closer to c0) goes to child 0
    x = np.array([[0.0], [10.0], [1.0], [9.0], [2.0], [8.0], [3.0], [7.0]])
    lab, _, _ = oracle.bisect(x, 4, 3)
    assert lab.tolist() == [0, 1, 0, 1, 0, 1, 0, 1]
    # all points equal: every delta ties, so the split is by token index
    lab, _, _ = oracle.bisect(np.ones((8, 2)), 2, 2)
    assert lab.tolist() == [0, 0, 1, 1, 2, 2, 3, 3]


# ----------------------------------------------------------------------------- compensation
# ClusterAttention, abstract: excluded clusters are compensated through their
# mean.  Where a cluster's members are indistinguishable from its mean, the
# compensated attention must equal dense attention whatever is selected.
def test_compensation_with_single_key_clusters_is_dense():
    rng = np.random.default_rng(11)
    N, D = 48, 8
    K, V, q = rng.standard_normal((N, D)), rng.standard_normal((N, D)), rng.standard_normal((5, D))
    dense = oracle.dense_attention(q, K, V)
    for sel in (np.array([], np.int32), np.array([3], np.int32), np.sort(rng.choice(N, 17, replace=False))):
        o = oracle.attention_rows_comp(q, K, V, sel.astype(np.int32), np.arange(N), 1 / np.sqrt(D))
        np.testing.assert_allclose(o, dense, rtol=1e-12, atol=1e-12)


def test_compensation_with_identical_members_is_dense():
    # 6 clusters of 4 identical keys (and identical values): an excluded
    # member counts exactly like the key it copies, so m_k must weight it.
    rng = np.random.default_rng(12)
    C, M, D = 6, 4, 5
    Kc, Vc = 2 * rng.standard_normal((C, D)), rng.standard_normal((C, D))
    klab = np.repeat(np.arange(C), M).astype(np.int32)
    K, V = Kc[klab], Vc[klab]
    q = rng.standard_normal((3, D))
    dense = oracle.dense_attention(q, K, V)
    # select all of cluster 0, one member of cluster 2, nothing else
    sel = np.array([0, 1, 2, 3, 9], np.int32)
    o = oracle.attention_rows_comp(q, K, V, sel, klab, 1 / np.sqrt(D))
    np.testing.assert_allclose(o, dense, rtol=1e-12, atol=1e-12)
    # the uncompensated sparse result differs (the excluded keys carry mass)
    assert np.abs(oracle.attention_rows(q, K, V, sel, 1 / np.sqrt(D)) - dense).max() > 1e-3


def test_compensation_with_everything_selected_is_plain_attention():
    rng = np.random.default_rng(13)
    N, D = 32, 6
    K, V, q = rng.standard_normal((N, D)), rng.standard_normal((N, D)), rng.standard_normal((4, D))
    klab = (np.arange(N) // 8).astype(np.int32)
    sel = np.arange(N, dtype=np.int32)
    np.testing.assert_allclose(oracle.attention_rows_comp(q, K, V, sel, klab, 0.4),
                               oracle.attention_rows(q, K, V, sel, 0.4), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- pipeline
def test_pipeline_tiny_config_invariants():
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_inputs(w)
    p = oracle.Params.of(w)
    for h in range(w.H):
        out = oracle.scope_plan_head(q[0, h].double().numpy(), k[0, h].double().numpy(), p)
        N = w.N
        assert out["q_sizes"].sum() == N
        assert (out["r"] >= min(N, p.k_min)).all() and (out["r"] <= N).all()
        nonempty = out["q_sizes"] > 0
        K = -(-int((out["q_sizes"] * out["r"]).sum()) // N)
        assert out["K_h"] == K
        assert (out["n"][nonempty] >= np.maximum(out["r"][nonempty], K).clip(max=N)).all()
        for c, lst in enumerate(out["lists"]):
            assert len(lst) == out["n"][c]
            assert (np.diff(lst) > 0).all()
        o = oracle.scope_attn_head(out["qr"], out["kr"], v[0, h].double().numpy(), out["q_labels"], out["lists"])
        assert np.isfinite(o).all()


# ----------------------------------------------------------------------------- EG-Sparse (reading R17)
def test_head_entropy_closed_forms():
    N = 64
    scale = 0.5
    assert oracle.head_entropy(np.zeros((3, N)), [1, 2, 3], scale) == pytest.approx(1.0, abs=1e-12)  # uniform rows
    # one key ahead by L: pi = (e^{aL}, 1, ..., 1) / (e^{aL} + N - 1), a two-valued distribution
    L = 12.0
    s = np.zeros((1, N))
    s[0, 5] = L
    z = np.exp(scale * L) + N - 1
    p1, p0 = np.exp(scale * L) / z, 1.0 / z
    H = -(p1 * np.log(p1) + (N - 1) * p0 * np.log(p0))
    assert oracle.head_entropy(s, [7], scale) == pytest.approx(H / np.log(N), rel=1e-12)
    # rows weigh by their query counts; an empty row weighs nothing
    s2 = np.vstack([np.zeros(N), s[0], np.full(N, 3.0)])
    e = oracle.head_entropy(s2, [3, 1, 0], scale)
    assert e == pytest.approx((3 * 1.0 + 1 * H / np.log(N)) / 4, rel=1e-12)


def test_head_entropy_matches_a_library_entropy():
    from scipy.stats import entropy
    rng = np.random.default_rng(11)
    C, N, scale = 5, 40, 0.3
    s = rng.standard_normal((C, N)) * 4
    sizes = rng.integers(1, 9, C)
    rows = [entropy(np.exp(scale * (r - r.max()))) for r in s]  # scipy normalises the weights itself
    ref = float(np.dot(sizes, rows) / (sizes.sum() * np.log(N)))
    assert oracle.head_entropy(s, sizes, scale) == pytest.approx(ref, rel=1e-12)


def test_pooled_topp_hand_examples():
    with open(os.path.join(os.path.dirname(__file__), "golden", "eg_pooled.json")) as f:
        cases = json.load(f)["cases"]
    for cs in cases:
        sizes = np.array(cs["sizes"])
        s = np.zeros(sizes.shape + (cs["N"],))  # equal scores: pi = 1/N everywhere
        assert oracle.pooled_topp(s, sizes, cs["p"], 1.0).tolist() == cs["counts"], cs["work"]


def test_pooled_topp_of_one_row_is_its_topp():
    rng = np.random.default_rng(12)
    for p in (0.3, 0.8, 0.9, 0.999):
        s = rng.standard_normal(50) * 6
        got = oracle.pooled_topp(s[None, None, :], np.array([[4]]), p, 0.4)
        assert got[0, 0] == oracle.topp_count(s, p, 0.4)


def test_pooled_topp_against_a_library_sort():
    """An independent restatement of the pooled prefix (numpy lexsort over all
    entries) on random tiny pools, with rows of unequal sizes and tied scores."""
    rng = np.random.default_rng(13)
    for trial in range(20):
        Hp, C, N = 2, 3, 6
        s = rng.integers(-3, 4, (Hp, C, N)).astype(np.float64)  # integer scores: many ties
        sizes = rng.integers(1, 5, (Hp, C))
        p, scale = rng.uniform(0.2, 0.95), 0.7
        logp, mass, hs, cs, pos = [], [], [], [], []
        for h in range(Hp):
            for c in range(C):
                row = s[h, c]
                order = np.lexsort((np.arange(N), -row))  # score desc, index asc
                a = (row[order] - row.max()) * scale
                a -= np.log(np.exp(a).sum())
                logp += list(a)
                mass += list(sizes[h, c] * np.exp(a))
                hs += [h] * N
                cs += [c] * N
                pos += list(range(N))
        rank = np.lexsort((pos, cs, hs, -np.array(logp)))
        cum = np.cumsum(np.array(mass)[rank])
        m = int(np.searchsorted(cum, p * cum[-1] * (1 - 1e-15))) + 1  # first prefix reaching p
        ref = np.zeros((Hp, C), np.int64)
        for i in rank[:m]:
            ref[hs[i], cs[i]] += 1
        got, frac = oracle.pooled_topp(s, sizes, p, scale, with_mass=True)
        assert (got == ref).all(), (trial, got, ref)
        assert frac >= p * (1 - 1e-12)


def test_eg_route_and_tau_zero_keeps_per_row_selection():
    assert oracle.eg_route([0.1, 0.9, 0.2, 0.3, 0.95], 0.5, 2) == [[0], [2, 3], []]
    assert oracle.eg_route([0.1, 0.2], 0.0, 2) == [[]]
    rng = np.random.default_rng(14)
    H, C, N = 3, 4, 30
    scores = [rng.standard_normal((C, N)) * 5 for _ in range(H)]
    sizes = [rng.integers(0, 6, C) for _ in range(H)]
    _, pools, counts = oracle.eg_counts(scores, sizes, 0.9, 0.0, 2, 0.3)
    assert all(not p for p in pools)
    for h in range(H):
        for c in range(C):
            assert counts[h, c] == oracle.topp_count(scores[h][c], 0.9, 0.3)
    # every head low-entropy, one group: the counts are one pool's
    _, pools, counts = oracle.eg_counts(scores, sizes, 0.9, 1.01, H, 0.3)
    assert pools == [list(range(H))]
    assert (counts == oracle.pooled_topp(np.stack(scores), np.stack(sizes), 0.9, 0.3)).all()


# ----------------------------------------------------------------------------- VMoBA blocks (reading R18)
@pytest.mark.parametrize("grid", [(3, 7, 8), (5, 4, 9), (1, 1, 13)])
@pytest.mark.parametrize("kind,block", [(1, (2, 2, 3)), (2, (1, 3, 4)), (3, (2, 3, 4)), (3, (1, 1, 1))])
def test_block_partition_geometry(grid, kind, block):
    T, Hh, W = grid
    N = T * Hh * W
    ids, nb = oracle.block_ids(grid, kind, block)
    assert ids.min() == 0 and ids.max() == nb - 1 and len(np.unique(ids)) == nb  # every block used
    n = np.arange(N)
    t, y, x = n // (Hh * W), (n // W) % Hh, n % W
    bt, bh, bw = block
    for b in range(nb):
        mem = np.nonzero(ids == b)[0]
        if kind == 1:  # runs of consecutive tokens
            assert (np.diff(mem) == 1).all() and len(mem) <= bt * bh * bw
        else:
            span_t = np.ptp(t[mem]) + 1
            assert span_t <= (1 if kind == 2 else bt)
            assert np.ptp(y[mem]) + 1 <= bh and np.ptp(x[mem]) + 1 <= bw
    sizes = np.bincount(ids)
    if kind == 1:
        assert nb == -(-N // (bt * bh * bw))
        assert (sizes[:-1] == bt * bh * bw).all()
    else:
        ct = T if kind == 2 else -(-T // bt)
        assert nb == ct * -(-Hh // bh) * -(-W // bw)
        assert sizes.max() == (1 if kind == 2 else min(bt, T)) * min(bh, Hh) * min(bw, W)


def test_block_mean_scores_are_member_averages():
    rng = np.random.default_rng(21)
    k = rng.standard_normal((3 * 7 * 8, 16))
    q = rng.standard_normal(16)
    ids, nb = oracle.block_ids((3, 7, 8), 3, (2, 3, 4))
    kbar = oracle.block_means(k, ids, nb)
    for b in range(nb):
        mem = ids == b
        assert q @ kbar[b] * mem.sum() == pytest.approx((k[mem] @ q).sum(), rel=1e-12, abs=1e-12)


def test_block_select_hand_examples():
    with open(os.path.join(os.path.dirname(__file__), "golden", "vmoba_blocks.json")) as f:
        cases = json.load(f)["cases"]
    for cs in cases:
        keep, n = oracle.block_select(np.array(cs["scores"]), np.array(cs["sizes"]), cs["p"], 1.0)
        assert keep.tolist() == cs["keep"] and n == cs["kept_keys"], cs["work"]


def test_single_token_blocks_reduce_to_per_key_topp():
    rng = np.random.default_rng(22)
    for p in (0.5, 0.9, 0.97):
        s = rng.standard_normal(200) * 5  # continuous scores: no ties
        keep, n = oracle.block_select(s, np.ones(200, np.int64), p, 0.3)
        m = oracle.topp_count(s, p, 0.3)
        assert n == m
        assert (np.nonzero(keep)[0] == oracle.emit(s, m)).all()


def test_block_select_grows_with_p():
    rng = np.random.default_rng(23)
    s = rng.standard_normal(60) * 3
    sizes = rng.integers(1, 20, 60)
    counts = [oracle.block_select(s, sizes, p, 0.5)[1] for p in np.linspace(0.05, 1.0, 40)]
    assert all(a <= b for a, b in zip(counts, counts[1:])) and counts[-1] == sizes.sum()
