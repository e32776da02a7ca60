"""fp64 CPU oracle for centroid-guided sparse attention (SCOPE formulation).

TEST INFRASTRUCTURE: only the test suite, the smoke check and the CPU
baseline leg of the benchmark may import this package.  It shares no code with
the CUDA path (its arithmetic lives in scope_oracle.c, compiled with gcc, and
in the plain numpy glue below) and never calls it.

Steps, in the order of the SCOPE abstract ("SCOPE: Subspace Clustering with
Online Per-Head Top-K Estimation for Sparse Video Attention"):
  1. 3D-RoPE on Q and K; post-RoPE keys split into t/h/w subspaces
  2. independent k-means per key subspace; k-means of the queries
  3. per-(query cluster, key) proxy scores = sum of centroid-dot lookup tables
  4. hybrid Top-p / fixed Top-k, then the online per-head Top-k top-up
  5. exact attention over the selected original keys and values
and, for the unstructured variant of "ClusterAttention: A training-free
speedup of bidirectional attention" (abstract), balanced recursive bisection
to fixed power-of-two clusters in place of steps 1-2.

Every function follows one step; the readings of points the pages leave open
are written beside the C functions (R1..R14).  Nothing here is pinned by a
value printed on the pages (they print none); the pins are closed forms,
invariants and brute force in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "scope_oracle.c")
_LIB = os.path.join(_HERE, "_scope_oracle.so")
_lib = None

_d = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32 = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64 = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_I = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/_scope_oracle.so (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.orc_rope3d.argtypes = [_d, _I, _I, _i32, _i32, ctypes.c_double]
        L.orc_rope3d.restype = ctypes.c_int
        L.orc_kmeans_assign.argtypes = [_d, _I, _I, _I, _d, _I, _I, _i32, ctypes.c_void_p, ctypes.c_void_p]
        L.orc_kmeans_update.argtypes = [_d, _I, _I, _I, _i32, _I, _d, _I, ctypes.c_void_p]
        L.orc_kmeans_objective.argtypes = [_d, _I, _I, _I, _i32, _d, _I]
        L.orc_kmeans_objective.restype = ctypes.c_double
        L.orc_kmeans.argtypes = [_d, _I, _I, _I, _I, ctypes.c_int, ctypes.c_uint32, _i32, _d, _i64]
        L.orc_kmeans.restype = ctypes.c_int
        L.orc_lut.argtypes = [_d, _I, _I, _d, _I, _I, _I, _d]
        L.orc_proxy_scores.argtypes = [_d, _d, _d, _i32, _i32, _i32, _I, _d]
        L.orc_order.argtypes = [_d, _I, _i64]
        L.orc_topp_count.argtypes = [_d, _I, ctypes.c_double, ctypes.c_double, ctypes.c_void_p]
        L.orc_topp_count.restype = ctypes.c_int64
        L.orc_prefix_mass.argtypes = [_d, _I, _I, ctypes.c_double]
        L.orc_prefix_mass.restype = ctypes.c_double
        L.orc_online_topk.argtypes = [_i64, _i64, _I, _I, ctypes.c_int, _i64]
        L.orc_online_topk.restype = ctypes.c_int64
        L.orc_emit.argtypes = [_d, _I, _I, _i32]
        L.orc_attn_rows.argtypes = [_d, _I, _d, _d, _I, _i32, _I, ctypes.c_double, _d]
        L.orc_bisect.argtypes = [_d, _I, _I, _I, ctypes.c_int, _i32, _d, _i64]
        L.orc_attn_rows_comp.argtypes = [_d, _I, _d, _d, _I, _I, _i32, _I, _i32, _I, ctypes.c_double, _d]
        L.orc_bisect.restype = ctypes.c_int
        L.orc_head_entropy.argtypes = [_d, _i64, _I, _I, ctypes.c_double]
        L.orc_head_entropy.restype = ctypes.c_double
        L.orc_pooled_topp.argtypes = [_d, _i64, _I, _I, _I, ctypes.c_double, ctypes.c_double, _i64]
        L.orc_pooled_topp.restype = ctypes.c_double
        L.orc_block_ids.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int, ctypes.c_int32,
                                    ctypes.c_int32, ctypes.c_int32, _i32]
        L.orc_block_ids.restype = ctypes.c_int64
        L.orc_block_select.argtypes = [_d, _i64, _I, ctypes.c_double, ctypes.c_double,
                                       np.ctypeslib.ndpointer(dtype=np.int8, flags="C_CONTIGUOUS")]
        L.orc_block_select.restype = ctypes.c_int64
        _lib = L
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------- steps
def rope3d(x, grid, d_split, theta) -> np.ndarray:
    """Step 1: 3D-RoPE of one head's [N, D] rows (identity without a grid)."""
    y = _f64(x).copy()
    N, D = y.shape
    rc = lib().orc_rope3d(y, N, D, np.asarray(grid, np.int32), np.asarray(d_split, np.int32), float(theta))
    if rc:
        raise ValueError(f"rope3d: bad shape (code {rc})")
    return y


def kmeans_assign(x, cent, with_dists: bool = False):
    """argmin_j ||x_n - c_j||^2 per row, lowest j on ties."""
    x, cent = _f64(x), _f64(cent)
    N, D = x.shape
    C = cent.shape[0]
    lab = np.empty(N, np.int32)
    d1 = np.empty(N) if with_dists else None
    d2 = np.empty(N) if with_dists else None
    lib().orc_kmeans_assign(x, N, D, D, cent, C, D, lab, _ptr(d1), _ptr(d2))
    return (lab, d1, d2) if with_dists else lab


def kmeans_update(x, labels, cent_prev):
    """New centroids = member means; an empty cluster keeps its previous centroid."""
    x = _f64(x)
    N, D = x.shape
    cent = _f64(cent_prev).copy()
    sizes = np.empty(cent.shape[0], np.int64)
    lib().orc_kmeans_update(x, N, D, D, np.ascontiguousarray(labels, np.int32), cent.shape[0], cent, D, _ptr(sizes))
    return cent, sizes


def kmeans_objective(x, labels, cent) -> float:
    x, cent = _f64(x), _f64(cent)
    N, D = x.shape
    return lib().orc_kmeans_objective(x, N, D, D, np.ascontiguousarray(labels, np.int32), cent, D)


def kmeans(x, C: int, iters: int, seed: int = 0):
    """Lloyd k-means with the strided init; returns (labels, centroids, sizes)."""
    x = _f64(x)
    N, D = x.shape
    lab = np.empty(N, np.int32)
    cent = np.empty((C, max(D, 1)), np.float64)[:, :D].copy()
    sizes = np.empty(C, np.int64)
    rc = lib().orc_kmeans(x, N, D, D, C, int(iters), int(seed) & 0xFFFFFFFF, lab, cent, sizes)
    if rc:
        raise ValueError("kmeans: need 1 <= C <= N")
    return lab, cent, sizes


def lut(qc_sub, kc_sub) -> np.ndarray:
    """[Cq, Ck] dot products of query centroids and key centroids of one subspace."""
    qc, kc = _f64(qc_sub), _f64(kc_sub)
    Cq, Ds = qc.shape
    Ck = kc.shape[0]
    out = np.empty((Cq, Ck))
    lib().orc_lut(qc, Cq, Ds, kc, Ck, Ds, Ds, out)
    return out


def proxy_scores(lut_rows, codes) -> np.ndarray:
    """Per-key proxy scores of one query cluster from its three table rows."""
    N = codes[0].shape[0]
    s = np.empty(N)
    lib().orc_proxy_scores(_f64(lut_rows[0]), _f64(lut_rows[1]), _f64(lut_rows[2]),
                           *[np.ascontiguousarray(c, np.int32) for c in codes], N, s)
    return s


def order(s) -> np.ndarray:
    s = _f64(s)
    o = np.empty(s.shape[0], np.int64)
    lib().orc_order(s, s.shape[0], o)
    return o


def topp_count(s, p: float, scale: float, with_mass: bool = False):
    s = _f64(s)
    mass = ctypes.c_double(0.0)
    m = lib().orc_topp_count(s, s.shape[0], float(p), float(scale), ctypes.byref(mass))
    return (int(m), mass.value) if with_mass else int(m)


def prefix_mass(s, m: int, scale: float) -> float:
    s = _f64(s)
    return lib().orc_prefix_mass(s, s.shape[0], int(m), float(scale))


def retained_count(s, p: float, k_min: int, scale: float) -> int:
    """Initial (hybrid Top-p / fixed Top-k) count r_c = min(N, max(|P_c|, k_min))."""
    return int(min(len(s), max(topp_count(s, p, scale), k_min)))


def online_topk(sizes, r, N: int, online: bool = True):
    """(K_h, n_c): the per-head Top-k and each cluster's final key count."""
    sizes = np.ascontiguousarray(sizes, np.int64)
    r = np.ascontiguousarray(r, np.int64)
    n = np.empty_like(r)
    K = lib().orc_online_topk(sizes, r, sizes.shape[0], int(N), int(bool(online)), n)
    return int(K), n


def emit(s, n: int) -> np.ndarray:
    """The first n keys of the (score desc, index asc) order, ascending."""
    s = _f64(s)
    out = np.empty(int(n), np.int32)
    lib().orc_emit(s, s.shape[0], int(n), out)
    return out


def head_entropy(scores, sizes, scale: float) -> float:
    """EG-Sparse head entropy: query-size-weighted mean row entropy of the
    proxy softmax, over ln N (R17).  scores [C, N], sizes [C]."""
    sc = _f64(scores)
    C, N = sc.shape
    return lib().orc_head_entropy(sc, np.ascontiguousarray(sizes, np.int64), C, N, float(scale))


def pooled_topp(scores, sizes, p: float, scale: float, with_mass: bool = False):
    """EG-Sparse pooled Top-p counts of one pool of heads (R17).
    scores [Hp, C, N], sizes [Hp, C] -> counts [Hp, C] (and the kept mass fraction)."""
    sc = _f64(scores)
    Hp, C, N = sc.shape
    counts = np.empty((Hp, C), np.int64)
    mass = lib().orc_pooled_topp(sc, np.ascontiguousarray(sizes, np.int64), Hp, C, N, float(p), float(scale),
                                 counts)
    return (counts, mass) if with_mass else counts


def eg_route(entropies, tau: float, group: int):
    """Pools of one batch entry: for each group of `group` consecutive heads,
    the list of its heads whose entropy is below tau (R17)."""
    H = len(entropies)
    pools = []
    for g0 in range(0, H, group):
        pools.append([h for h in range(g0, min(H, g0 + group)) if entropies[h] < tau])
    return pools


def eg_counts(scores_heads, sizes_heads, p: float, tau: float, group: int, scale: float):
    """EG-Sparse Top-p counts of one batch entry's heads (R17).
    scores_heads: per head [C, N] proxy scores; sizes_heads: per head [C].
    Returns (entropies [H], pools, counts [H, C]): pooled heads take their
    counts from their pool, the others from their own rows."""
    H = len(scores_heads)
    ent = [head_entropy(s, z, scale) for s, z in zip(scores_heads, sizes_heads)]
    pools = eg_route(ent, tau, group)
    C, N = np.asarray(scores_heads[0]).shape
    counts = np.empty((H, C), np.int64)
    for h in range(H):
        for c in range(C):
            counts[h, c] = topp_count(scores_heads[h][c], p, scale) if p < 1.0 else N
    for pool in pools:
        if pool:
            counts[pool] = pooled_topp(np.stack([scores_heads[h] for h in pool]),
                                       np.stack([sizes_heads[h] for h in pool]), p, scale)
    return ent, pools, counts


def block_ids(grid, kind: int, block):
    """VMoBA block partition (R18): block id of every token and the block count."""
    T, Hh, W = grid
    ids = np.empty(T * Hh * W, np.int32)
    nb = lib().orc_block_ids(T, Hh, W, int(kind), *[int(x) for x in block], ids)
    return ids, int(nb)


def block_means(x, ids, nb: int) -> np.ndarray:
    """Mean row of every block (fp64); an empty block has a zero mean."""
    x = _f64(x)
    out = np.zeros((nb, x.shape[1]))
    cnt = np.bincount(ids, minlength=nb).astype(np.float64)
    np.add.at(out, ids, x)
    return out / np.maximum(cnt, 1.0)[:, None]


def block_select(s, sizes, p: float, scale: float):
    """VMoBA threshold selection of one query cluster over blocks (R18):
    (kept block flags, kept key count)."""
    s = _f64(s)
    keep = np.empty(s.shape[0], np.int8)
    n = lib().orc_block_select(s, np.ascontiguousarray(sizes, np.int64), s.shape[0], float(p), float(scale), keep)
    return keep.astype(bool), int(n)


def vmoba_plan_head(q, k, p: "Params", kind: int, block, store_bf16: bool = False) -> dict:
    """Block-granular variant for one head: SCOPE's RoPE and query k-means,
    key blocks of the given partition scored by their mean key, threshold
    selection of whole blocks; lists = the kept blocks' keys, ascending."""
    q, k = _f64(q), _f64(k)
    N, D = q.shape
    scale = 1.0 / np.sqrt(D)
    qr = rope3d(q, p.grid, p.d_split, p.theta)
    kr = rope3d(k, p.grid, p.d_split, p.theta)
    if store_bf16:
        qr, kr = _round_bf16(qr), _round_bf16(kr)
    qlab, qcent, qsizes = kmeans(qr, p.c_q, p.iters, p.seed)
    ids, nb = block_ids(p.grid, kind, block)
    kbar = block_means(kr, ids, nb)
    bsizes = np.bincount(ids, minlength=nb).astype(np.int64)
    lists, n = [], np.zeros(p.c_q, np.int64)
    for c in range(p.c_q):
        keep, n[c] = block_select(qcent[c] @ kbar.T, bsizes, p.top_p, scale)
        lists.append(np.nonzero(keep[ids])[0].astype(np.int32))
    return dict(qr=qr, kr=kr, q_labels=qlab, q_centroids=qcent, q_sizes=qsizes, block_ids=ids,
                block_means=kbar, n=n, lists=lists)


def attention_rows(q_rows, K, V, sel, scale: float) -> np.ndarray:
    q_rows, K, V = _f64(q_rows), _f64(K), _f64(V)
    sel = np.ascontiguousarray(sel, np.int32)
    o = np.empty_like(q_rows)
    lib().orc_attn_rows(q_rows, q_rows.shape[0], K, V, K.shape[1], sel, sel.shape[0], float(scale), o)
    return o


def attention_rows_comp(q_rows, K, V, sel, klab, scale: float) -> np.ndarray:
    """Attention over the selected keys plus every excluded key entering through
    its key cluster's mean key and mean value (ClusterAttention compensation,
    reading R16); klab[j] is key j's cluster."""
    q_rows, K, V = _f64(q_rows), _f64(K), _f64(V)
    sel = np.ascontiguousarray(sel, np.int32)
    klab = np.ascontiguousarray(klab, np.int32)
    C = int(klab.max()) + 1 if klab.size else 0
    o = np.empty_like(q_rows)
    lib().orc_attn_rows_comp(q_rows, q_rows.shape[0], K, V, K.shape[0], K.shape[1], sel, sel.shape[0], klab, C,
                             float(scale), o)
    return o


def bisect(x, leaf: int, iters: int):
    """Balanced recursive bisection: (labels, leaf centroids, permutation)."""
    x = _f64(x)
    N, D = x.shape
    lab = np.empty(N, np.int32)
    cent = np.empty((N // leaf, D))
    perm = np.empty(N, np.int64)
    if lib().orc_bisect(x, N, D, int(leaf), int(iters), lab, cent, perm):
        raise ValueError("bisect: N must be leaf * 2^L")
    return lab, cent, perm


# --------------------------------------------------------------------------- pipeline
@dataclass
class Params:
    grid: tuple
    d_split: tuple
    theta: float
    c_q: int
    c_sub: tuple
    iters: int
    top_p: float
    k_min: int
    online_topk: int
    fixed_cluster_size: int
    seed: int = 0

    @staticmethod
    def of(w) -> "Params":
        return Params(tuple(w.grid), tuple(w.d_split), w.theta, w.c_q, tuple(w.c_sub), w.iters,
                      w.top_p, w.k_min, w.online_topk, w.fixed_cluster_size)


def _round_bf16(x: np.ndarray) -> np.ndarray:
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float64).numpy()


def scope_plan_head(q, k, p: Params, store_bf16: bool = False, clusters=None) -> dict:
    """Steps 1-4 for one head.  `store_bf16` rounds the post-RoPE Q/K to bf16
    before clustering (the CUDA path stores them that way); `clusters`
    optionally restricts the selection work to those query clusters."""
    q, k = _f64(q), _f64(k)
    N, D = q.shape
    scale = 1.0 / np.sqrt(D)
    qr = rope3d(q, p.grid, p.d_split, p.theta)
    kr = rope3d(k, p.grid, p.d_split, p.theta)
    if store_bf16:
        qr, kr = _round_bf16(qr), _round_bf16(kr)
    offs = np.cumsum((0,) + tuple(p.d_split))
    if p.fixed_cluster_size > 0:
        qlab, qcent, _ = bisect(qr, p.fixed_cluster_size, p.iters)
        klab, kcent, _ = bisect(kr, p.fixed_cluster_size, p.iters)
        C = N // p.fixed_cluster_size
        qsizes = np.bincount(qlab, minlength=C).astype(np.int64)
        codes = [klab, np.zeros(N, np.int32), np.zeros(N, np.int32)]
        kcents = [kcent, np.zeros((1, 0)), np.zeros((1, 0))]
        sub = [(0, D), (D, D), (D, D)]
    else:
        codes, kcents, sub = [], [], []
        for s in range(3):
            a, b = int(offs[s]), int(offs[s + 1])
            lab_s, cent_s, _ = kmeans(kr[:, a:b], p.c_sub[s], p.iters, p.seed)
            codes.append(lab_s)
            kcents.append(cent_s)
            sub.append((a, b))
        qlab, qcent, qsizes = kmeans(qr, p.c_q, p.iters, p.seed)
        C = p.c_q
    luts = [lut(qcent[:, a:b], kc) for (a, b), kc in zip(sub, kcents)]
    cl = range(C) if clusters is None else clusters
    r = np.zeros(C, np.int64)
    for c in cl:
        s = proxy_scores([L[c] for L in luts], codes)
        r[c] = retained_count(s, p.top_p, p.k_min, scale)
    out = dict(qr=qr, kr=kr, q_labels=qlab, q_centroids=qcent, q_sizes=qsizes, codes=codes,
               k_centroids=kcents, luts=luts, r=r)
    if clusters is None:
        K, n = online_topk(qsizes, r, N, bool(p.online_topk))
        lists = [emit(proxy_scores([L[c] for L in luts], codes), n[c]) for c in range(C)]
        out.update(K_h=K, n=n, lists=lists)
    return out


def scope_attn_head(qr, kr, v, q_labels, lists, rows=None) -> np.ndarray:
    """Step 5 for one head: each query attends over its cluster's selected keys."""
    qr, kr, v = _f64(qr), _f64(kr), _f64(v)
    N, D = qr.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    o = np.zeros((len(rows), D))
    for i, n in enumerate(rows):
        o[i] = attention_rows(qr[n:n + 1], kr, v, lists[q_labels[n]], 1.0 / np.sqrt(D))[0]
    return o


def dense_attention(qr, kr, v) -> np.ndarray:
    """Plain softmax attention over all keys (fp64), for fidelity reports."""
    qr, kr, v = _f64(qr), _f64(kr), _f64(v)
    lg = qr @ kr.T / np.sqrt(qr.shape[1])
    lg -= lg.max(axis=1, keepdims=True)
    w = np.exp(lg)
    return (w / w.sum(axis=1, keepdims=True)) @ v
