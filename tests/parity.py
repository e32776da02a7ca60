"""Stage-fed parity between the CUDA path and the fp64 oracle.

Each check feeds the oracle the GPU's own inputs to that stage (post-RoPE
bf16 rows, fp32 centroids, fp32 lookup tables, codes) so integer outputs can
be compared exactly:
  * RoPE: every element within one bf16 ulp of the fp64 rotation.
  * assignment: labels equal the fp64 argmin except near-ties (the two fp64
    distances within 1e-5 relative); near-ties < 0.01% of the checked rows.
  * update: centroids within 1e-5 of the centroid norm of the fp64 mean.
  * LUT: within 1e-6 of |q_c^s| |mu^s| of the fp64 dot.
  * Top-p counts: equal, or a near-tie (the fp64 prefix mass at both cuts
    within 1e-5 relative of p); K_h, n_c and the lists exact given the GPU's
    counts.
  * attention: max-abs <= 2e-2 and rel-L2 <= 5e-3 against fp64 attention over
    the GPU's selected lists.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TIE_REL = 1e-5
TIE_FRAC = 1e-4
ATTN_MAX_ABS = 2e-2
ATTN_REL_L2 = 5e-3


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 7), 2.0 ** -133)


def check_rope(gpu_rows: np.ndarray, raw: np.ndarray, w, rows=None) -> None:
    """gpu_rows: the device's post-RoPE rows `rows` of one head; raw: all N input rows."""
    ref = oracle.rope3d(raw, w.grid, w.d_split, w.theta)
    if rows is not None:
        ref = ref[rows]
    err = np.abs(gpu_rows - ref)
    bad = err > bf16_ulp(ref) * 1.0000001
    assert not bad.any(), f"RoPE: {bad.sum()} elements beyond 1 bf16 ulp (max err {err.max():.3g})"


class TieCounter:
    def __init__(self):
        self.checked = 0
        self.ties = 0

    def assert_ok(self, what=""):
        assert self.ties <= TIE_FRAC * max(self.checked, 1), \
            f"{what}: {self.ties} near-ties in {self.checked} checks (> {TIE_FRAC:.0e})"


def check_assign(x: np.ndarray, cent: np.ndarray, labels: np.ndarray, tc: TieCounter, what="assign") -> None:
    ref, d1, _ = oracle.kmeans_assign(x, cent, with_dists=True)
    mism = np.nonzero(ref != labels)[0]
    tc.checked += len(labels)
    for n in mism:
        dg = float(((x[n] - cent[labels[n]]) ** 2).sum())
        do = float(d1[n])
        assert abs(dg - do) <= TIE_REL * max(dg, do, 1e-30), \
            f"{what}: row {n} label {labels[n]} vs oracle {ref[n]} (d {dg:.9g} vs {do:.9g})"
        tc.ties += 1


def check_update(x: np.ndarray, labels_prev: np.ndarray, cent_prev: np.ndarray, cent: np.ndarray,
                 what="update") -> None:
    ref, _ = oracle.kmeans_update(x, labels_prev, cent_prev)
    if ref.shape[1] == 0:
        return
    err = np.linalg.norm(cent - ref, axis=1)
    tol = TIE_REL * np.maximum(np.linalg.norm(ref, axis=1), 1e-3)
    assert (err <= tol).all(), f"{what}: max centroid err {err.max():.3g} (tol {tol[err.argmax()]:.3g})"


def check_lut(qcent: np.ndarray, kcents, d_split, lut: np.ndarray) -> None:
    offs = np.cumsum((0,) + tuple(d_split))
    col = 0
    for s, kc in enumerate(kcents):
        a, b = int(offs[s]), int(offs[s + 1])
        Cs = kc.shape[0]
        if b > a:
            ref = oracle.lut(qcent[:, a:b], kc)
            scale = np.outer(np.linalg.norm(qcent[:, a:b], axis=1), np.linalg.norm(kc, axis=1))
            err = np.abs(lut[:, col:col + Cs] - ref)
            assert (err <= 1e-6 * scale + 1e-30).all(), f"LUT subspace {s}: max rel err {(err / (scale + 1e-30)).max():.3g}"
        else:
            assert (lut[:, col:col + Cs] == 0).all()
        col += Cs


def scores_f32(lut_row: np.ndarray, codes, C_sub) -> np.ndarray:
    """Per-key proxy scores exactly as the device forms them: fp32 (t + h) + w."""
    L = lut_row.astype(np.float32)
    Ct, Ch, _ = C_sub
    return ((L[codes[0]] + L[Ct + codes[1]]) + L[Ct + Ch + codes[2]]).astype(np.float64)


def check_selection(lut, codes, sizes, r_gpu, kh_gpu, n_gpu, lists_gpu, w, N, D, clusters, tc: TieCounter):
    """lut [Cq, Csum] f32; codes 3x[N]; lists_gpu: callable c -> int32 array."""
    p32 = float(np.float32(w.top_p))
    scale = 1.0 / np.sqrt(D)
    for c in clusters:
        s = scores_f32(lut[c], codes, w.c_sub)
        m_orc = oracle.topp_count(s, p32, scale) if p32 < 1.0 else N
        r_orc = min(N, max(m_orc, w.k_min))
        tc.checked += 1
        if r_orc != int(r_gpu[c]):
            lo, hi = sorted((r_orc, int(r_gpu[c])))
            m_lo, m_hi = oracle.prefix_mass(s, lo, scale), oracle.prefix_mass(s, hi - 1, scale)
            assert abs(m_lo - p32) <= TIE_REL * p32 and abs(m_hi - p32) <= TIE_REL * p32, \
                f"cluster {c}: r {int(r_gpu[c])} vs oracle {r_orc} (mass {m_lo:.9f}/{m_hi:.9f}, p {p32})"
            tc.ties += 1
    K, n_ref = oracle.online_topk(sizes, r_gpu, N, bool(w.online_topk))
    assert (not w.online_topk) or K == int(kh_gpu), f"K_h {int(kh_gpu)} vs {K}"
    assert (n_ref == n_gpu).all(), "n_c differs from the oracle given the device's r_c"
    for c in clusters:
        s = scores_f32(lut[c], codes, w.c_sub)
        ref = oracle.emit(s, int(n_gpu[c]))
        got = lists_gpu(c)
        assert len(got) == len(ref) and (got == ref).all(), f"cluster {c}: selected list differs"


def attn_error(o_gpu: np.ndarray, o_ref: np.ndarray):
    max_abs = float(np.abs(o_gpu - o_ref).max())
    rel = float(np.linalg.norm(o_gpu - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    return max_abs, rel


def check_attention(qr, kr, v, labels, lists_gpu, o_gpu, rows) -> tuple:
    D = qr.shape[1]
    ref = np.stack([oracle.attention_rows(qr[n:n + 1], kr, v, lists_gpu(labels[n]), 1.0 / np.sqrt(D))[0]
                    for n in rows])
    max_abs, rel = attn_error(o_gpu[rows], ref)
    assert max_abs <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, f"attention: max-abs {max_abs:.3g}, rel-L2 {rel:.3g}"
    return max_abs, rel
