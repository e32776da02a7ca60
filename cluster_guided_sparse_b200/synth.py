"""Seeded synthetic inputs shaped like the workloads of the SCOPE and
ClusterAttention pages.

The pages measure on video-DiT activations (HunyuanVideo 720p, Wan 2.1 480p)
and on tabular TabPFN-3 activations; none of those models, weights or datasets
exist here, so these generators stand in for them with the same shapes and a
controllable cluster structure:

* per head, M unit-norm component means shared by Q and K (V has its own),
* every token draws a component label (uniform, or Zipf-sized for the
  unstructured variant) and adds isotropic noise of norm ~sigma,
* grid workloads add a smooth field whose (t, h, w) dimension blocks hold
  (sin(pos/4), cos(pos/4)) pairs, normalised to norm 0.5,
* Q and K are scaled by sqrt(L * sqrt(d)), L = 8, so a same-component,
  same-position logit q.k/sqrt(d) is about 8 (without a gain the attention
  would be uniform and there would be nothing to sparsify).

This module holds none of the method's arithmetic (no RoPE, clustering,
scoring or selection); both the oracle tests and the CUDA path read their
inputs from here, which is the only code they share.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

BASE_SEED = 20261202
LOGIT_GAIN = 8.0
FIELD_NORM = 0.5


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, input recipe and the method's knobs."""

    name: str
    config_id: int
    B: int
    H: int
    N: int
    D: int
    grid: tuple  # (T, Hh, W) or (0, 0, 0)
    dtype: str  # "f32" | "bf16"
    components: int
    sigma: tuple  # (lo, hi): per-head noise norm, linear over heads
    zipf_alpha: float  # 0 = uniform component labels
    # method parameters
    d_split: tuple  # (d_t, d_h, d_w)
    theta: float
    c_q: int
    c_sub: tuple  # (C_t, C_h, C_w)
    iters: int
    top_p: float
    k_min: int
    online_topk: int
    fixed_cluster_size: int
    # (bt, bh, bw): tokens of one grid block share one component label, blocks
    # draw their labels independently (objects occupying regions); None = every
    # token draws its own label.
    label_block: Optional[tuple] = None
    # ClusterAttention variant: compensate excluded key clusters through their mean
    compensate: int = 0
    # EG-Sparse routing: entropy threshold (0 = off) and head group size
    eg_tau: float = 0.0
    eg_group: int = 1
    # VMoBA block-granular selection: 0 off, 1/2/3 = 1D/2D/3D key blocks of block_dims
    block_kind: int = 0
    block_dims: tuple = (4, 4, 4)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def dense_flops(self) -> float:
        """4 * B * H * N^2 * d: QK^T plus PV of dense attention."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.D


WORKLOADS = {
    "tiny": Workload(
        name="tiny SCOPE call (B=1,H=2,d=64, grid 4x8x8, N=256, fp32)",
        config_id=1, B=1, H=2, N=256, D=64, grid=(4, 8, 8), dtype="f32",
        components=8, sigma=(0.3, 0.3), zipf_alpha=0.0,
        d_split=(16, 24, 24), theta=10000.0, c_q=8, c_sub=(4, 4, 4), iters=10,
        top_p=0.9, k_min=16, online_topk=1, fixed_cluster_size=0),
    "small": Workload(
        name="small video shape (B=1,H=8,d=128, grid 8x16x16, N=2048, bf16)",
        config_id=2, B=1, H=8, N=2048, D=128, grid=(8, 16, 16), dtype="bf16",
        components=16, sigma=(0.3, 0.3), zipf_alpha=0.0,
        d_split=(16, 56, 56), theta=10000.0, c_q=32, c_sub=(8, 16, 16), iters=10,
        top_p=0.9, k_min=64, online_topk=1, fixed_cluster_size=0),
    "wan480p": Workload(
        name="Wan-2.1-480p-shaped layer (B=1,H=40,d=128, grid 21x30x52, N=32760, bf16)",
        config_id=3, B=1, H=40, N=32760, D=128, grid=(21, 30, 52), dtype="bf16",
        components=64, sigma=(0.1, 1.0), zipf_alpha=0.0,
        d_split=(16, 56, 56), theta=10000.0, c_q=256, c_sub=(16, 32, 32), iters=10,
        top_p=0.9, k_min=256, online_topk=1, fixed_cluster_size=0),
    "hunyuan720p": Workload(
        name="HunyuanVideo-720p-shaped layer (B=1,H=24,d=128, grid 33x45x80, N=118800, bf16)",
        config_id=4, B=1, H=24, N=118800, D=128, grid=(33, 45, 80), dtype="bf16",
        components=128, sigma=(0.1, 1.0), zipf_alpha=0.0,
        d_split=(16, 56, 56), theta=10000.0, c_q=512, c_sub=(16, 32, 32), iters=10,
        top_p=0.9, k_min=0, online_topk=1, fixed_cluster_size=0),
    # The same layer with spatially coherent content: tokens of one 11x15x16
    # grid block share a component label (objects occupying regions), which
    # the proxy scores resolve far more sharply than i.i.d. labels.  A second,
    # separately labelled measurement; the 720p line above stays the headline.
    "hunyuan720p_regions": Workload(
        name="HunyuanVideo-720p-shaped layer, region-coherent content (B=1,H=24,d=128, grid 33x45x80, "
             "N=118800, bf16, labels shared by 11x15x16 blocks)",
        config_id=6, B=1, H=24, N=118800, D=128, grid=(33, 45, 80), dtype="bf16",
        components=128, sigma=(0.1, 1.0), zipf_alpha=0.0,
        d_split=(16, 56, 56), theta=10000.0, c_q=512, c_sub=(16, 32, 32), iters=10,
        top_p=0.9, k_min=0, online_topk=1, fixed_cluster_size=0, label_block=(11, 15, 16)),
    "unstructured": Workload(
        name="unstructured bidirectional variant (B=1,H=6,d=64, N=65536, no grid, bf16)",
        config_id=5, B=1, H=6, N=65536, D=64, grid=(0, 0, 0), dtype="bf16",
        components=1024, sigma=(0.3, 0.3), zipf_alpha=1.2,
        d_split=(64, 0, 0), theta=10000.0, c_q=1024, c_sub=(1024, 1, 1), iters=10,
        top_p=0.9, k_min=512, online_topk=1, fixed_cluster_size=64),
}


def head_sigma(w: Workload, h: int) -> float:
    lo, hi = w.sigma
    if w.H == 1 or lo == hi:
        return float(lo)
    return float(lo + (hi - lo) * h / (w.H - 1))


def _streams(w: Workload, seed: int):
    root = np.random.SeedSequence(BASE_SEED + w.config_id + 1000 * seed)
    means, labels, qn, kn, vn = root.spawn(5)
    return [s.spawn(w.B * w.H) for s in (means, labels, qn, kn, vn)]


def grid_field(w: Workload) -> Optional[np.ndarray]:
    """[N, D] float64 field: each (t|h|w) dimension block holds the pair
    (sin(pos/4), cos(pos/4)) of its own axis, scaled to norm FIELD_NORM."""
    T, Hh, W = w.grid
    if T == 0:
        return None
    n = np.arange(w.N)
    pos = (n // (Hh * W), (n // W) % Hh, n % W)
    f = np.zeros((w.N, w.D))
    off = 0
    for ds, p in zip(w.d_split, pos):
        for i in range(ds // 2):
            f[:, off + 2 * i] = np.sin(p / 4.0)
            f[:, off + 2 * i + 1] = np.cos(p / 4.0)
        off += ds
    return f * (FIELD_NORM / np.sqrt(w.D / 2.0))


def make_head(w: Workload, b: int, h: int, seed: int = 0, field=None):
    """Q, K, V of one (batch, head) as float32 numpy arrays [N, D]."""
    st = _streams(w, seed)
    bh = b * w.H + h
    g_means = np.random.Generator(np.random.PCG64(st[0][bh]))
    g_lab = np.random.Generator(np.random.PCG64(st[1][bh]))
    M, D, N = w.components, w.D, w.N
    mu = g_means.standard_normal((M, D))
    mu /= np.linalg.norm(mu, axis=1, keepdims=True)
    nu = g_means.standard_normal((M, D))
    nu /= np.linalg.norm(nu, axis=1, keepdims=True)
    if w.zipf_alpha > 0:
        pm = (np.arange(M) + 1.0) ** (-w.zipf_alpha)
        lab = g_lab.choice(M, size=N, p=pm / pm.sum())
    elif w.label_block is not None:
        T, Hh, W = w.grid
        lbt, lbh, lbw = w.label_block
        nb = (-(-T // lbt), -(-Hh // lbh), -(-W // lbw))
        n = np.arange(N)
        t, y, x = n // (Hh * W), (n // W) % Hh, n % W
        block = ((t // lbt) * nb[1] + y // lbh) * nb[2] + x // lbw
        lab = g_lab.integers(0, M, size=nb[0] * nb[1] * nb[2])[block]
    else:
        lab = g_lab.integers(0, M, size=N)
    s = head_sigma(w, h) / np.sqrt(D)
    out = []
    for which, (mean, stream) in enumerate(((mu, st[2]), (mu, st[3]), (nu, st[4]))):
        g = np.random.Generator(np.random.PCG64(stream[bh]))
        x = mean[lab].astype(np.float32)
        x += (s * g.standard_normal((N, D), dtype=np.float32))
        if field is not None:
            x += field.astype(np.float32)
        if which < 2:
            x *= np.float32(np.sqrt(LOGIT_GAIN * np.sqrt(D)))
        out.append(x)
    return out[0], out[1], out[2], lab


def make_inputs(w: Workload, seed: int = 0, heads=None):
    """Q, K, V as CPU torch tensors [B, H', N, D] in the workload's dtype.

    heads: optional list of head indices (all heads by default); a head's
    values do not depend on which other heads are generated.
    """
    heads = list(range(w.H)) if heads is None else list(heads)
    field = grid_field(w)
    td = w.torch_dtype
    q = torch.empty((w.B, len(heads), w.N, w.D), dtype=td)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    for b in range(w.B):
        for i, h in enumerate(heads):
            qh, kh, vh, _ = make_head(w, b, h, seed, field)
            q[b, i] = torch.from_numpy(qh).to(td)
            k[b, i] = torch.from_numpy(kh).to(td)
            v[b, i] = torch.from_numpy(vh).to(td)
    return q, k, v


def tiny_case(N=64, D=16, grid=(2, 4, 8), d_split=(4, 6, 6), H=1, c_q=4,
              c_sub=(2, 3, 3), dtype="f32", seed=0, **kw) -> tuple:
    """A small custom workload (for edge cases) and its inputs."""
    base = WORKLOADS["tiny"]
    w = base.with_(name=f"custom N={N} D={D}", config_id=100 + seed, H=H, N=N, D=D,
                   grid=grid, d_split=d_split, c_q=c_q, c_sub=c_sub, dtype=dtype,
                   components=kw.pop("components", 4), **kw)
    return w, make_inputs(w, seed=0)
