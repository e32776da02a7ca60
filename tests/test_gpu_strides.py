"""Strided tensors through the C ABI: a call on any accepted layout of the
same values gives exactly the results of the contiguous call.

Every stage after RoPE reads the plan's own contiguous post-RoPE copies, and
the caller's rows are read and written in place, so the plan and the output
must agree bit for bit.  Slicing heads (every second head of a tensor) is the
layout a head-sharded caller hands the library; heads are independent in the
SCOPE formulation (per-head clustering, per-head Top-k), so a plan of a head
slice equals the same heads of the full plan."""
import pytest
import torch

import cluster_guided_sparse_b200 as scope
from cluster_guided_sparse_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"

PLAN_VIEWS = ("qr", "kr", "q_labels", "q_centroids", "q_sizes", "k_codes", "k_cent_t", "k_cent_h", "k_cent_w",
              "lut", "r", "kh", "n")


def bhnd_memory(t):
    """The same values held in [B, N, H, D] memory, seen as [B, H, N, D]."""
    return t.transpose(1, 2).contiguous().transpose(1, 2)


def lists(pl):
    tot = int(pl.view("offsets")[-1])
    return pl.view("offsets"), pl.view("indices")[:tot]


@pytest.mark.parametrize("name", ["tiny", "small"])  # f32 and bf16 inputs
def test_bnhd_layout_equals_contiguous(name):
    w = synth.WORKLOADS[name]
    qd, kd, vd = (t.to(DEV) for t in synth.make_inputs(w))
    params, grid = scope.make_params(w)
    pl = scope.plan(qd, kd, params, grid)
    o = scope.attn(qd, kd, vd, pl)
    qs, ks, vs = (bhnd_memory(t) for t in (qd, kd, vd))
    assert not qs.is_contiguous()
    pl2 = scope.plan(qs, ks, params, grid)
    o2 = torch.full((w.B, w.N, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV).transpose(1, 2)
    scope.attn(qs, ks, vs, pl2, out=o2)
    torch.cuda.synchronize()
    pl2.sync_status()
    for v in PLAN_VIEWS:
        assert torch.equal(pl.view(v), pl2.view(v)), v
    a, b = lists(pl), lists(pl2)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert torch.equal(o, o2)


def test_head_slice_equals_heads_of_full_plan():
    w = synth.WORKLOADS["small"]
    qd, kd, vd = (t.to(DEV) for t in synth.make_inputs(w))
    params, grid = scope.make_params(w)
    pl = scope.plan(qd, kd, params, grid)
    o = scope.attn(qd, kd, vd, pl)
    for r, world in ((0, 2), (1, 2), (2, 3)):
        qs, ks, vs = (t[:, r::world] for t in (qd, kd, vd))
        pls = scope.plan(qs, ks, params, grid)
        os_ = scope.attn(qs, ks, vs, pls)
        torch.cuda.synchronize()
        pls.sync_status()
        heads = list(range(r, w.H, world))
        for v in ("q_labels", "q_centroids", "lut", "r", "kh", "n"):
            assert torch.equal(pls.view(v)[0], pl.view(v)[0, heads]), v
        assert torch.equal(pls.view("k_codes")[:, 0], pl.view("k_codes")[:, 0, heads])
        assert torch.equal(os_, o[:, heads])
        off, idx = pl.view("offsets"), pl.view("indices")
        offs, idxs = pls.view("offsets"), pls.view("indices")
        for i, h in enumerate(heads):
            a0, a1 = int(off[h * w.c_q]), int(off[(h + 1) * w.c_q])
            b0, b1 = int(offs[i * w.c_q]), int(offs[(i + 1) * w.c_q])
            assert torch.equal(idx[a0:a1], idxs[b0:b1]), h
