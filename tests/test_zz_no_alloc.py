"""scope_kmeans_noalloc: clustering for callers that cannot allocate device
memory (its scratch is a fixed array inside libscope.so), checked through the
C ABI against the same clustering inside scope_plan and, at 512 clusters,
against the fp64 oracle on the device's own centroids.  Calls run back to
back, so each starts from the previous call's leftover scratch."""
import ctypes

import numpy as np
import pytest
import torch

import cluster_guided_sparse_b200 as scope
import parity as P
from cluster_guided_sparse_b200 import synth

pytestmark = pytest.mark.gpu


def test_noalloc_kmeans_matches_plan_twice():
    w = synth.WORKLOADS["small"]
    q, k, _ = (t.cuda() for t in synth.make_inputs(w))
    params, grid = scope.make_params(w)
    pl = scope.plan(q, k, params, grid)
    torch.cuda.synchronize()
    qr, kr = pl.view("qr").clone(), pl.view("kr").clone()
    ref_q_lab, ref_q_cent = pl.view("q_labels").clone(), pl.view("q_centroids").clone()
    ref_h_lab, ref_h_cent = pl.view("k_codes")[1].clone(), pl.view("k_cent_h").clone()
    d_t, d_h, _ = w.d_split
    for _call in range(2):
        lab = torch.full_like(ref_q_lab, -1)
        cent = torch.full_like(ref_q_cent, float("nan"))
        scope.kmeans_noalloc(qr, 0, w.D, w.c_q, w.iters, 0, lab, cent)
        klab = torch.full_like(ref_h_lab, -1)
        kcent = torch.full_like(ref_h_cent, float("nan"))
        scope.kmeans_noalloc(kr, d_t, d_h, w.c_sub[1], w.iters, 0, klab, kcent)
        torch.cuda.synchronize()
        # queries: the same kernels and per-head fixed-point scale as the plan's
        # (32 clusters, direct form): identical results
        assert torch.equal(lab, ref_q_lab)
        assert torch.equal(cent, ref_q_cent)
        # key subspace h: the plan decides labels exactly on the tensor cores,
        # this entry point by the fp32 direct form; they may differ only on rows
        # whose two nearest centroids are within fp32 rounding (near-ties), and
        # when they agree everywhere the centroids agree too
        if torch.equal(klab, ref_h_lab):
            assert torch.equal(kcent, ref_h_cent)
        else:
            tc = P.TieCounter()
            for h in range(w.H):
                x = P.np64(kr[0, h, :, d_t:d_t + d_h])
                P.check_assign(x, P.np64(kcent[0, h]), klab[0, h].cpu().numpy(), tc, f"noalloc keys h{h}")
            tc.assert_ok("noalloc keys")


def test_noalloc_kmeans_512_clusters_against_oracle():
    """Query clustering of one 720p-shaped head (N = 118 800, 512 clusters):
    init, two Lloyd rounds, stage-fed.  Labels equal the fp64 argmin on the
    call's own centroids except near-ties; every update equals the fp64 mean
    of the previous round's labels; round 0 agrees with the plan's exact
    tensor-core assignment except near-ties."""
    w = synth.WORKLOADS["hunyuan720p"]
    q, k, _ = (t.cuda() for t in synth.make_inputs(w, heads=[0]))
    params, grid = scope.make_params(w, iters=0)
    pl = scope.plan(q, k, params, grid)
    torch.cuda.synchronize()
    qr = pl.view("qr").clone()
    x = P.np64(qr[0, 0])
    rows = np.sort(np.random.default_rng(3).choice(w.N, 4000, replace=False))
    tc = P.TieCounter()
    out = {}
    for it in (0, 1, 2):
        lab = torch.full((1, 1, w.N), -1, dtype=torch.int32, device="cuda")
        cent = torch.full((1, 1, w.c_q, w.D), float("nan"), device="cuda")
        scope.kmeans_noalloc(qr, 0, w.D, w.c_q, it, 0, lab, cent)
        torch.cuda.synchronize()
        out[it] = (lab[0, 0].cpu().numpy(), P.np64(cent[0, 0]))
        if it == 0:
            np.testing.assert_array_equal(out[0][1], x[np.arange(w.c_q) * (w.N // w.c_q)])  # strided init
            plan_lab = pl.view("q_labels")[0, 0].cpu().numpy()
            P.check_assign(x, out[0][1], plan_lab, P.TieCounter(), "plan round 0")
        P.check_assign(x[rows], out[it][1], out[it][0][rows], tc, f"noalloc round {it}")
        if it > 0:
            P.check_update(x, out[it - 1][0], out[it - 1][1], out[it][1], f"noalloc update {it}")
    tc.assert_ok("noalloc assign")
    # and the labels of round 0 differ from the plan's only on near-ties
    mism = np.nonzero(out[0][0] != pl.view("q_labels")[0, 0].cpu().numpy())[0]
    assert len(mism) <= P.TIE_FRAC * w.N


def test_noalloc_rejects_shapes_beyond_its_scratch():
    L = scope.lib()
    L.scope_kmeans_noalloc_scratch_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32]
    L.scope_kmeans_noalloc_scratch_bytes.restype = ctypes.c_size_t
    assert L.scope_kmeans_noalloc_scratch_bytes(1, 24, 118800, 512) <= (32 << 20)  # one 720p layer fits
    assert L.scope_kmeans_noalloc_scratch_bytes(2, 24, 118800, 512) > (32 << 20)
    # the size check runs before any device access: a fake, aligned pointer is never touched
    x = scope.ScopeTensor(0x7F0000000000, scope.SCOPE_BF16, 2, 24, 118800, 128)
    f = L.scope_kmeans_noalloc
    f.argtypes = [ctypes.POINTER(scope.ScopeTensor), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    st = f(ctypes.byref(x), 0, 128, 512, 10, 0, ctypes.c_void_p(0x7F0000000000), ctypes.c_void_p(0x7F0000000000),
           None)
    assert st == 6 and "SCRATCH" in L.scope_last_error().decode()


def test_noalloc_binding_rejects_wrong_buffers():
    x = torch.zeros((1, 2, 256, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        scope.kmeans_noalloc(x, 0, 64, 8, 1, labels=torch.zeros((1, 2, 255), dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError):
        scope.kmeans_noalloc(x, 0, 64, 8, 1, centroids=torch.zeros((1, 2, 8, 64), dtype=torch.float64,
                                                                     device="cuda"))
    with pytest.raises(ValueError):
        scope.kmeans_noalloc(x.float(), 0, 64, 8, 1)
