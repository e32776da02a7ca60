"""scope_kmeans_noalloc: clustering for callers that cannot allocate device
memory (its scratch is a fixed array inside libscope.so), checked through the
C ABI against the same clustering inside scope_plan.  Two calls run back to
back, so the second one starts from the first one's leftover scratch."""
import ctypes

import pytest
import torch

import cluster_guided_sparse_b200 as scope
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
        # same kernels on the same rows: labels identical, centroids within the
        # update tolerance of the parity tests (1e-5 of the centroid norm)
        assert torch.equal(lab, ref_q_lab)
        assert torch.equal(klab, ref_h_lab)
        tol = 1e-5 * ref_q_cent.norm(dim=-1).clamp_min(1e-3)
        assert ((cent - ref_q_cent).norm(dim=-1) <= tol).all()
        tol = 1e-5 * ref_h_cent.norm(dim=-1).clamp_min(1e-3)
        assert ((kcent - ref_h_cent).norm(dim=-1) <= tol).all()


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
