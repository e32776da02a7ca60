"""VMoBA block-granular selection on the GPU against the oracle ("VMoBA:
Mixture-of-Block Attention for Video Diffusion Models", abstract items (1)
and (3); reading R18 in the oracle).

Stage-fed: block ids exactly; block means within 1e-6 of the fp64 means of
the device's own rotated keys; the lookup table within 1e-6 of the fp64
dots of the device's query centroids and block means; kept key counts equal
to the oracle's threshold selection over the device's fp32 block scores
(whole blocks, ties kept) or a near-tie; lists exactly the kept blocks'
keys; attention within the usual tolerance."""
import numpy as np
import pytest
import torch

import cluster_guided_sparse_b200 as scope
import oracle
import parity as P
from cluster_guided_sparse_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("kind,dims", [(1, (4, 4, 4)), (2, (1, 4, 8)), (3, (2, 4, 8)), (3, (3, 5, 7))])
def test_block_selection_parity(kind, dims):
    w = synth.WORKLOADS["small"].with_(block_kind=kind, block_dims=dims, k_min=0, online_topk=0,
                                       config_id=230 + kind)
    q, k, v = synth.make_inputs(w)
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    pl = scope.plan(qd, kd, *scope.make_params(w))
    o = scope.attn(qd, kd, vd, pl)
    torch.cuda.synchronize()
    pl.sync_status()
    N, D = w.N, w.D
    scale = 1.0 / np.sqrt(D)
    p32 = float(np.float32(w.top_p))
    ids, nb = oracle.block_ids(w.grid, kind, dims)
    bsizes = np.bincount(ids, minlength=nb).astype(np.int64)
    off = pl.view("offsets").cpu().numpy()
    idx = pl.view("indices")
    ties = 0
    for h in range(w.H):
        codes = pl.view("k_codes")[:, 0, h].cpu().numpy()
        assert (codes[0] == ids).all() and (codes[1] == 0).all() and (codes[2] == 0).all()
        kr = P.np64(pl.view("kr")[0, h])
        kbar = P.np64(pl.view("k_cent_t")[0, h])
        ref = oracle.block_means(kr, ids, nb)
        assert np.abs(kbar - ref).max() <= 1e-6 * max(1.0, np.abs(ref).max())
        qcent = P.np64(pl.view("q_centroids")[0, h])
        lut = pl.view("lut")[0, h].cpu().numpy()
        P.check_lut(qcent, [kbar, np.zeros((1, 0)), np.zeros((1, 0))], (D, 0, 0), lut.astype(np.float64))
        n = pl.view("n")[0, h].cpu().numpy()
        r = pl.view("r")[0, h].cpu().numpy()
        sizes = pl.view("q_sizes")[0, h].cpu().numpy()
        assert (n == np.where(sizes > 0, r, 0)).all()  # no k_min, no online Top-k in block mode
        for c in range(w.c_q):
            s = lut[c, :nb].astype(np.float64)  # (L[b] + 0) + 0 in fp32 is L[b]
            keep, m = oracle.block_select(s, bsizes, p32, scale)
            if m != int(r[c]):
                # a near-tie: the kept weight fractions at both counts lie within 1e-5 of p
                order = oracle.order(s)
                wgt = bsizes[order] * np.exp((s[order] - s.max()) * scale)
                cum = np.cumsum(wgt) / wgt.sum()
                keys = np.cumsum(bsizes[order])
                f = [cum[np.searchsorted(keys, x)] for x in (m, int(r[c]))]
                assert all(abs(x - p32) <= P.TIE_REL * p32 for x in f), (h, c, m, int(r[c]))
                ties += 1
                continue
            if sizes[c] == 0:
                continue
            got = idx[int(off[h * w.c_q + c]):int(off[h * w.c_q + c]) + int(n[c])].cpu().numpy()
            assert (got == np.nonzero(keep[ids])[0]).all(), (h, c)
        rows = np.arange(0, N, 37)
        get = lambda c: idx[int(off[h * w.c_q + c]):int(off[h * w.c_q + c]) + int(n[c])].cpu().numpy()
        P.check_attention(P.np64(pl.view("qr")[0, h]), kr, v[0, h].double().numpy(),
                          pl.view("q_labels")[0, h].cpu().numpy(), get, P.np64(o[0, h]), rows)
    assert ties <= 2


def test_block_mode_argument_rules():
    w = synth.WORKLOADS["small"].with_(block_kind=3, block_dims=(2, 4, 8), k_min=0, online_topk=0)
    qd, kd, _ = (t.to(DEV) for t in synth.make_inputs(w, heads=[0]))
    for bad in (dict(k_min=4), dict(online_topk=1), dict(block_kind=4), dict(block_t=0), dict(eg_tau=0.5, eg_group=2)):
        with pytest.raises(scope.ScopeError):
            scope.plan(qd, kd, *scope.make_params(w.with_(H=1), **bad))
    with pytest.raises(scope.ScopeError):
        scope.plan(qd, kd, *scope.make_params(w.with_(H=1), grid=(0, 0, 0)))


def test_block_selection_second_batch_entry():
    """B = 2: batch entry 1's block means, kept blocks and lists against the oracle."""
    kind, dims = 3, (2, 4, 8)
    w = synth.WORKLOADS["small"].with_(B=2, block_kind=kind, block_dims=dims, k_min=0, online_topk=0,
                                       config_id=239)
    q, k, v = synth.make_inputs(w)
    qd, kd = q.to(DEV), k.to(DEV)
    pl = scope.plan(qd, kd, *scope.make_params(w))
    torch.cuda.synchronize()
    pl.sync_status()
    b, D = 1, w.D
    scale = 1.0 / np.sqrt(D)
    p32 = float(np.float32(w.top_p))
    ids, nb = oracle.block_ids(w.grid, kind, dims)
    bsizes = np.bincount(ids, minlength=nb).astype(np.int64)
    off = pl.view("offsets").cpu().numpy()
    idx = pl.view("indices")
    ties = 0
    for h in range(w.H):
        assert (pl.view("k_codes")[0, b, h].cpu().numpy() == ids).all()
        kbar = P.np64(pl.view("k_cent_t")[b, h])
        ref = oracle.block_means(P.np64(pl.view("kr")[b, h]), ids, nb)
        assert np.abs(kbar - ref).max() <= 1e-6 * max(1.0, np.abs(ref).max())
        lut = pl.view("lut")[b, h].cpu().numpy()
        n = pl.view("n")[b, h].cpu().numpy()
        sizes = pl.view("q_sizes")[b, h].cpu().numpy()
        for c in range(w.c_q):
            if sizes[c] == 0:
                continue
            keep, m = oracle.block_select(lut[c, :nb].astype(np.float64), bsizes, p32, scale)
            if m != int(n[c]):
                ties += 1
                continue
            i0 = int(off[(b * w.H + h) * w.c_q + c])
            assert (idx[i0:i0 + int(n[c])].cpu().numpy() == np.nonzero(keep[ids])[0]).all(), (h, c)
    assert ties <= 2
