"""EG-Sparse routing and pooled selection on the GPU against the oracle
("EG-Sparse", abstract; reading R17 in the oracle).

Stage-fed like the other parity tests: the oracle takes the device's own
lookup tables and key codes, forms the proxy scores exactly as the device
does (fp32 (t + h) + w), and computes the head entropies, the routing and
the pooled Top-p counts in fp64.  Entropies must agree to 1e-5; routing
exactly (thresholds are placed away from every entropy); pooled counts
exactly, or as a near-tie (the pool's kept mass fraction at both the device's
and the oracle's counts within 1e-5 relative of p); K_h, n_c and the lists
exactly given the device's counts."""
import numpy as np
import pytest
import torch

import cluster_guided_sparse_b200 as scope
import oracle
import parity as P
from cluster_guided_sparse_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _lists(pl, w, h):
    off = pl.view("offsets").cpu().numpy()
    n = pl.view("n").cpu().numpy()
    idx = pl.view("indices")
    return lambda c: idx[int(off[h * w.c_q + c]):int(off[h * w.c_q + c]) + int(n[0, h, c])].cpu().numpy()


def _scores(pl, w, h):
    lut = pl.view("lut")[0, h].cpu().numpy()
    codes = [pl.view("k_codes")[s, 0, h].cpu().numpy() for s in range(3)]
    return np.stack([P.scores_f32(lut[c], codes, w.c_sub) for c in range(w.c_q)]), lut, codes


def _pool_mass(scores, sizes, counts, scale):
    """Kept mass fraction of a pool for per-row prefix counts (fp64)."""
    num = sum(float(sizes[i, c]) * oracle.prefix_mass(scores[i][c], int(counts[i, c]), scale)
              for i in range(len(scores)) for c in range(scores[0].shape[0]) if sizes[i, c] > 0)
    return num / float(sizes[sizes > 0].sum())


@pytest.mark.parametrize("group,sigma", [(4, (0.3, 0.3)), (3, (0.1, 1.0)), (8, (0.1, 1.0))])
def test_eg_routing_and_pooled_selection(group, sigma):
    w = synth.WORKLOADS["small"].with_(k_min=0, sigma=sigma, config_id=210 + group)
    q, k, v = synth.make_inputs(w)
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    N, D = w.N, w.D
    scale = 1.0 / np.sqrt(D)
    p32 = float(np.float32(w.top_p))
    # entropies first (a threshold that routes no head), then a threshold between two of them
    probe = scope.plan(qd, kd, *scope.make_params(w.with_(eg_tau=1e-9, eg_group=group)))
    ent = probe.view("eg_entropy")[0].cpu().numpy()
    srt = np.sort(ent)
    i = int(np.argmax(np.diff(srt[1:-1]))) + 1  # the widest gap inside the spread
    tau = float((srt[i] + srt[i + 1]) / 2)
    wq = w.with_(eg_tau=tau, eg_group=group)
    pl = scope.plan(qd, kd, *scope.make_params(wq))
    o = scope.attn(qd, kd, vd, pl)
    torch.cuda.synchronize()
    pl.sync_status()
    ent = pl.view("eg_entropy")[0].cpu().numpy()
    pool = pl.view("eg_pool")[0].cpu().numpy()
    sizes = pl.view("q_sizes")[0].cpu().numpy().astype(np.int64)
    r = pl.view("r")[0].cpu().numpy()
    sc = {}
    for h in range(w.H):
        sc[h] = _scores(pl, wq, h)
        e_orc = oracle.head_entropy(sc[h][0], sizes[h], scale)
        assert abs(ent[h] - e_orc) <= 1e-5, (h, ent[h], e_orc)
    routed = [h for h in range(w.H) if ent[h] < tau]
    assert 0 < len(routed) < w.H
    assert (pool == np.array([h // group if h in routed else -1 for h in range(w.H)])).all()
    pools = oracle.eg_route(list(ent), tau, group)
    tc = P.TieCounter()
    for members in pools:
        if not members:
            continue
        scores = [sc[h][0] for h in members]
        sz = np.stack([sizes[h] for h in members])
        counts, _ = oracle.pooled_topp(np.stack(scores), sz, p32, scale, with_mass=True)
        dev = np.stack([r[h] for h in members]).astype(np.int64)
        tc.checked += 1
        if not (dev == counts).all():
            f_dev, f_orc = _pool_mass(scores, sz, dev, scale), _pool_mass(scores, sz, counts, scale)
            assert abs(f_dev - p32) <= P.TIE_REL * p32 and abs(f_orc - p32) <= P.TIE_REL * p32, \
                f"pool {members}: counts differ beyond a near-tie (mass {f_dev:.9f} vs {f_orc:.9f})"
            tc.ties += 1
    # every head: K_h, n_c and the lists given the device's counts; un-routed
    # heads also their own per-row Top-p counts
    tcs = P.TieCounter()
    for h in range(w.H):
        scores, lut, codes = sc[h]
        clusters = range(w.c_q) if h not in routed else []
        P.check_selection(lut, codes, sizes[h], r[h], pl.view("kh")[0, h].item(), pl.view("n")[0, h].cpu().numpy(),
                          _lists(pl, wq, h), wq, N, D, clusters, tcs)
        get = _lists(pl, wq, h)
        for c in range(w.c_q):  # lists of routed heads too (check_selection only checked un-routed clusters)
            if h in routed:
                ref = oracle.emit(scores[c], int(pl.view("n")[0, h, c]))
                assert (get(c) == ref).all(), (h, c)
    tcs.assert_ok("per-row counts")
    # attention over the pooled lists, sampled rows of a routed head
    h = routed[0]
    qr, kr = P.np64(pl.view("qr")[0, h]), P.np64(pl.view("kr")[0, h])
    rows = np.sort(np.random.default_rng(7).choice(N, 48, replace=False))
    P.check_attention(qr, kr, v[0, h].double().numpy(), pl.view("q_labels")[0, h].cpu().numpy(), _lists(pl, wq, h),
                      P.np64(o[0, h]), rows)


def test_eg_off_and_all_routed():
    w = synth.WORKLOADS["small"]
    qd, kd, _ = (t.to(DEV) for t in synth.make_inputs(w))
    base = scope.plan(qd, kd, *scope.make_params(w))
    tiny = scope.plan(qd, kd, *scope.make_params(w.with_(eg_tau=1e-9, eg_group=2)))  # routes no head
    allr = scope.plan(qd, kd, *scope.make_params(w.with_(eg_tau=1.5, eg_group=8)))  # one pool of every head
    torch.cuda.synchronize()
    for v in ("r", "n", "kh", "offsets"):
        assert torch.equal(base.view(v), tiny.view(v)), v
    assert (allr.view("eg_pool") == 0).all()
    with pytest.raises(scope.ScopeError):
        base.view("eg_entropy")  # no routing in a plain plan


def test_eg_pools_are_per_batch_entry():
    """B = 2: each batch entry routes and pools its own heads; batch entry 1's
    entropies, pools and pooled counts against the oracle."""
    group = 4
    w = synth.WORKLOADS["small"].with_(B=2, k_min=0, sigma=(0.1, 1.0), config_id=219)
    q, k, v = synth.make_inputs(w)
    qd, kd = q.to(DEV), k.to(DEV)
    scale = 1.0 / np.sqrt(w.D)
    p32 = float(np.float32(w.top_p))
    probe = scope.plan(qd, kd, *scope.make_params(w.with_(eg_tau=1e-9, eg_group=group)))
    srt = np.sort(probe.view("eg_entropy")[1].cpu().numpy())
    i = int(np.argmax(np.diff(srt[1:-1]))) + 1
    tau = float((srt[i] + srt[i + 1]) / 2)
    wq = w.with_(eg_tau=tau, eg_group=group)
    pl = scope.plan(qd, kd, *scope.make_params(wq))
    torch.cuda.synchronize()
    pl.sync_status()
    b = 1
    ent = pl.view("eg_entropy")[b].cpu().numpy()
    pool = pl.view("eg_pool")[b].cpu().numpy()
    sizes = pl.view("q_sizes")[b].cpu().numpy().astype(np.int64)
    r = pl.view("r")[b].cpu().numpy()
    scores = {}
    for h in range(w.H):
        lut = pl.view("lut")[b, h].cpu().numpy()
        codes = [pl.view("k_codes")[s, b, h].cpu().numpy() for s in range(3)]
        scores[h] = np.stack([P.scores_f32(lut[c], codes, w.c_sub) for c in range(w.c_q)])
        assert abs(ent[h] - oracle.head_entropy(scores[h], sizes[h], scale)) <= 1e-5, h
    routed = [h for h in range(w.H) if ent[h] < tau]
    ngroups = (w.H + group - 1) // group  # pool ids are global: batch entry b owns b*ngroups ..
    assert (pool == np.array([b * ngroups + h // group if h in routed else -1 for h in range(w.H)])).all()
    for members in oracle.eg_route(list(ent), tau, group):
        if not members:
            continue
        counts = oracle.pooled_topp(np.stack([scores[h] for h in members]), np.stack([sizes[h] for h in members]),
                                    p32, scale)
        dev = np.stack([r[h] for h in members]).astype(np.int64)
        if not (dev == counts).all():
            f = [_pool_mass([scores[h] for h in members], np.stack([sizes[h] for h in members]), x, scale)
                 for x in (dev, counts)]
            assert all(abs(x - p32) <= P.TIE_REL * p32 for x in f), f"pool {members}: beyond a near-tie"
