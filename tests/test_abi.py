"""Host-only checks of the C ABI: the library loads, exports every symbol
include/scope.h declares, and rejects bad arguments before any device work.

The pointers used here are fake, 16-byte aligned addresses: every call below
must fail in argument validation, which runs before any CUDA call."""
import ctypes
import os
import re

import pytest

import cluster_guided_sparse_b200 as scope
from cluster_guided_sparse_b200 import build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FAKE = 0x7F0000000000  # aligned, never dereferenced


@pytest.fixture(scope="module")
def L():
    build.build()
    return scope.lib()


def T(N=256, D=64, dtype=scope.SCOPE_BF16, ptr=FAKE, B=1, H=2):
    return scope.ScopeTensor(ptr, dtype, B, H, N, D)


def P(**kw):
    return scope.make_params(synth.WORKLOADS["tiny"], **kw)


def plan_status(L, q, k, params, grid, ws=FAKE, ws_bytes=1 << 40):
    h = ctypes.c_void_p()
    st = L.scope_plan(ctypes.byref(q), ctypes.byref(k), ctypes.byref(grid), ctypes.byref(params),
                      ctypes.c_void_p(ws), ws_bytes, None, ctypes.byref(h))
    return st, L.scope_last_error().decode()


def test_exports_every_declared_symbol(L):
    names = scope.header_symbols()
    assert "scope_plan" in names and "scope_attn" in names
    for n in names:
        assert hasattr(L, n), n
    assert L.scope_version() >= 1


def test_workspace_bytes_counts_list_capacity(L):
    p, g = P()
    q = T()
    n = L.scope_plan_workspace_bytes(ctypes.byref(q), ctypes.byref(g), ctypes.byref(p))
    # worst-case lists (c_q * N per head), post-RoPE copies, and more
    assert n >= 2 * 8 * 256 * 4 + 2 * 2 * 256 * 64 * 2
    q2 = T(H=4)
    assert L.scope_plan_workspace_bytes(ctypes.byref(q2), ctypes.byref(g), ctypes.byref(p)) > n


@pytest.mark.parametrize("mut,code,msg", [
    (dict(top_p=0.0), 1, "top_p"),
    (dict(top_p=1.5), 1, "top_p"),
    (dict(k_min=-1), 1, "k_min"),
    (dict(d_t=15, d_h=25), 2, "even"),
    (dict(d_t=16, d_h=24, d_w=26), 2, "equal D"),
    (dict(c_q=0), 1, "c_q"),
    (dict(c_q=257), 1, "c_q"),
    (dict(c_t=300), 1, "c_t"),
    (dict(grid=(4, 8, 7)), 2, "grid"),
    (dict(grid=(4, 0, 64)), 2, "grid"),
    (dict(iters=-1), 1, "iters"),
    (dict(online_topk=2), 1, "online_topk"),
    (dict(fixed_cluster_size=64), 1, "grid"),
    (dict(compensate=2), 1, "compensate"),
    (dict(compensate=1), 1, "compensate"),
    (dict(eg_tau=0.5, eg_group=0), 1, "eg_group"),
    (dict(eg_tau=-0.1), 1, "eg_tau"),
    (dict(block_kind=5), 1, "block_kind"),
    (dict(block_kind=3, block_t=2, block_h=4, block_w=8), 1, "k_min"),
    (dict(block_kind=3, block_t=0, block_h=4, block_w=8, k_min=0, online_topk=0), 1, "block_t"),
])
def test_bad_params_rejected_on_host(L, mut, code, msg):
    p, g = P(**mut)
    st, err = plan_status(L, T(), T(), p, g)
    assert st == code and msg in err, (st, err)
    assert L.scope_plan_workspace_bytes(ctypes.byref(T()), ctypes.byref(g), ctypes.byref(p)) == 0


def test_bad_tensors_rejected_on_host(L):
    p, g = P()
    assert plan_status(L, T(ptr=FAKE + 8), T(), p, g)[0] == 4  # misaligned
    assert plan_status(L, T(ptr=0), T(), p, g)[0] == 1  # null
    assert plan_status(L, T(D=96), T(D=96), p, g)[0] == 2  # head dim
    assert plan_status(L, T(), T(N=128), p, g)[0] == 2  # shape mismatch
    assert plan_status(L, T(), T(dtype=scope.SCOPE_F32), p, g)[0] == 3  # dtype mismatch
    assert plan_status(L, T(dtype=7), T(dtype=7), p, g)[0] == 3


def test_workspace_checks_on_host(L):
    p, g = P()
    assert plan_status(L, T(), T(), p, g, ws=0)[0] == 5
    assert plan_status(L, T(), T(), p, g, ws=FAKE + 16)[0] == 4
    st, err = plan_status(L, T(), T(), p, g, ws_bytes=1024)
    assert st == 5 and "too small" in err


def test_fixed_cluster_size_shape_rules(L):
    q = T(N=65536 - 64, D=64)  # 1023 clusters of 64: not a power of two
    p, g = scope.make_params(synth.WORKLOADS["unstructured"])
    assert plan_status(L, q, q, p, g)[0] == 2
    p2, g2 = scope.make_params(synth.WORKLOADS["unstructured"], d_t=32, d_h=32)
    assert plan_status(L, T(N=65536), T(N=65536), p2, g2)[0] == 2


def test_attn_and_views_reject_null_plan(L):
    q = T()
    assert L.scope_attn(ctypes.byref(q), ctypes.byref(q), ctypes.byref(q), None, ctypes.byref(q), None) == 1
    v = scope.ScopeView()
    assert L.scope_plan_view(None, 0, ctypes.byref(v)) == 1
    assert L.scope_sync_status(None, None) == 1
    L.scope_plan_destroy(None)  # freeing a null handle is a no-op


def test_dense_rejects_bad_grid(L):
    p, g = P(grid=(4, 8, 9))
    q = T()
    o = T()
    st = L.scope_dense_attn(ctypes.byref(q), ctypes.byref(q), ctypes.byref(q), ctypes.byref(g), ctypes.byref(p),
                            ctypes.byref(o), ctypes.c_void_p(FAKE), 1 << 40, None)
    assert st == 2
    f = T(dtype=scope.SCOPE_F32)
    p, g = P()
    st = L.scope_dense_attn(ctypes.byref(q), ctypes.byref(q), ctypes.byref(q), ctypes.byref(g), ctypes.byref(p),
                            ctypes.byref(f), ctypes.c_void_p(FAKE), 1 << 40, None)
    assert st == 3  # output must be bf16


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(scope, "_lib", None)
    monkeypatch.setattr(scope, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        scope.lib()


def test_compensation_workspace_holds_cluster_means_and_virtual_lists(L):
    # ClusterAttention shape: N = 4096, 64-token clusters -> 64 key clusters, D = 64; leaves
    # of 64 queries are grouped four to a work item (16 groups per head)
    w = synth.WORKLOADS["unstructured"].with_(N=4096, D=64, H=2, d_split=(64, 0, 0), c_q=64, c_sub=(64, 1, 1))
    q = T(N=4096, D=64, H=2)
    sizes = []
    for comp in (0, 1):
        p, g = scope.make_params(w, compensate=comp)
        sizes.append(L.scope_plan_workspace_bytes(ctypes.byref(q), ctypes.byref(g), ctypes.byref(p)))
    BH, C, D, groups, leaves, tiles = 2, 64, 64, 2 * 16, 4, 1
    tables = 4 * BH * C * D * 2                    # mean keys and values, bf16 hi + lo
    lists = groups * tiles * 64 * 4                # virtual key clusters
    bias = groups * tiles * leaves * 64 * 4        # per-leaf logit offsets
    assert sizes[0] > 0 and sizes[1] >= sizes[0] + tables + lists + bias


def test_view_names_match_the_header():
    hdr = open(os.path.join(ROOT, "include", "scope.h")).read()
    ids = dict((m.group(1).lower(), int(m.group(2))) for m in re.finditer(r"SCOPE_VIEW_(\w+)\s*=\s*(\d+)", hdr))
    count = ids.pop("count")
    assert len(scope.VIEWS) == count
    assert {name: i for i, name in enumerate(scope.VIEWS)} == ids


def S(strides, N=256, D=64, H=2, B=1, dtype=scope.SCOPE_BF16):
    return scope.ScopeTensor(FAKE, dtype, B, H, N, D, (ctypes.c_int64 * 4)(*strides))


def test_strided_layouts_checked_on_host(L):
    p, g = P()
    N, D, H = 256, 64, 2
    ws_of = lambda t: L.scope_plan_workspace_bytes(ctypes.byref(t), ctypes.byref(g), ctypes.byref(p))
    contiguous = ws_of(T())
    # accepted: explicit contiguous strides, [B, N, H, D] memory, every second head of a 4-head tensor
    for st in ((H * N * D, N * D, D, 1), (N * H * D, D, H * D, 1), (4 * N * D, 2 * N * D, D, 1)):
        assert ws_of(S(st)) == contiguous, st
    # rejected before any device work: D not contiguous, misaligned row starts, rows that overlap
    for st, msg in (((H * N * D, N * D, D, 2), "strides[3]"), ((H * N * D, N * D, 68, 1), "16 bytes"),
                    ((H * N * D, N * D, 32, 1), "overlap"), ((N * D, 0, D, 1), "overlap"),
                    ((H * N * D, -N * D, D, 1), ">= 0")):
        q = S(st)
        assert plan_status(L, q, q, p, g)[0] == 2, st
        assert msg in L.scope_last_error().decode(), (st, L.scope_last_error())
    # f32 rows need 16-byte alignment too: a stride of 4 floats is fine, 2 is not
    p32 = S((H * N * 68, N * 68, 68, 1), dtype=scope.SCOPE_F32)
    assert ws_of(p32) == ws_of(T(dtype=scope.SCOPE_F32))
    bad = S((H * N * 66, N * 66, 66, 1), dtype=scope.SCOPE_F32)
    assert plan_status(L, bad, bad, p, g)[0] == 2


def test_selftest_wait_timeout_checks_arguments(L):
    L.scope_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    assert L.scope_selftest_wait_timeout(None, 2_000_000, None) == 1
    # the cycle limit is checked before the plan is touched (fake handle)
    assert L.scope_selftest_wait_timeout(ctypes.c_void_p(FAKE), 10, None) == 1
    assert "wait_cycles" in L.scope_last_error().decode()
    assert L.scope_selftest_wait_timeout(ctypes.c_void_p(FAKE), 5_000_000_000, None) == 1


def test_block_mode_block_count_limit(L):
    p, g = P(block_kind=1, block_t=1, block_h=1, block_w=1, k_min=0, online_topk=0, grid=(64, 64, 64))
    q = T(N=64 * 64 * 64, H=1)
    st, err = plan_status(L, q, q, p, g)
    assert st == 1 and "blocks >" in err  # 262 144 one-token blocks > 16 384
    p, g = P(block_kind=3, block_t=4, block_h=4, block_w=4, k_min=0, online_topk=0, grid=(64, 64, 64))
    assert L.scope_plan_workspace_bytes(ctypes.byref(q), ctypes.byref(g), ctypes.byref(p)) > 0  # 4096 blocks
