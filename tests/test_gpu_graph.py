"""A whole SCOPE call (scope_plan + scope_attn) captured in a CUDA graph and
replayed: the library enqueues everything on the caller's stream, never
allocates and never waits on the host inside a call, so the captured graph
reproduces the eager call bit for bit, and one capture serves new inputs
copied into the same buffers."""
import pytest
import torch

import cluster_guided_sparse_b200 as scope
from cluster_guided_sparse_b200 import synth

pytestmark = pytest.mark.gpu


def test_plan_and_attention_replay_from_a_cuda_graph():
    w = synth.WORKLOADS["small"]
    q, k, v = (t.cuda() for t in synth.make_inputs(w))
    params, grid = scope.make_params(w)
    ws = torch.empty(scope.workspace_bytes(q, params, grid), dtype=torch.uint8, device="cuda")
    o = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    pl = scope.plan(q, k, params, grid, workspace=ws)  # eager call first (one-time kernel set-up)
    scope.attn(q, k, v, pl, out=o)
    torch.cuda.synchronize()
    ref_o, ref_n = o.clone(), pl.view("n").clone()
    tot = int(pl.view("offsets")[-1])
    ref_idx = pl.view("indices")[:tot].clone()

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            gp = scope.plan(q, k, params, grid, workspace=ws)
            scope.attn(q, k, v, gp, out=o)
    torch.cuda.current_stream().wait_stream(side)
    o.zero_()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    gp.sync_status()
    assert torch.equal(o, ref_o)
    assert torch.equal(gp.view("n"), ref_n) and torch.equal(gp.view("indices")[:tot], ref_idx)

    # new inputs in the same buffers: the replay equals an eager call on them
    q2, k2, v2 = (t.cuda() for t in synth.make_inputs(w, seed=1))
    q.copy_(q2), k.copy_(k2), v.copy_(v2)
    g.replay()
    torch.cuda.synchronize()
    o_graph = o.clone()
    ws2 = torch.empty_like(ws)
    pl2 = scope.plan(q, k, params, grid, workspace=ws2)
    o2 = scope.attn(q, k, v, pl2)
    torch.cuda.synchronize()
    assert torch.equal(o_graph, o2)
    del g
