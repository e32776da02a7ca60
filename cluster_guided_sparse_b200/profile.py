"""Runs SCOPE calls on a synthetic workload, for profilers and quick timing.

    python -m cluster_guided_sparse_b200.profile --workload hunyuan720p --heads 2 [--dense] [--reps 1]

--heads keeps the first H' heads of the workload (a smaller case with the same
per-head shape, e.g. for an ncu capture); every call is a full scope_plan +
scope_attn (and, with --dense, a scope_dense_attn) on those heads.
"""
import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import cluster_guided_sparse_b200 as scope  # noqa: E402
from cluster_guided_sparse_b200 import synth  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="hunyuan720p", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--heads", type=int, default=0)
    ap.add_argument("--reps", type=int, default=1)
    ap.add_argument("--dense", action="store_true")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    heads = list(range(args.heads)) if args.heads else None
    q, k, v = (t.cuda() for t in synth.make_inputs(w, heads=heads))
    params, grid = scope.make_params(w)
    ws = torch.empty(scope.workspace_bytes(q, params, grid), dtype=torch.uint8, device="cuda")
    o = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    for _ in range(args.reps):
        pl = scope.plan(q, k, params, grid, workspace=ws)
        scope.attn(q, k, v, pl, out=o)
        if args.dense:
            scope.dense_attn(q, k, v, params, grid, out=o)
    torch.cuda.synchronize()
    pl.sync_status()
    print("ok", args.workload, tuple(q.shape), "reps", args.reps)


if __name__ == "__main__":
    main()
