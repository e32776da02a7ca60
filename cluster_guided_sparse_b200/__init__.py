"""B200-native centroid-guided sparse attention (SCOPE formulation).

Thin ctypes binding over libscope.so (include/scope.h): argument marshalling
only.  Every step of the method runs in the library's CUDA kernels; PyTorch
supplies device memory (the workspace and outputs) and the current stream.
There is no CPU fallback: if libscope.so is missing the first call raises.

    plan = scope.plan(q, k, params, grid)      # steps 1-4 (SCOPE abstract)
    o = scope.attn(q, k, v, plan)              # step 5
    o_dense = scope.dense_attn(q, k, v, params, grid)
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libscope.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "scope.h")

SCOPE_F32, SCOPE_BF16, SCOPE_I32, SCOPE_I64 = 0, 1, 2, 3
STATUS = {0: "SCOPE_OK", 1: "SCOPE_EINVAL", 2: "SCOPE_ESHAPE", 3: "SCOPE_EDTYPE", 4: "SCOPE_EALIGN",
          5: "SCOPE_EWORKSPACE", 6: "SCOPE_ECAPACITY", 7: "SCOPE_ECUDA", 8: "SCOPE_ETIMEOUT", 9: "SCOPE_EDEVICE"}
VIEWS = ["qr", "kr", "q_labels", "q_centroids", "q_sizes", "q_perm", "q_start", "k_codes", "k_cent_t",
         "k_cent_h", "k_cent_w", "lut", "r", "kh", "n", "offsets", "indices", "error", "eg_entropy", "eg_pool", "fixup",
         "group_indices", "group_n", "group_masks"]
_TORCH_DT = {SCOPE_F32: torch.float32, SCOPE_BF16: torch.bfloat16, SCOPE_I32: torch.int32, SCOPE_I64: torch.int64}


class ScopeTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("dtype", ctypes.c_int), ("B", ctypes.c_int64), ("H", ctypes.c_int64),
                ("N", ctypes.c_int64), ("D", ctypes.c_int64), ("strides", ctypes.c_int64 * 4)]


class ScopeGrid(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("Hh", ctypes.c_int32), ("W", ctypes.c_int32)]


class ScopeParams(ctypes.Structure):
    _fields_ = [("d_t", ctypes.c_int32), ("d_h", ctypes.c_int32), ("d_w", ctypes.c_int32),
                ("theta", ctypes.c_double), ("c_q", ctypes.c_int32), ("c_t", ctypes.c_int32),
                ("c_h", ctypes.c_int32), ("c_w", ctypes.c_int32), ("iters", ctypes.c_int32),
                ("init_seed", ctypes.c_uint32), ("top_p", ctypes.c_float), ("k_min", ctypes.c_int32),
                ("online_topk", ctypes.c_int32), ("fixed_cluster_size", ctypes.c_int32),
                ("compensate", ctypes.c_int32), ("eg_tau", ctypes.c_float), ("eg_group", ctypes.c_int32),
                ("block_kind", ctypes.c_int32), ("block_t", ctypes.c_int32), ("block_h", ctypes.c_int32),
                ("block_w", ctypes.c_int32)]


class ScopeView(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("dtype", ctypes.c_int), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4)]


class ScopeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """libscope.so, loaded once.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m cluster_guided_sparse_b200.build "
                               "(no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        L.scope_plan_workspace_bytes.argtypes = [P(ScopeTensor), P(ScopeGrid), P(ScopeParams)]
        L.scope_plan_workspace_bytes.restype = ctypes.c_size_t
        L.scope_plan.argtypes = [P(ScopeTensor), P(ScopeTensor), P(ScopeGrid), P(ScopeParams), ctypes.c_void_p,
                                 ctypes.c_size_t, ctypes.c_void_p, P(ctypes.c_void_p)]
        L.scope_attn.argtypes = [P(ScopeTensor), P(ScopeTensor), P(ScopeTensor), ctypes.c_void_p, P(ScopeTensor),
                                 ctypes.c_void_p]
        L.scope_dense_workspace_bytes.argtypes = [P(ScopeTensor), P(ScopeGrid), P(ScopeParams)]
        L.scope_dense_workspace_bytes.restype = ctypes.c_size_t
        L.scope_dense_attn.argtypes = [P(ScopeTensor), P(ScopeTensor), P(ScopeTensor), P(ScopeGrid),
                                       P(ScopeParams), P(ScopeTensor), ctypes.c_void_p, ctypes.c_size_t,
                                       ctypes.c_void_p]
        L.scope_plan_view.argtypes = [ctypes.c_void_p, ctypes.c_int, P(ScopeView)]
        L.scope_sync_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        L.scope_plan_destroy.argtypes = [ctypes.c_void_p]
        L.scope_plan_destroy.restype = None
        L.scope_last_error.restype = ctypes.c_char_p
        L.scope_version.restype = ctypes.c_int
        L.scope_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        for name in ("scope_plan", "scope_attn", "scope_dense_attn", "scope_plan_view", "scope_sync_status",
                     "scope_selftest_wait_timeout"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def header_symbols() -> list:
    """Function names declared in include/scope.h."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(scope_[a-z_]+)\s*\(", text)))


def _check(status: int):
    if status != 0:
        raise ScopeError(status, lib().scope_last_error().decode())


def _stream(stream, device=None) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def as_tensor(x: torch.Tensor) -> ScopeTensor:
    """scope_tensor of a [B, H, N, D] tensor with its element strides (the
    library checks them: last stride 1, 16-byte aligned rows, no overlap)."""
    if x.dim() != 4:
        raise ValueError("expected a [B, H, N, D] tensor")
    dt = {torch.float32: SCOPE_F32, torch.bfloat16: SCOPE_BF16}.get(x.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {x.dtype}")
    B, H, N, D = x.shape
    return ScopeTensor(x.data_ptr(), dt, B, H, N, D, (ctypes.c_int64 * 4)(*x.stride()))


def make_params(w=None, **kw):
    """(ScopeParams, ScopeGrid) from a synth.Workload and/or keyword overrides."""
    f = {}
    if w is not None:
        f = dict(d_t=w.d_split[0], d_h=w.d_split[1], d_w=w.d_split[2], theta=w.theta, c_q=w.c_q,
                 c_t=w.c_sub[0], c_h=w.c_sub[1], c_w=w.c_sub[2], iters=w.iters, init_seed=0, top_p=w.top_p,
                 k_min=w.k_min, online_topk=w.online_topk, fixed_cluster_size=w.fixed_cluster_size,
                 compensate=w.compensate, eg_tau=w.eg_tau, eg_group=w.eg_group, block_kind=w.block_kind,
                 block_t=w.block_dims[0], block_h=w.block_dims[1], block_w=w.block_dims[2])
        grid = tuple(w.grid)
    else:
        grid = (0, 0, 0)
    grid = kw.pop("grid", grid)
    f.update(kw)
    return ScopeParams(**f), ScopeGrid(*grid)


class Plan:
    """Host handle of a plan; its results live in `workspace` (device)."""

    def __init__(self, handle, workspace, q, k):
        self._h = handle
        self.workspace = workspace
        self._q, self._k = q, k

    def view(self, name: str) -> torch.Tensor:
        v = ScopeView()
        _check(lib().scope_plan_view(self._h, VIEWS.index(name), ctypes.byref(v)))
        dt = _TORCH_DT[v.dtype]
        shape = [v.shape[i] for i in range(v.ndim)]
        n = 1
        for s in shape:
            n *= s
        off = v.ptr - self.workspace.data_ptr()
        nbytes = n * torch.empty((), dtype=dt).element_size()
        return self.workspace[off:off + nbytes].view(dt).view(shape)

    def sync_status(self, stream=None):
        _check(lib().scope_sync_status(self._h, _stream(stream)))

    def selftest_wait_timeout(self, cycles: int = 2_000_000, stream=None):
        """Enqueue the library's failure-handling self-test: a bounded wait on a
        barrier nothing completes, which sets this plan's timeout bit (the next
        sync_status raises ScopeError with SCOPE_ETIMEOUT)."""
        _check(lib().scope_selftest_wait_timeout(self._h, int(cycles), _stream(stream)))

    def __del__(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.scope_plan_destroy(self._h)
            self._h = None


def workspace_bytes(q: torch.Tensor, params: ScopeParams, grid: ScopeGrid) -> int:
    n = lib().scope_plan_workspace_bytes(ctypes.byref(as_tensor(q)), ctypes.byref(grid), ctypes.byref(params))
    if n == 0:
        raise ScopeError(1, lib().scope_last_error().decode())
    return n


def plan(q: torch.Tensor, k: torch.Tensor, params: ScopeParams, grid: ScopeGrid, stream=None,
         workspace: Optional[torch.Tensor] = None) -> Plan:
    """Steps 1-4 on the device: returns a Plan whose results stay in `workspace`."""
    tq, tk = as_tensor(q), as_tensor(k)
    need = workspace_bytes(q, params, grid)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    h = ctypes.c_void_p()
    with torch.cuda.device(q.device):
        _check(lib().scope_plan(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(grid), ctypes.byref(params),
                                ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(stream, q.device),
                                ctypes.byref(h)))
    return Plan(h, workspace, q, k)


def attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, p: Plan, out: Optional[torch.Tensor] = None,
         stream=None) -> torch.Tensor:
    """Step 5 on the device: bf16 [B, H, N, D] attention output."""
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    with torch.cuda.device(q.device):
        _check(lib().scope_attn(ctypes.byref(as_tensor(q)), ctypes.byref(as_tensor(k)), ctypes.byref(as_tensor(v)),
                                p._h, ctypes.byref(as_tensor(out)), _stream(stream, q.device)))
    return out


def dense_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, params: ScopeParams, grid: ScopeGrid,
               out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """Dense baseline (RoPE + attention over all keys) on the same device pipeline."""
    tq = as_tensor(q)
    need = lib().scope_dense_workspace_bytes(ctypes.byref(tq), ctypes.byref(grid), ctypes.byref(params))
    if need == 0:
        raise ScopeError(1, lib().scope_last_error().decode())
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    with torch.cuda.device(q.device):
        _check(lib().scope_dense_attn(ctypes.byref(tq), ctypes.byref(as_tensor(k)), ctypes.byref(as_tensor(v)),
                                      ctypes.byref(grid), ctypes.byref(params), ctypes.byref(as_tensor(out)),
                                      ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                      _stream(stream, q.device)))
    return out


def kmeans_noalloc(x: torch.Tensor, dim_off: int, dim_n: int, C: int, iters: int, seed: int = 0,
                   labels: Optional[torch.Tensor] = None, centroids: Optional[torch.Tensor] = None,
                   stream=None):
    """scope_kmeans_noalloc: k-means of columns [dim_off, dim_off+dim_n) of a bf16
    [B, H, N, D] device tensor using the library's fixed scratch (no workspace).
    Returns (labels int32 [B,H,N], centroids f32 [B,H,C,dim_n])."""
    L = lib()
    f = L.scope_kmeans_noalloc
    f.argtypes = [ctypes.POINTER(ScopeTensor), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    if not x.is_cuda or x.dim() != 4 or x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 [B, H, N, D] CUDA tensor")
    B, H, N, _ = x.shape
    if labels is None:
        labels = torch.empty((B, H, N), dtype=torch.int32, device=x.device)
    if centroids is None:
        centroids = torch.empty((B, H, C, dim_n), dtype=torch.float32, device=x.device)
    # the library writes B*H*N labels and B*H*C*dim_n centroids through raw pointers
    for t, dt, shape, name in ((labels, torch.int32, (B, H, N), "labels"),
                               (centroids, torch.float32, (B, H, C, dim_n), "centroids")):
        if t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous() or t.device != x.device:
            raise ValueError(f"{name} must be a contiguous {dt} tensor of shape {shape} on {x.device}")
    with torch.cuda.device(x.device):
        _check(f(ctypes.byref(as_tensor(x)), dim_off, dim_n, C, iters, seed & 0xFFFFFFFF,
                 ctypes.c_void_p(labels.data_ptr()), ctypes.c_void_p(centroids.data_ptr()),
                 _stream(stream, x.device)))
    return labels, centroids
