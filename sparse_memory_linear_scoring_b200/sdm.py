"""ctypes binding of libsdm.so (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Dict, Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdm.so")

SDM_DTYPE_F32 = 0
SDM_DTYPE_BF16 = 1


class SDMError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("sdm error %d: %s" % (code, what))
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "T", "d_qk", "d_v", "n_sub", "k", "W", "R", "in_dtype")]

    def as_dict(self) -> Dict[str, int]:
        return {n: int(getattr(self, n)) for n, _ in self._fields_}


class GdnDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "T", "d_k", "d_v", "in_dtype")]


_lib = None
_lock = threading.Lock()
_ws_cache: Dict[Tuple[int, int], torch.Tensor] = {}


def load_library():
    """Load libsdm.so from the package directory (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("libsdm.so not found at %s; build it with "
                                   "`python -m sparse_memory_linear_scoring_b200.build`" % LIB_PATH)
            lib = ctypes.CDLL(LIB_PATH)
            P, S = ctypes.c_void_p, ctypes.c_size_t
            DP = ctypes.POINTER(Dims)
            lib.sdm_workspace_bytes.argtypes = [DP]
            lib.sdm_workspace_bytes.restype = S
            lib.sdm_forward.argtypes = [P] * 9 + [DP, P, S, P]
            lib.sdm_forward.restype = ctypes.c_int
            lib.sdm_select.argtypes = [P] * 8 + [DP, P, S, P]
            lib.sdm_select.restype = ctypes.c_int
            lib.sdm_recur.argtypes = [P] * 9 + [DP, P, S, P]
            lib.sdm_recur.restype = ctypes.c_int
            lib.sdm_get_device_status.argtypes = [P, S, ctypes.POINTER(ctypes.c_int32),
                                                  ctypes.POINTER(ctypes.c_int32), P]
            lib.sdm_get_device_status.restype = ctypes.c_int
            lib.sdm_status_string.argtypes = [ctypes.c_int]
            lib.sdm_status_string.restype = ctypes.c_char_p
            lib.sdm_forward_timed.argtypes = [P] * 9 + [DP, P, S, P, P, ctypes.c_int]
            lib.sdm_forward_timed.restype = ctypes.c_int
            lib.sdm_query_plan.argtypes = [DP, P, ctypes.c_int]
            lib.sdm_query_plan.restype = ctypes.c_int
            lib.sdm_gdn_workspace_bytes.argtypes = [ctypes.POINTER(GdnDims)]
            lib.sdm_gdn_workspace_bytes.restype = S
            lib.sdm_gdn_forward.argtypes = [P] * 7 + [ctypes.POINTER(GdnDims), P, S, P]
            lib.sdm_gdn_forward.restype = ctypes.c_int
            lib.sdm_forward_decay.argtypes = [P] * 8 + [DP, P, S, P]
            lib.sdm_forward_decay.restype = ctypes.c_int
            lib.sdm_backward_workspace_bytes.argtypes = [DP]
            lib.sdm_backward_workspace_bytes.restype = S
            lib.sdm_backward.argtypes = [P] * 22 + [DP, P, S, P]
            lib.sdm_backward.restype = ctypes.c_int
            lib.sdm_step.argtypes = [P] * 13 + [DP, P]
            lib.sdm_step.restype = ctypes.c_int
            lib.sdm_version.argtypes = []
            lib.sdm_version.restype = ctypes.c_int
            _lib = lib
    return _lib


def _check(rc: int):
    if rc != 0:
        raise SDMError(rc, load_library().sdm_status_string(rc).decode())


_IN_DTYPES = {torch.float32: SDM_DTYPE_F32, torch.bfloat16: SDM_DTYPE_BF16}


def make_dims(B, H, T, d_qk, d_v, n_sub, k, W, R, in_dtype) -> Dims:
    """Problem sizes; in_dtype is SDM_DTYPE_F32 / SDM_DTYPE_BF16 or the torch dtype
    (float32 or bfloat16 only) of q', k', v, C1 and C2."""
    if isinstance(in_dtype, torch.dtype):
        if in_dtype not in _IN_DTYPES:
            raise TypeError("input dtype must be torch.float32 or torch.bfloat16, not %s"
                            % in_dtype)
        in_dtype = _IN_DTYPES[in_dtype]
    return Dims(int(B), int(H), int(T), int(d_qk), int(d_v), int(n_sub), int(k), int(W), int(R),
                int(in_dtype))


def workspace_bytes(dims: Dims) -> int:
    return int(load_library().sdm_workspace_bytes(ctypes.byref(dims)))


def _workspace(dims: Dims, device: torch.device, workspace: Optional[torch.Tensor]):
    need = workspace_bytes(dims)
    if need == 0:
        _check(load_library().sdm_forward(*([None] * 9), ctypes.byref(dims), None, 0, None))
    if workspace is not None:
        if workspace.device != device or _nbytes(workspace) < need:
            raise SDMError(4, "workspace too small or on another device")
        if not workspace.is_contiguous():
            raise ValueError("workspace must be contiguous")
        return workspace
    key = (device.index if device.index is not None else torch.cuda.current_device(), need)
    with _lock:
        ws = _ws_cache.get(key)
        if ws is None:
            for k_old in [k for k in _ws_cache if k[0] == key[0]]:
                del _ws_cache[k_old]
            ws = torch.empty(need, dtype=torch.uint8, device=device)
            _ws_cache[key] = ws
    return ws


def _dev(*ts) -> torch.device:
    dev = ts[0].device
    for t in ts:
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (there is no CPU path)")
        if t.device != dev:
            raise ValueError("all tensors must be on one device")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
    return dev


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _expect(t: torch.Tensor, name: str, shape, dtypes) -> None:
    """Raise before any launch unless `t` has exactly `shape` and one of `dtypes`."""
    if tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if t.dtype not in dtypes:
        raise TypeError("%s has dtype %s, expected %s" % (name, t.dtype,
                                                           " or ".join(map(str, dtypes))))


def _check_inputs(q, k, v, C1, C2, alpha=None, beta=None):
    """Shapes and dtypes of the projected inputs; returns (B, H, T, d_qk, n_sub, dtype)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, T, d_qk], got shape %s" % (tuple(q.shape),))
    B, H, T, d_qk = q.shape
    if q.dtype not in _IN_DTYPES:
        raise TypeError("q has dtype %s, expected torch.float32 or torch.bfloat16" % q.dtype)
    if d_qk % 2:
        raise ValueError("d_qk = %d must be even" % d_qk)
    if C1.dim() != 3:
        raise ValueError("C1 must be [H, n_sub, d_qk/2], got shape %s" % (tuple(C1.shape),))
    n_sub = C1.shape[1]
    _expect(k, "k", (B, H, T, d_qk), (q.dtype,))
    _expect(C1, "C1", (H, n_sub, d_qk // 2), (q.dtype,))
    _expect(C2, "C2", (H, n_sub, d_qk // 2), (q.dtype,))
    if v is not None:
        if v.dim() != 4:
            raise ValueError("v must be [B, H, T, d_v], got shape %s" % (tuple(v.shape),))
        _expect(v, "v", (B, H, T, v.shape[-1]), (q.dtype,))
    for name, t in (("alpha", alpha), ("beta", beta)):
        if t is not None:
            _expect(t, name, (B, H, T), (torch.float32,))
    return B, H, T, d_qk, n_sub, q.dtype


def _no_alias(outs, ins) -> None:
    """Outputs must not overlap each other or any input (raise before any launch)."""
    def span(t):
        return t.data_ptr(), t.data_ptr() + _nbytes(t)
    for i, (no, o) in enumerate(outs):
        if o.numel() == 0:
            continue
        a0, a1 = span(o)
        for nt, t in list(outs[i + 1:]) + list(ins):
            if t is None or t.numel() == 0:
                continue
            b0, b1 = span(t)
            if a0 < b1 and b0 < a1:
                raise ValueError("%s overlaps %s; outputs must not alias other tensors" % (no, nt))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev, stream):
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    return ctypes.c_void_p(stream.cuda_stream)


PLAN_FIELDS = ("tensor_core_scoring", "survivor_capacity", "block_steps", "streams_per_head",
               "chunk_steps", "chunks", "launches_per_call", "buckets_per_head", "scoring_mode")


def query_plan(dims: Dims) -> Dict[str, int]:
    """How the library runs `dims` (sdm_query_plan)."""
    out = (ctypes.c_int64 * len(PLAN_FIELDS))()
    _check(load_library().sdm_query_plan(ctypes.byref(dims), out, len(PLAN_FIELDS)))
    return {n: int(v) for n, v in zip(PLAN_FIELDS, out)}


def forward(q, k, v, alpha, beta, C1, C2, M, *, topk: int, W: int, R: int,
            o: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            stream=None, events=None) -> torch.Tensor:
    """SDM forward pass.  q, k [B,H,T,d_qk]; v [B,H,T,d_v]; alpha, beta [B,H,T] float32;
    C1, C2 [H,n_sub,d_qk/2]; M [B,H,n_sub^2,d_v] float32, updated in place to M_T.
    q, k, v, C1, C2 share one dtype (float32 or bfloat16).  Returns o [B,H,T,d_v] float32.
    events: optional list of torch.cuda.Event recorded at the kernel-phase
    boundaries (see sdm_forward_timed in include/sdm.h)."""
    B, H, T, d_qk, n_sub, dt = _check_inputs(q, k, v, C1, C2, alpha, beta)
    d_v = v.shape[-1]
    _expect(M, "M", (B, H, n_sub * n_sub, d_v), (torch.float32,))
    if o is not None:
        _expect(o, "o", (B, H, T, d_v), (torch.float32,))
    dev = _dev(q, k, v, alpha, beta, C1, C2, M, *([o] if o is not None else []))
    dims = make_dims(B, H, T, d_qk, d_v, n_sub, topk, W, R, dt)
    if o is None:
        o = torch.empty(B, H, T, d_v, dtype=torch.float32, device=dev)
    _no_alias([("M", M), ("o", o)], [("q", q), ("k", k), ("v", v), ("alpha", alpha),
                                     ("beta", beta), ("C1", C1), ("C2", C2)])
    ws = _workspace(dims, dev, workspace)
    lib = load_library()
    if events:
        ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        _check(lib.sdm_forward_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(C1),
                                     _ptr(C2), _ptr(M), _ptr(o), ctypes.byref(dims), _ptr(ws),
                                     _nbytes(ws), _stream(dev, stream), ev, len(events)))
        return o
    _check(lib.sdm_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(C1), _ptr(C2),
                           _ptr(M), _ptr(o), ctypes.byref(dims), _ptr(ws), _nbytes(ws),
                           _stream(dev, stream)))
    return o


def forward_decay(q, k, v, a, C1, C2, M, *, topk: int, W: int, R: int,
                  o: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """SDM with the Raven page's selective-decay write (sdm_forward_decay): a
    [B,H,T] float32 decay rates (<= 0) in place of alpha and beta; otherwise as
    forward.  Returns o; M is updated in place."""
    B, H, T, d_qk, n_sub, dt = _check_inputs(q, k, v, C1, C2, a, None)
    d_v = v.shape[-1]
    _expect(M, "M", (B, H, n_sub * n_sub, d_v), (torch.float32,))
    if o is not None:
        _expect(o, "o", (B, H, T, d_v), (torch.float32,))
    dev = _dev(q, k, v, a, C1, C2, M, *([o] if o is not None else []))
    dims = make_dims(B, H, T, d_qk, d_v, n_sub, topk, W, R, dt)
    if o is None:
        o = torch.empty(B, H, T, d_v, dtype=torch.float32, device=dev)
    _no_alias([("M", M), ("o", o)], [("q", q), ("k", k), ("v", v), ("a", a), ("C1", C1),
                                     ("C2", C2)])
    ws = _workspace(dims, dev, workspace)
    _check(load_library().sdm_forward_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(C1),
                                            _ptr(C2), _ptr(M), _ptr(o), ctypes.byref(dims),
                                            _ptr(ws), _nbytes(ws), _stream(dev, stream)))
    return o


def step(q, k, v, alpha, beta, C1, C2, M, *, topk: int, W: int, R: int,
         o: Optional[torch.Tensor] = None, lists: bool = False, stream=None):
    """Short calls (decoding) through the fused single-step kernel (sdm_step):
    same arguments and layouts as forward (T steps, typically 1), no workspace.
    Returns o, or (o, idx_w, w_w, idx_r, w_r) with lists=True."""
    B, H, T, d_qk, n_sub, dt = _check_inputs(q, k, v, C1, C2, alpha, beta)
    d_v = v.shape[-1]
    _expect(M, "M", (B, H, n_sub * n_sub, d_v), (torch.float32,))
    if o is not None:
        _expect(o, "o", (B, H, T, d_v), (torch.float32,))
    dev = _dev(q, k, v, alpha, beta, C1, C2, M, *([o] if o is not None else []))
    dims = make_dims(B, H, T, d_qk, d_v, n_sub, topk, W, R, dt)
    if o is None:
        o = torch.empty(B, H, T, d_v, dtype=torch.float32, device=dev)
    outs = [("M", M), ("o", o)]
    lw = [None] * 4
    if lists:
        lw = [torch.empty(B, H, T, W, dtype=torch.int32, device=dev),
              torch.empty(B, H, T, W, dtype=torch.float32, device=dev),
              torch.empty(B, H, T, R, dtype=torch.int32, device=dev),
              torch.empty(B, H, T, R, dtype=torch.float32, device=dev)]
    _no_alias(outs, [("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                     ("C1", C1), ("C2", C2)])
    _check(load_library().sdm_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(C1),
                                   _ptr(C2), _ptr(M), _ptr(o), *[_ptr(x) for x in lw],
                                   ctypes.byref(dims), _stream(dev, stream)))
    return (o, *lw) if lists else o


def backward(q, k, v, alpha, beta, C1, C2, M0, idx_w, w_w, idx_r, w_r, d_o, dM_T=None, *,
             topk: int, workspace: Optional[torch.Tensor] = None, stream=None,
             dM_T_inplace: bool = False):
    """Gradients of the forward pass at its selections (sdm_backward).  M0 is the
    table the forward started from; the lists are sdm_select's; d_o = dL/do,
    dM_T = dL/dM_T (None: 0).  Returns a dict of float32 gradients: q, k, v,
    alpha, beta, C1, C2, M0.  With dM_T_inplace, dL/dM_0 is accumulated in dM_T
    itself (returned as "M0"), which saves copying it."""
    B, H, T, d_qk, n_sub, dt = _check_inputs(q, k, v, C1, C2, alpha, beta)
    d_v = v.shape[-1]
    W, R = idx_w.shape[-1], idx_r.shape[-1]
    N = n_sub * n_sub
    _expect(M0, "M0", (B, H, N, d_v), (torch.float32,))
    _expect(idx_w, "idx_w", (B, H, T, W), (torch.int32,))
    _expect(w_w, "w_w", (B, H, T, W), (torch.float32,))
    _expect(idx_r, "idx_r", (B, H, T, R), (torch.int32,))
    _expect(w_r, "w_r", (B, H, T, R), (torch.float32,))
    _expect(d_o, "d_o", (B, H, T, d_v), (torch.float32,))
    if dM_T is not None:
        _expect(dM_T, "dM_T", (B, H, N, d_v), (torch.float32,))
    dev = _dev(q, k, v, alpha, beta, C1, C2, M0, idx_w, w_w, idx_r, w_r, d_o,
               *([dM_T] if dM_T is not None else []))
    dims = make_dims(B, H, T, d_qk, d_v, n_sub, topk, W, R, dt)
    f32 = dict(dtype=torch.float32, device=dev)
    g = dict(q=torch.empty(B, H, T, d_qk, **f32), k=torch.empty(B, H, T, d_qk, **f32),
             v=torch.empty(B, H, T, d_v, **f32), alpha=torch.empty(B, H, T, **f32),
             beta=torch.empty(B, H, T, **f32), C1=torch.empty(H, n_sub, d_qk // 2, **f32),
             C2=torch.empty(H, n_sub, d_qk // 2, **f32),
             M0=dM_T if (dM_T_inplace and dM_T is not None) else torch.empty(B, H, N, d_v, **f32))
    if dM_T_inplace and (dM_T is None or not dM_T.is_contiguous()):
        raise ValueError("dM_T_inplace needs a contiguous dM_T")
    lib = load_library()
    need = int(lib.sdm_backward_workspace_bytes(ctypes.byref(dims)))
    if need == 0:
        _check(lib.sdm_backward(*([None] * 22), ctypes.byref(dims), None, 0, None))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    elif workspace.device != dev or _nbytes(workspace) < need or not workspace.is_contiguous():
        raise SDMError(4, "workspace too small, not contiguous or on another device")
    _check(lib.sdm_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(C1),
                            _ptr(C2), _ptr(M0), _ptr(idx_w), _ptr(w_w), _ptr(idx_r), _ptr(w_r),
                            _ptr(d_o), _ptr(dM_T), _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]),
                            _ptr(g["alpha"]), _ptr(g["beta"]), _ptr(g["C1"]), _ptr(g["C2"]),
                            _ptr(g["M0"]), ctypes.byref(dims), _ptr(workspace),
                            _nbytes(workspace), _stream(dev, stream)))
    return g


def gdn_forward(q, k, v, alpha, beta, S, *, o: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Dense Gated DeltaNet baseline (sdm_gdn_forward).  q, k [B,H,T,d_k];
    v [B,H,T,d_v] (one dtype, float32 or bfloat16); alpha, beta [B,H,T] float32;
    S [B,H,d_v,d_k] float32, updated in place to S_T.  Returns o [B,H,T,d_v]."""
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q must be [B, H, T, d_k] and v [B, H, T, d_v]")
    B, H, T, d_k = q.shape
    d_v = v.shape[-1]
    if q.dtype not in _IN_DTYPES:
        raise TypeError("q has dtype %s, expected torch.float32 or torch.bfloat16" % q.dtype)
    _expect(k, "k", (B, H, T, d_k), (q.dtype,))
    _expect(v, "v", (B, H, T, d_v), (q.dtype,))
    _expect(alpha, "alpha", (B, H, T), (torch.float32,))
    _expect(beta, "beta", (B, H, T), (torch.float32,))
    _expect(S, "S", (B, H, d_v, d_k), (torch.float32,))
    if o is not None:
        _expect(o, "o", (B, H, T, d_v), (torch.float32,))
    dev = _dev(q, k, v, alpha, beta, S, *([o] if o is not None else []))
    dims = GdnDims(int(B), int(H), int(T), int(d_k), int(d_v), _IN_DTYPES[q.dtype])
    if o is None:
        o = torch.empty(B, H, T, d_v, dtype=torch.float32, device=dev)
    _no_alias([("S", S), ("o", o)], [("q", q), ("k", k), ("v", v), ("alpha", alpha),
                                     ("beta", beta)])
    lib = load_library()
    need = int(lib.sdm_gdn_workspace_bytes(ctypes.byref(dims)))
    if need == 0:
        _check(lib.sdm_gdn_forward(*([None] * 7), ctypes.byref(dims), None, 0, None))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    elif workspace.device != dev or _nbytes(workspace) < need or not workspace.is_contiguous():
        raise SDMError(4, "workspace too small, not contiguous or on another device")
    _check(lib.sdm_gdn_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S),
                               _ptr(o), ctypes.byref(dims), _ptr(workspace), _nbytes(workspace),
                               _stream(dev, stream)))
    return o


def gdn_workspace_bytes(B, H, T, d_k, d_v, in_dtype) -> int:
    dt = _IN_DTYPES[in_dtype] if isinstance(in_dtype, torch.dtype) else int(in_dtype)
    dims = GdnDims(int(B), int(H), int(T), int(d_k), int(d_v), dt)
    return int(load_library().sdm_gdn_workspace_bytes(ctypes.byref(dims)))


def select(q, k, C1, C2, *, topk: int, W: int, R: int, d_v: int = 4,
           workspace: Optional[torch.Tensor] = None, stream=None):
    """Selection lists (item 2): returns idx_w [B,H,T,W] int32, w_w float32, idx_r, w_r."""
    B, H, T, d_qk, n_sub, dt = _check_inputs(q, k, None, C1, C2)
    dev = _dev(q, k, C1, C2)
    dims = make_dims(B, H, T, d_qk, d_v, n_sub, topk, W, R, dt)
    idx_w = torch.empty(B, H, T, W, dtype=torch.int32, device=dev)
    w_w = torch.empty(B, H, T, W, dtype=torch.float32, device=dev)
    idx_r = torch.empty(B, H, T, R, dtype=torch.int32, device=dev)
    w_r = torch.empty(B, H, T, R, dtype=torch.float32, device=dev)
    ws = _workspace(dims, dev, workspace)
    lib = load_library()
    _check(lib.sdm_select(_ptr(q), _ptr(k), _ptr(C1), _ptr(C2), _ptr(idx_w), _ptr(w_w),
                          _ptr(idx_r), _ptr(w_r), ctypes.byref(dims), _ptr(ws), _nbytes(ws),
                          _stream(dev, stream)))
    return idx_w, w_w, idx_r, w_r


def recur(v, alpha, beta, idx_w, w_w, idx_r, w_r, M, *, d_qk: int, n_sub: int, topk: int,
          o: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
          stream=None) -> torch.Tensor:
    """Recurrence from given lists (items 3-4).  Returns o; M is updated in place."""
    if v.dim() != 4 or idx_w.dim() != 4 or idx_r.dim() != 4:
        raise ValueError("v, idx_w and idx_r must be 4-D ([B, H, T, d_v], [B, H, T, W], "
                         "[B, H, T, R])")
    B, H, T, d_v = v.shape
    W, R = idx_w.shape[-1], idx_r.shape[-1]
    if v.dtype not in _IN_DTYPES:
        raise TypeError("v has dtype %s, expected torch.float32 or torch.bfloat16" % v.dtype)
    _expect(alpha, "alpha", (B, H, T), (torch.float32,))
    _expect(beta, "beta", (B, H, T), (torch.float32,))
    _expect(idx_w, "idx_w", (B, H, T, W), (torch.int32,))
    _expect(w_w, "w_w", (B, H, T, W), (torch.float32,))
    _expect(idx_r, "idx_r", (B, H, T, R), (torch.int32,))
    _expect(w_r, "w_r", (B, H, T, R), (torch.float32,))
    _expect(M, "M", (B, H, int(n_sub) * int(n_sub), d_v), (torch.float32,))
    if o is not None:
        _expect(o, "o", (B, H, T, d_v), (torch.float32,))
    dev = _dev(v, alpha, beta, idx_w, w_w, idx_r, w_r, M, *([o] if o is not None else []))
    dims = make_dims(B, H, T, d_qk, d_v, n_sub, topk, W, R, v.dtype)
    if o is None:
        o = torch.empty(B, H, T, d_v, dtype=torch.float32, device=dev)
    _no_alias([("M", M), ("o", o)], [("v", v), ("alpha", alpha), ("beta", beta),
                                     ("idx_w", idx_w), ("w_w", w_w), ("idx_r", idx_r),
                                     ("w_r", w_r)])
    ws = _workspace(dims, dev, workspace)
    lib = load_library()
    _check(lib.sdm_recur(_ptr(v), _ptr(alpha), _ptr(beta), _ptr(idx_w), _ptr(w_w), _ptr(idx_r),
                         _ptr(w_r), _ptr(M), _ptr(o), ctypes.byref(dims), _ptr(ws), _nbytes(ws),
                         _stream(dev, stream)))
    return o


def device_status(workspace: Optional[torch.Tensor] = None, stream=None) -> Tuple[int, int]:
    """(SDM_DEV_* flags, first offending index) of the last call on `workspace`
    (default: the cached workspace of the current device)."""
    if workspace is None:
        dev = torch.cuda.current_device()
        cands = [w for (d, _), w in _ws_cache.items() if d == dev]
        if not cands:
            return 0, -1
        workspace = cands[-1]
    st = ctypes.c_int32(0)
    info = ctypes.c_int32(0)
    _check(load_library().sdm_get_device_status(_ptr(workspace), _nbytes(workspace),
                                                ctypes.byref(st), ctypes.byref(info),
                                                _stream(workspace.device, stream)))
    return int(st.value), int(info.value)
