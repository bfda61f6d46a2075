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
            lib.sdm_version.argtypes = []
            lib.sdm_version.restype = ctypes.c_int
            _lib = lib
    return _lib


def _check(rc: int):
    if rc != 0:
        raise SDMError(rc, load_library().sdm_status_string(rc).decode())


def make_dims(B, H, T, d_qk, d_v, n_sub, k, W, R, in_dtype) -> Dims:
    if isinstance(in_dtype, torch.dtype):
        in_dtype = SDM_DTYPE_BF16 if in_dtype == torch.bfloat16 else SDM_DTYPE_F32
    return Dims(int(B), int(H), int(T), int(d_qk), int(d_v), int(n_sub), int(k), int(W), int(R),
                int(in_dtype))


def workspace_bytes(dims: Dims) -> int:
    return int(load_library().sdm_workspace_bytes(ctypes.byref(dims)))


def _workspace(dims: Dims, device: torch.device, workspace: Optional[torch.Tensor]):
    need = workspace_bytes(dims)
    if need == 0:
        _check(load_library().sdm_forward(*([None] * 9), ctypes.byref(dims), None, 0, None))
    if workspace is not None:
        if workspace.device != device or workspace.numel() * workspace.element_size() < need:
            raise SDMError(4, "workspace too small or on another device")
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


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev, stream):
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    return ctypes.c_void_p(stream.cuda_stream)


def _dims_of(q: torch.Tensor, v: torch.Tensor, C1: torch.Tensor, topk: int, W: int, R: int) -> Dims:
    B, H, T, d_qk = q.shape
    return make_dims(B, H, T, d_qk, v.shape[-1], C1.shape[1], topk, W, R, q.dtype)


PLAN_FIELDS = ("tensor_core_scoring", "survivor_capacity", "block_steps", "streams_per_head",
               "chunk_steps", "chunks", "launches_per_call", "buckets_per_head")


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
    dev = _dev(q, k, v, alpha, beta, C1, C2, M)
    dims = _dims_of(q, v, C1, topk, W, R)
    if o is None:
        o = torch.empty(q.shape[0], q.shape[1], q.shape[2], v.shape[-1], dtype=torch.float32,
                        device=dev)
    _dev(o, q)
    ws = _workspace(dims, dev, workspace)
    lib = load_library()
    if events:
        ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        _check(lib.sdm_forward_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(C1),
                                     _ptr(C2), _ptr(M), _ptr(o), ctypes.byref(dims), _ptr(ws),
                                     ws.numel(), _stream(dev, stream), ev, len(events)))
        return o
    _check(lib.sdm_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(C1), _ptr(C2),
                           _ptr(M), _ptr(o), ctypes.byref(dims), _ptr(ws), ws.numel(),
                           _stream(dev, stream)))
    return o


def select(q, k, C1, C2, *, topk: int, W: int, R: int, d_v: int = 4,
           workspace: Optional[torch.Tensor] = None, stream=None):
    """Selection lists (item 2): returns idx_w [B,H,T,W] int32, w_w float32, idx_r, w_r."""
    dev = _dev(q, k, C1, C2)
    B, H, T, d_qk = q.shape
    dims = make_dims(B, H, T, d_qk, d_v, C1.shape[1], topk, W, R, q.dtype)
    idx_w = torch.empty(B, H, T, W, dtype=torch.int32, device=dev)
    w_w = torch.empty(B, H, T, W, dtype=torch.float32, device=dev)
    idx_r = torch.empty(B, H, T, R, dtype=torch.int32, device=dev)
    w_r = torch.empty(B, H, T, R, dtype=torch.float32, device=dev)
    ws = _workspace(dims, dev, workspace)
    lib = load_library()
    _check(lib.sdm_select(_ptr(q), _ptr(k), _ptr(C1), _ptr(C2), _ptr(idx_w), _ptr(w_w),
                          _ptr(idx_r), _ptr(w_r), ctypes.byref(dims), _ptr(ws), ws.numel(),
                          _stream(dev, stream)))
    return idx_w, w_w, idx_r, w_r


def recur(v, alpha, beta, idx_w, w_w, idx_r, w_r, M, *, d_qk: int, n_sub: int, topk: int,
          o: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
          stream=None) -> torch.Tensor:
    """Recurrence from given lists (items 3-4).  Returns o; M is updated in place."""
    dev = _dev(v, alpha, beta, idx_w, w_w, idx_r, w_r, M)
    B, H, T, d_v = v.shape
    dims = make_dims(B, H, T, d_qk, d_v, n_sub, topk, idx_w.shape[-1], idx_r.shape[-1], v.dtype)
    if o is None:
        o = torch.empty(B, H, T, d_v, dtype=torch.float32, device=dev)
    ws = _workspace(dims, dev, workspace)
    lib = load_library()
    _check(lib.sdm_recur(_ptr(v), _ptr(alpha), _ptr(beta), _ptr(idx_w), _ptr(w_w), _ptr(idx_r),
                         _ptr(w_r), _ptr(M), _ptr(o), ctypes.byref(dims), _ptr(ws), ws.numel(),
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
    _check(load_library().sdm_get_device_status(_ptr(workspace), workspace.numel(),
                                                ctypes.byref(st), ctypes.byref(info),
                                                _stream(workspace.device, stream)))
    return int(st.value), int(info.value)


def probe_random_rows(table: torch.Tensor, *, rmw: bool, rows_in_flight: int, ctas: int,
                      iters: int, stream=None) -> None:
    """Measurement helper (sdm_probe_random_rows): random whole-row gathers
    (rmw=False) or read-modify-writes (rmw=True) of a float32 [nrows, 64] table."""
    dev = _dev(table)
    if table.dtype != torch.float32 or table.dim() != 2 or table.shape[1] != 64 or \
            not table.is_contiguous():
        raise ValueError("table must be a contiguous float32 [nrows, 64] CUDA tensor")
    _check(load_library().sdm_probe_random_rows(_ptr(table), ctypes.c_longlong(table.shape[0]),
                                                int(bool(rmw)), int(rows_in_flight), int(ctas),
                                                int(iters), _stream(dev, stream)))
