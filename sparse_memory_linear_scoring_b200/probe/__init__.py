"""Benchmark helper: the HBM ceiling of random whole-row gathers and
read-modify-writes (libsdm_probe.so, built beside libsdm.so; not part of the
SDM C ABI)."""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(os.path.dirname(_HERE), "libsdm_probe.so")
_lib = None
_lock = threading.Lock()


def load_library():
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("libsdm_probe.so not found at %s; build it with "
                                   "`python -m sparse_memory_linear_scoring_b200.build`" % LIB_PATH)
            lib = ctypes.CDLL(LIB_PATH)
            lib.sdm_probe_random_rows.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_void_p]
            lib.sdm_probe_random_rows.restype = ctypes.c_int
            _lib = lib
    return _lib


def probe_random_rows(table: torch.Tensor, *, rmw: bool, rows_in_flight: int, ctas: int,
                      iters: int, stream=None) -> None:
    """Random whole-row gathers (rmw=False) or read-modify-writes (rmw=True) of a
    contiguous float32 [nrows, 64] CUDA table (sdm_probe_random_rows)."""
    if not table.is_cuda or table.dtype != torch.float32 or table.dim() != 2 or \
            table.shape[1] != 64 or not table.is_contiguous():
        raise ValueError("table must be a contiguous float32 [nrows, 64] CUDA tensor")
    if stream is None:
        stream = torch.cuda.current_stream(table.device)
    rc = load_library().sdm_probe_random_rows(
        ctypes.c_void_p(table.data_ptr()), ctypes.c_longlong(table.shape[0]), int(bool(rmw)),
        int(rows_in_flight), int(ctas), int(iters), ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise ValueError("sdm_probe_random_rows failed with code %d" % rc)
