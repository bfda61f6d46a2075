"""ctypes wrapper and build step of the C oracle (oracle/sdm_oracle.c).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  The oracle computes in
float64 with a float32 slot table; inputs are passed as float32 arrays holding
the exact input values (bf16 inputs are exactly representable in float32).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE_SRC = os.path.join(_HERE, "sdm_oracle.c")
ORACLE_SO = os.path.join(_HERE, "libsdm_oracle.so")
GDN_SRC = os.path.join(_HERE, "gdn_oracle.c")
GDN_SO = os.path.join(_HERE, "libgdn_oracle.so")

_libs = {}
_lock = threading.Lock()
_CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
           "-msse2", "-mfpmath=sse", "-pthread"]


def compile_source(src: str, so: str) -> str:
    """gcc build with plain IEEE float semantics (no fast-math, no FMA contraction)."""
    tmp = so + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc"] + _CFLAGS + ["-o", tmp, src, "-lm"])
    os.replace(tmp, so)
    return so


def build(force: bool = False) -> str:
    """Compile oracle/sdm_oracle.c into oracle/libsdm_oracle.so and
    oracle/gdn_oracle.c into oracle/libgdn_oracle.so (each if stale)."""
    for src, so in ((GDN_SRC, GDN_SO), (ORACLE_SRC, ORACLE_SO)):
        if (force or not os.path.exists(so)
                or os.path.getmtime(so) < os.path.getmtime(src)):
            compile_source(src, so)
    return ORACLE_SO


def load(so: Optional[str] = None):
    """ctypes handle of the oracle library (the default build, or another .so
    built from a copy of the source, e.g. by the mutation tests)."""
    with _lock:
        if so is None:
            build()
            so = ORACLE_SO
        if so not in _libs:
            lib = ctypes.CDLL(so)
            P = ctypes.c_void_p
            lib.sdm_oracle_forward.argtypes = [P] * 9 + [P, ctypes.c_int, ctypes.c_int] + [P] * 5 + \
                [P, ctypes.c_int, ctypes.c_int]
            lib.sdm_oracle_forward.restype = ctypes.c_int
            lib.sdm_oracle_select.argtypes = [P, P, P, P, ctypes.c_int, P, P, P, P]
            lib.sdm_oracle_select.restype = ctypes.c_int
            if hasattr(lib, "sdm_oracle_forward_decay"):
                lib.sdm_oracle_forward_decay.argtypes = [P] * 8 + [P, ctypes.c_int, ctypes.c_int] + \
                    [P] * 5 + [P, ctypes.c_int, ctypes.c_int]
                lib.sdm_oracle_forward_decay.restype = ctypes.c_int
            _libs[so] = lib
        return _libs[so]


def _f32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dims(d: Dict[str, int]) -> np.ndarray:
    return np.array([d['B'], d['H'], d['T'], d['d_qk'], d['d_v'], d['n_sub'], d['k'], d['W'],
                     d['R']], dtype=np.int32)


def forward(inp: Dict[str, np.ndarray], dims: Dict[str, int], t_begin: int = 0,
            t_end: Optional[int] = None, heads: Optional[Sequence[int]] = None,
            nthreads: int = 1, lists: bool = False, M=None, so: Optional[str] = None
            ) -> Dict[str, np.ndarray]:
    """Run the oracle on full-layout inputs (see sdm_oracle_forward).

    inp: q, k [B,H,T,d_qk]; v [B,H,T,d_v]; alpha, beta [B,H,T]; C1, C2 [H,n,d_h];
    M0 [B,H,N,d_v] (ignored when M is given; M is then updated in place).
    Returns o (and the selection lists + near-tie flags when lists=True) and M.
    """
    lib = load(so)
    T = dims['T']
    t_end = T if t_end is None else t_end
    q, k, v = _f32(inp['q']), _f32(inp['k']), _f32(inp['v'])
    al, be = _f32(inp['alpha']), _f32(inp['beta'])
    C1, C2 = _f32(inp['C1']), _f32(inp['C2'])
    if M is None:
        M = _f32(inp['M0']).copy()
    assert M.dtype == np.float32 and M.flags['C_CONTIGUOUS']
    B, H, dv = dims['B'], dims['H'], dims['d_v']
    o = np.zeros((B, H, T, dv), dtype=np.float32)
    out = {'o': o, 'M': M}
    iw = ww = ir = wr = fl = None
    if lists:
        iw = np.full((B, H, T, dims['W']), -1, dtype=np.int64)
        ww = np.zeros((B, H, T, dims['W']), dtype=np.float64)
        ir = np.full((B, H, T, dims['R']), -1, dtype=np.int64)
        wr = np.zeros((B, H, T, dims['R']), dtype=np.float64)
        fl = np.zeros((B, H, T), dtype=np.uint8)
        out.update(idx_w=iw, w_w=ww, idx_r=ir, w_r=wr, flags=fl)
    hs = None
    nh = 0
    if heads is not None:
        hs = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
        nh = int(hs.size)
    rc = lib.sdm_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(al), _ptr(be), _ptr(C1), _ptr(C2),
                                _ptr(M), _ptr(o), _ptr(_dims(dims)), int(t_begin), int(t_end),
                                _ptr(iw), _ptr(ww), _ptr(ir), _ptr(wr), _ptr(fl), _ptr(hs), nh,
                                int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the dimensions or ran out of memory")
    return out


def forward_decay(inp: Dict[str, np.ndarray], dims: Dict[str, int], t_begin: int = 0,
                  t_end: Optional[int] = None, heads: Optional[Sequence[int]] = None,
                  nthreads: int = 1, lists: bool = False, M=None, so: Optional[str] = None
                  ) -> Dict[str, np.ndarray]:
    """The forward pass with the Raven page's selective-decay write
    (sdm_oracle_forward_decay): inp as for forward with 'a' [B,H,T] (the decay
    rate a_t <= 0) in place of alpha and beta.  w_w holds the normalised
    router weights."""
    lib = load(so)
    T = dims['T']
    t_end = T if t_end is None else t_end
    q, k, v, a = _f32(inp['q']), _f32(inp['k']), _f32(inp['v']), _f32(inp['a'])
    C1, C2 = _f32(inp['C1']), _f32(inp['C2'])
    if M is None:
        M = _f32(inp['M0']).copy()
    B, H, dv = dims['B'], dims['H'], dims['d_v']
    o = np.zeros((B, H, T, dv), dtype=np.float32)
    out = {'o': o, 'M': M}
    iw = ww = ir = wr = fl = None
    if lists:
        iw = np.full((B, H, T, dims['W']), -1, dtype=np.int64)
        ww = np.zeros((B, H, T, dims['W']), dtype=np.float64)
        ir = np.full((B, H, T, dims['R']), -1, dtype=np.int64)
        wr = np.zeros((B, H, T, dims['R']), dtype=np.float64)
        fl = np.zeros((B, H, T), dtype=np.uint8)
        out.update(idx_w=iw, w_w=ww, idx_r=ir, w_r=wr, flags=fl)
    hs = None
    nh = 0
    if heads is not None:
        hs = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
        nh = int(hs.size)
    rc = lib.sdm_oracle_forward_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(C1), _ptr(C2),
                                      _ptr(M), _ptr(o), _ptr(_dims(dims)), int(t_begin),
                                      int(t_end), _ptr(iw), _ptr(ww), _ptr(ir), _ptr(wr), _ptr(fl),
                                      _ptr(hs), nh, int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the dimensions or ran out of memory")
    return out


def forward_head(h_inp: Dict[str, np.ndarray], dims: Dict[str, int], t_begin: int = 0,
                 t_end: Optional[int] = None, lists: bool = False, M=None,
                 so: Optional[str] = None):
    """One head given as per-head arrays (q [T,d_qk], C1 [n,d_h], M0 [N,d_v], ...)."""
    d = dict(dims)
    d['B'] = 1
    d['H'] = 1
    d['T'] = int(np.asarray(h_inp['q'].shape)[0])
    full = {}
    for name in ('q', 'k', 'v', 'alpha', 'beta'):
        full[name] = _f32(h_inp[name])[None, None]
    for name in ('C1', 'C2'):
        full[name] = _f32(h_inp[name])[None]
    if M is None:
        M = _f32(h_inp['M0']).copy()
    M4 = M.reshape((1, 1) + M.shape)
    out = forward(full, d, t_begin=t_begin, t_end=t_end, lists=lists, M=M4, so=so)
    res = {}
    for name, val in out.items():
        res[name] = val[0, 0] if name != 'M' else M
    return res


def select(x, C1, C2, dims: Dict[str, int], n_sel: int, so: Optional[str] = None):
    """Selection of one projected vector x [d_qk] against one head's codebooks.
    Returns (slots int64 [n_sel] in rank order, weights float64, scores float32, flag)."""
    lib = load(so)
    x, C1, C2 = _f32(x), _f32(C1), _f32(C2)
    slots = np.zeros(n_sel, dtype=np.int64)
    w = np.zeros(n_sel, dtype=np.float64)
    s = np.zeros(n_sel, dtype=np.float32)
    flag = ctypes.c_int(0)
    rc = lib.sdm_oracle_select(_ptr(x), _ptr(C1), _ptr(C2), _ptr(_dims(dims)), int(n_sel),
                               _ptr(slots), _ptr(w), _ptr(s), ctypes.byref(flag))
    if rc != 0:
        raise ValueError("oracle rejected the dimensions")
    return slots, w, s, flag.value


# ---------------------------------------------------------------- dense GDN
def load_gdn(so: Optional[str] = None):
    """ctypes handle of the GDN oracle (the default build, or another .so)."""
    with _lock:
        if so is None:
            so = GDN_SO
            if (not os.path.exists(so)) or os.path.getmtime(so) < os.path.getmtime(GDN_SRC):
                compile_source(GDN_SRC, so)
        if so not in _libs:
            lib = ctypes.CDLL(so)
            P = ctypes.c_void_p
            lib.gdn_oracle_forward.argtypes = [P] * 7 + [P, ctypes.c_int, ctypes.c_int,
                                                         ctypes.c_int]
            lib.gdn_oracle_forward.restype = ctypes.c_int
            _libs[so] = lib
        return _libs[so]


def gdn_forward(inp: Dict[str, np.ndarray], dims: Dict[str, int], t_begin: int = 0,
                t_end: Optional[int] = None, nthreads: int = 1, S=None,
                so: Optional[str] = None) -> Dict[str, np.ndarray]:
    """The dense GDN oracle (gdn_oracle_forward).  inp: q, k [B,H,T,d_k];
    v [B,H,T,d_v]; alpha, beta [B,H,T]; S0 [B,H,d_v,d_k] (ignored when S is
    given; S is then updated in place).  dims: B, H, T, d_k, d_v.
    Returns o [B,H,T,d_v] and S."""
    lib = load_gdn(so)
    T = dims['T']
    t_end = T if t_end is None else t_end
    q, k, v = _f32(inp['q']), _f32(inp['k']), _f32(inp['v'])
    al, be = _f32(inp['alpha']), _f32(inp['beta'])
    if S is None:
        S = _f32(inp['S0']).copy()
    assert S.dtype == np.float32 and S.flags['C_CONTIGUOUS']
    o = np.zeros((dims['B'], dims['H'], T, dims['d_v']), dtype=np.float32)
    d = np.array([dims['B'], dims['H'], T, dims['d_k'], dims['d_v']], dtype=np.int32)
    rc = lib.gdn_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(al), _ptr(be), _ptr(S), _ptr(o),
                                _ptr(d), int(t_begin), int(t_end), int(nthreads))
    if rc != 0:
        raise ValueError("GDN oracle rejected the dimensions or ran out of memory")
    return {'o': o, 'S': S}
