"""The C-ABI library loads, exports every symbol include/sdm.h declares, and
rejects bad arguments on the host, before anything reaches a GPU (these tests
make no compute call and need no GPU)."""
import ctypes
import os
import re

import pytest

import sparse_memory_linear_scoring_b200 as sdm
from sparse_memory_linear_scoring_b200 import build as sdm_build
from synth import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdm.h")

OK, ERR_NULL, ERR_DIMS, ERR_ALIGN, ERR_WS, ERR_UNSUP = 0, 1, 2, 3, 4, 5


@pytest.fixture(scope="module")
def lib():
    sdm_build.build()
    return sdm.load_library()


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"SDM_API[^;(]*?\b(sdm_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 7, names
    for name in names:
        assert hasattr(lib, name), name
    assert lib.sdm_version() >= 100


def test_status_strings(lib):
    for code in range(0, 9):
        assert lib.sdm_status_string(code)


@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: c.name)
def test_workspace_for_every_workload(lib, cfg):
    d = sdm.make_dims(**cfg.dims())
    n = sdm.workspace_bytes(d)
    # the scratch of one time chunk is held to about 4 GiB; long sequences run
    # as several chunks
    assert 0 < n < (9 << 29)


def _good():
    return dict(B=2, H=3, T=50, d_qk=16, d_v=16, n_sub=8, k=4, W=6, R=5, in_dtype=0)


@pytest.mark.parametrize("field,value,code", [
    ("d_qk", 15, ERR_DIMS), ("d_qk", 0, ERR_DIMS), ("k", 9, ERR_DIMS), ("k", 0, ERR_DIMS),
    ("W", 17, ERR_DIMS), ("R", 0, ERR_DIMS), ("B", 0, ERR_DIMS), ("T", -1, ERR_DIMS),
    ("in_dtype", 7, ERR_DIMS), ("n_sub", 46341, ERR_DIMS), ("d_v", 12, ERR_UNSUP),
    ("d_v", 256, ERR_UNSUP),
])
def test_bad_dims_rejected(lib, field, value, code):
    d = _good()
    d[field] = value
    dims = sdm.make_dims(**d)
    assert sdm.workspace_bytes(dims) == 0
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.sdm_forward(*([fake] * 9), ctypes.byref(dims), fake, 1 << 40, None)
    assert rc == code


def test_pointer_checks(lib):
    dims = sdm.make_dims(**_good())
    need = sdm.workspace_bytes(dims)
    fake = ctypes.c_void_p(1 << 20)
    args = [fake] * 9
    assert lib.sdm_forward(*args, ctypes.byref(dims), None, need, None) == ERR_WS
    assert lib.sdm_forward(*args, ctypes.byref(dims), fake, need - 1, None) == ERR_WS
    for i in range(9):
        a = list(args)
        a[i] = None
        assert lib.sdm_forward(*a, ctypes.byref(dims), fake, need, None) == ERR_NULL
        a[i] = ctypes.c_void_p((1 << 20) + 4)
        assert lib.sdm_forward(*a, ctypes.byref(dims), fake, need, None) == ERR_ALIGN
    sel = [fake] * 8
    assert lib.sdm_select(*sel[:4], None, *sel[5:], ctypes.byref(dims), fake, need, None) == ERR_NULL
    rec = [fake] * 9
    assert lib.sdm_recur(*rec, ctypes.byref(dims), fake, need - 1, None) == ERR_WS
    assert lib.sdm_get_device_status(None, 64, None, None, None) == ERR_NULL


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 4, 8)
    with pytest.raises(ValueError):
        sdm.forward(q, q, torch.zeros(1, 1, 4, 4), torch.zeros(1, 1, 4), torch.zeros(1, 1, 4),
                    torch.zeros(1, 4, 4), torch.zeros(1, 4, 4), torch.zeros(1, 1, 16, 4),
                    topk=2, W=2, R=2)
