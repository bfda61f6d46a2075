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
        gate = i in (3, 4)                   # alpha, beta: 4-byte alignment suffices
        a[i] = ctypes.c_void_p((1 << 20) + (2 if gate else 4))
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


def _cpu_args(**over):
    """Consistent CPU tensors of a small bf16 problem (B=2, H=3, T=5, d_qk=8,
    d_v=4, n_sub=4), with named replacements."""
    import torch
    B, H, T, dqk, dv, n = 2, 3, 5, 8, 4, 4
    bf = torch.bfloat16
    a = dict(q=torch.zeros(B, H, T, dqk, dtype=bf), k=torch.zeros(B, H, T, dqk, dtype=bf),
             v=torch.zeros(B, H, T, dv, dtype=bf), alpha=torch.zeros(B, H, T),
             beta=torch.zeros(B, H, T), C1=torch.zeros(H, n, dqk // 2, dtype=bf),
             C2=torch.zeros(H, n, dqk // 2, dtype=bf), M=torch.zeros(B, H, n * n, dv))
    a.update(over)
    return a


def _fwd(a, **kw):
    return sdm.forward(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["C1"], a["C2"], a["M"],
                       topk=2, W=2, R=2, **kw)


@pytest.mark.parametrize("name,bad,exc", [
    ("q", "float16", TypeError),
    ("k", (2, 3, 5, 6), ValueError),
    ("k", "float32", TypeError),
    ("v", "float32", TypeError),
    ("v", (2, 3, 4, 4), ValueError),
    ("alpha", (2, 3, 1), ValueError),
    ("alpha", "bfloat16", TypeError),
    ("beta", (3, 2, 5), ValueError),
    ("C2", (3, 5, 4), ValueError),
    ("C1", (3, 4, 3), ValueError),
    ("M", (2, 3, 15, 4), ValueError),
    ("M", "bfloat16", TypeError),
])
def test_binding_rejects_mismatches(name, bad, exc):
    """Every tensor is checked against the dims before anything is launched (a
    short M or a float16 input would otherwise reach a kernel)."""
    import torch
    a = _cpu_args()
    if isinstance(bad, str):
        a[name] = a[name].to(getattr(torch, bad))
    else:
        a[name] = torch.zeros(bad, dtype=a[name].dtype)
    with pytest.raises(exc):
        _fwd(a)


def test_binding_rejects_bad_output_and_lists():
    import torch
    a = _cpu_args()
    with pytest.raises(ValueError):
        _fwd(a, o=torch.zeros(2, 3, 5, 8))
    with pytest.raises(TypeError):
        _fwd(a, o=torch.zeros(2, 3, 5, 4, dtype=torch.float64))
    with pytest.raises(TypeError):
        sdm.make_dims(1, 1, 1, 8, 4, 4, 2, 2, 2, torch.float16)
    B, H, T = 2, 3, 5
    lists = dict(idx_w=torch.zeros(B, H, T, 2, dtype=torch.int64),
                 w_w=torch.zeros(B, H, T, 2), idx_r=torch.zeros(B, H, T, 2, dtype=torch.int32),
                 w_r=torch.zeros(B, H, T, 2))
    with pytest.raises(TypeError):
        sdm.recur(a["v"], a["alpha"], a["beta"], lists["idx_w"], lists["w_w"], lists["idx_r"],
                  lists["w_r"], a["M"], d_qk=8, n_sub=4, topk=2)
    lists["idx_w"] = lists["idx_w"].to(torch.int32)
    with pytest.raises(ValueError):
        sdm.recur(a["v"], a["alpha"], a["beta"], lists["idx_w"], lists["w_w"], lists["idx_r"],
                  torch.zeros(B, H, T, 3), a["M"], d_qk=8, n_sub=4, topk=2)
    with pytest.raises(ValueError):
        sdm.select(a["q"], a["k"][:, :, :4], a["C1"], a["C2"], topk=2, W=2, R=2)
