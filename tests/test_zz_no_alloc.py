"""sdm_forward_noalloc: the entry point for callers that cannot allocate device
memory (its scratch is a fixed 64 MiB device array inside the library).

Called through the C ABI twice in a row, it must give the results of the
workspace-taking entry point sdm_forward within the parity tolerance (1e-4
relative per head), on CUDA-core and tensor-core scoring shapes and on a
workload whose usual workspace is larger than the array (it then runs in
shorter time chunks); and it must refuse a problem that does not fit the array
even in the shortest chunks.  This file is collected last so that a failure
here comes after every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_memory_linear_scoring_b200 as sdm
from gpu_util import REL_TOL, head_rel_err, to_device
from synth import config, gen_inputs

pytestmark = pytest.mark.gpu

SDM_ERR_SCRATCH_LIMIT = 8


def _lib():
    lib = sdm.load_library()
    fn = lib.sdm_forward_noalloc
    fn.argtypes = [ctypes.c_void_p] * 9 + [ctypes.POINTER(sdm.Dims), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _call(fn, d, M, o, dims):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(p(d["q"]), p(d["k"]), p(d["v"]), p(d["alpha"]), p(d["beta"]), p(d["C1"]),
              p(d["C2"]), p(M), p(o), ctypes.byref(dims), stream)


@pytest.mark.parametrize("cfg", [
    config(0).with_(m0_sd=0.5),
    config(1).with_(B=1, H=2, T=300, n_sub=64, k=16, W=32, R=32, m0_sd=0.5),
    config(1).with_(B=1, H=2, T=300, n_sub=256, k=32, W=64, R=64, m0_sd=0.5),
    config(1).with_(m0_sd=0.5),
], ids=["tiny-fp32", "small-bf16-cuda-cores", "small-bf16-tensor-cores", "small-full-chunked"])
def test_noalloc_matches_forward(cfg):
    fn = _lib()
    inp = gen_inputs(cfg)
    d = to_device(inp, cfg)
    dims = sdm.make_dims(**cfg.dims())
    if cfg.n_sub == 256:
        assert sdm.query_plan(dims)["tensor_core_scoring"] == 1
    if cfg.B == 4:
        # its one-chunk workspace (~194 MiB) exceeds the array: shorter chunks
        assert sdm.workspace_bytes(dims) > 64 << 20
    M_ref = d["M"].clone()
    o_ref = sdm.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["C1"], d["C2"], M_ref,
                        topk=cfg.k, W=cfg.W, R=cfg.R)
    torch.cuda.synchronize()
    for _ in range(2):                       # two calls in a row share the scratch
        M = d["M"].clone()
        o = torch.full_like(o_ref, float("nan"))
        assert _call(fn, d, M, o, dims) == 0
        torch.cuda.synchronize()
        assert (head_rel_err(o.cpu().numpy(), o_ref.cpu().numpy()) <= REL_TOL).all()
        assert (head_rel_err(M.cpu().numpy(), M_ref.cpu().numpy()) <= REL_TOL).all()


def test_noalloc_rejects_oversize():
    fn = _lib()
    # 1024 heads: one plan block of steps alone needs ~0.5 GiB of scratch
    cfg = config(4)
    dims = sdm.make_dims(**cfg.dims())
    assert sdm.workspace_bytes(dims) > 64 << 20
    t = torch.zeros(16, device="cuda")
    d = {n: t for n in ("q", "k", "v", "alpha", "beta", "C1", "C2")}
    assert _call(fn, d, t, t, dims) == SDM_ERR_SCRATCH_LIMIT
