"""The dense Gated DeltaNet baseline (sdm_gdn_forward, chunked on the GPU)
against its CPU oracle (the plain step-by-step recurrence in float64): every
o_t and the final state within 1e-4 of the head's largest |o|, |S|, at the
pages-scale matched size (d_k = W = 64, d_v = 64, T = 8192) and at ragged and
edge sizes (partial and single chunks, d_k and d_v from 16 to 128, float32
and bf16 inputs, a nonzero S_0)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_memory_linear_scoring_b200 as sdm
from gpu_util import REL_TOL, elem_rel_err, ncpu, report
from synth import config, gen_gdn_inputs

pytestmark = pytest.mark.gpu


def _run(cfg, d_k, s0_sd):
    inp = gen_gdn_inputs(cfg, d_k=d_k, s0_sd=s0_sd)
    dt = torch.bfloat16 if cfg.in_dtype == "bf16" else torch.float32
    d = {n: inp[n].to("cuda", dt if n in ("q", "k", "v") else torch.float32).contiguous()
         for n in inp}
    S = d["S0"].clone()
    o = sdm.gdn_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S)
    torch.cuda.synchronize()
    ref = oracle.gdn_forward({n: v.numpy() for n, v in inp.items()},
                             dict(B=cfg.B, H=cfg.H, T=cfg.T, d_k=d_k, d_v=cfg.d_v),
                             nthreads=ncpu())
    return o.cpu().numpy(), S.cpu().numpy(), ref


def _check(cfg, d_k, s0_sd=0.0):
    o, S, ref = _run(cfg, d_k, s0_sd)
    for name, g, r in (("o", o, ref["o"]), ("S", S, ref["S"])):
        g64, r64 = g.astype(np.float64), r.astype(np.float64)
        axes = tuple(range(2, r.ndim))
        err = np.abs(g64 - r64).max(axis=axes) / np.maximum(np.abs(r64).max(axis=axes), 1e-30)
        report("gdn %s %s d_k=%d" % (name, cfg.name, d_k), err, elem_rel_err(g64, r64))
        assert (err <= REL_TOL).all(), (name, err.max())


def test_gdn_pages_scale_matched():
    cfg = config(2)
    _check(cfg, d_k=cfg.W)


@pytest.mark.parametrize("shape,d_k,s0", [
    (dict(T=1), 64, 0.5), (dict(T=63), 64, 0.5), (dict(T=64), 64, 0.5), (dict(T=65), 64, 0.5),
    (dict(T=300, d_v=16), 16, 0.5), (dict(T=300, d_v=128), 128, 0.5),
    (dict(T=200, d_v=32), 128, 0.0), (dict(T=200, in_dtype="f32"), 32, 0.5),
    (dict(T=500, alpha_mu=0.0), 64, 0.5),
])
def test_gdn_shapes(shape, d_k, s0):
    cfg = config(2).with_(B=1, H=3, **shape)
    _check(cfg, d_k, s0)


def test_gdn_reproducible():
    cfg = config(2).with_(B=1, H=2, T=257)
    o1, S1, _ = _run(cfg, 64, 0.5)
    o2, S2, _ = _run(cfg, 64, 0.5)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)
