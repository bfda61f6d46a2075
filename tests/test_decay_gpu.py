"""The selective-decay write rule (the Raven page's router weights and
exp(a r) decay on SDM's product-key selection; sdm_forward_decay) against the
oracle's forward_decay: the same write and read sets as the oracle except at
flagged near-ties, and o and M within 1e-4 per head where every selection
agrees; rows never written stay bit-identical.  Runs on the CUDA-core, the
tensor-core (in-kernel top-k) and the tensor-core filter scoring paths."""
import numpy as np
import pytest
import torch

import oracle
import sparse_memory_linear_scoring_b200 as sdm
from gpu_util import (READ_BITS, REL_TOL, WRITE_BITS, elem_rel_err, head_rel_err, ncpu, np_inputs,
                      report, to_device)
from synth import config, gen_decay_rate, gen_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [
    config(0).with_(B=2, H=2, T=200, m0_sd=0.5),
    config(1).with_(B=1, H=2, T=300, n_sub=64, k=16, W=32, R=32, m0_sd=0.5),
    config(1).with_(B=1, H=2, T=300, n_sub=256, k=32, W=64, R=64, m0_sd=0.5),
    config(3).with_(B=1, H=2, T=160, m0_sd=0.5),
], ids=["fp32-cuda-cores", "bf16-cuda-cores", "bf16-tensor-cores", "bf16-tensor-core-filter"])
def test_decay_rule_against_oracle(cfg):
    inp = gen_inputs(cfg)
    inp["a"] = gen_decay_rate(cfg)
    d = to_device(inp, cfg)
    a = inp["a"].cuda().contiguous()
    M = d["M"].clone()
    o = sdm.forward_decay(d["q"], d["k"], d["v"], a, d["C1"], d["C2"], M, topk=cfg.k, W=cfg.W,
                          R=cfg.R)
    iw, _, ir, _ = sdm.select(d["q"], d["k"], d["C1"], d["C2"], topk=cfg.k, W=cfg.W, R=cfg.R)
    torch.cuda.synchronize()
    st, info = sdm.device_status()
    assert st == 0, (st, info)
    ref = oracle.forward_decay(np_inputs(inp), cfg.dims(), lists=True, nthreads=ncpu())
    same = np.ones((cfg.B, cfg.H, cfg.T), dtype=bool)
    for g, r, bits in ((iw, ref["idx_w"], WRITE_BITS), (ir, ref["idx_r"], READ_BITS)):
        eq = (np.sort(g.cpu().numpy().astype(np.int64), -1) == np.sort(r, -1)).all(-1)
        assert ((ref["flags"] & bits) != 0)[~eq].all(), "unflagged selection difference"
        same &= eq
    clean = same.all(-1)
    assert clean.any()
    og, Mg = o.cpu().numpy(), M.cpu().numpy()
    eo = head_rel_err(og, ref["o"])
    eM = head_rel_err(Mg, ref["M"])
    report("decay o %s" % cfg.name, eo[clean], elem_rel_err(og, ref["o"])[clean])
    report("decay M %s" % cfg.name, eM[clean], elem_rel_err(Mg, ref["M"])[clean])
    assert (eo[clean] <= REL_TOL).all(), eo
    assert (eM[clean] <= REL_TOL).all(), eM
    Mg, M0 = M.cpu().numpy(), inp["M0"].numpy()
    for b in range(cfg.B):
        for h in range(cfg.H):
            untouched = np.ones(cfg.N, dtype=bool)
            untouched[np.unique(ref["idx_w"][b, h])] = False
            untouched[np.unique(iw[b, h].cpu().numpy())] = False
            assert np.array_equal(Mg[b, h][untouched], M0[b, h][untouched])


def test_decay_zero_rate_freezes_the_table():
    """a = 0: exp(0) = 1 exactly, so every row keeps its bits."""
    cfg = config(1).with_(B=1, H=2, T=100, n_sub=256, k=32, W=64, R=64, m0_sd=0.5)
    inp = gen_inputs(cfg)
    d = to_device(inp, cfg)
    M = d["M"].clone()
    a = torch.zeros(cfg.B, cfg.H, cfg.T, device="cuda")
    sdm.forward_decay(d["q"], d["k"], d["v"], a, d["C1"], d["C2"], M, topk=cfg.k, W=cfg.W, R=cfg.R)
    torch.cuda.synchronize()
    assert torch.equal(M, d["M"])
