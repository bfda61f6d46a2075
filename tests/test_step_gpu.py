"""sdm_step, the fused single-step kernel for decoding, against the CPU oracle.

Each test decodes a sequence through sdm_step -- one step per call (or a few),
with the table M carried from call to call -- and compares every step with the
oracle's run of the whole sequence:
  * the write and read sets of every step equal, except at near-ties the
    oracle flagged; weights within 2e-5;
  * every o_t and the final M within 1e-4 of the head's largest |o|, |M|, up to
    the first flagged selection difference of the head (after it the two runs
    legitimately diverge); at least one head of each test is compared whole.
Also: identical calls give identical bits (o is reduced in a fixed order), and
sizes the kernel does not serve are refused before anything runs."""
import numpy as np
import pytest
import torch

import sparse_memory_linear_scoring_b200 as sdm
from gpu_util import READ_BITS, REL_TOL, W_TOL, WRITE_BITS, oracle_full, report, elem_rel_err, \
    to_device
from synth import config, gen_inputs

pytestmark = pytest.mark.gpu


def _decode(cfg, d, per_call):
    """Run the sequence through sdm_step, per_call steps per call, M carried."""
    M = d["M"].clone()
    outs = []
    for t0 in range(0, cfg.T, per_call):
        t1 = min(cfg.T, t0 + per_call)
        sl = {n: d[n][:, :, t0:t1].contiguous() for n in ("q", "k", "v", "alpha", "beta")}
        outs.append(sdm.step(sl["q"], sl["k"], sl["v"], sl["alpha"], sl["beta"], d["C1"],
                             d["C2"], M, topk=cfg.k, W=cfg.W, R=cfg.R, lists=True))
    torch.cuda.synchronize()
    cat = [torch.cat([o[i] for o in outs], dim=2).cpu().numpy() for i in range(5)]
    return cat, M.cpu().numpy()


def _check_decode(cfg, inp, per_call=1):
    d = to_device(inp, cfg)
    (o, iw, ww, ir, wr), M = _decode(cfg, d, per_call)
    ref = oracle_full(inp, cfg, lists=True)
    whole = 0
    for b in range(cfg.B):
        for h in range(cfg.H):
            fl = ref["flags"][b, h]
            upto = cfg.T
            for gi, gw, oi, ow, bits in ((iw, ww, ref["idx_w"], ref["w_w"], WRITE_BITS),
                                         (ir, wr, ref["idx_r"], ref["w_r"], READ_BITS)):
                same = (np.sort(gi[b, h], -1) == np.sort(oi[b, h], -1)).all(-1)
                assert ((fl & bits) != 0)[~same].all(), \
                    "unflagged selection difference at (%d,%d,%s)" % (b, h, np.argwhere(~same)[:3])
                if not same.all():
                    upto = min(upto, int(np.argmin(same)))
                # weights where the sets agree, matched by slot
                go, oo = np.argsort(gi[b, h], -1), np.argsort(oi[b, h], -1)
                e = np.abs(np.take_along_axis(gw[b, h].astype(np.float64), go, -1)
                           - np.take_along_axis(ow[b, h], oo, -1))[same]
                assert e.size == 0 or e.max() <= W_TOL, e.max()
            if upto == 0:
                continue
            r_o = ref["o"][b, h, :upto].astype(np.float64)
            g_o = o[b, h, :upto].astype(np.float64)
            err = np.abs(g_o - r_o).max() / max(1e-30, np.abs(r_o).max())
            report("step o %s (%d,%d)" % (cfg.name, b, h), err,
                   elem_rel_err(g_o[None, None], r_o[None, None]))
            assert err <= REL_TOL, ("o", b, h, err)
            if upto == cfg.T:
                whole += 1
                r_M = ref["M"][b, h].astype(np.float64)
                g_M = M[b, h].astype(np.float64)
                errM = np.abs(g_M - r_M).max() / max(1e-30, np.abs(r_M).max())
                report("step M %s (%d,%d)" % (cfg.name, b, h), errM,
                       elem_rel_err(g_M[None, None], r_M[None, None]))
                assert errM <= REL_TOL, ("M", b, h, errM)
    assert whole >= 1, "no head compared over the whole sequence"
    return o, M


@pytest.mark.parametrize("ci,shape,per_call", [
    (2, dict(B=1, H=2, T=96), 1),
    (2, dict(B=1, H=2, T=96), 7),
    (3, dict(B=1, H=2, T=64), 1),
    (4, dict(B=2, H=2, T=80), 1),
    (1, dict(B=2, H=2, T=96), 1),
    (0, dict(T=128), 1),
    (0, dict(T=128), 128),
], ids=["pages-scale", "pages-scale-7-per-call", "long-context", "high-batch", "small",
        "tiny-fp32", "tiny-fp32-one-call"])
def test_step_decode_against_oracle(ci, shape, per_call):
    cfg = config(ci).with_(**shape)
    if cfg.m0_sd == 0:
        cfg = cfg.with_(m0_sd=0.5)
    _check_decode(cfg, gen_inputs(cfg), per_call)


def test_step_ties():
    """Duplicated codebook rows (exact ties at every rank) and an all-zero key
    (every score 0): the lower index wins, as in the oracle."""
    cfg = config(2).with_(B=1, H=2, T=48, m0_sd=0.5)
    inp = gen_inputs(cfg)
    for name in ("C1", "C2"):
        c = inp[name].clone()
        c[:, 1::2] = c[:, 0::2]
        inp[name] = c
    inp["k"][:, :, 5] = 0
    _check_decode(cfg, inp, 1)


def test_step_reproducible():
    cfg = config(2).with_(B=1, H=2, T=32, m0_sd=0.5)
    d = to_device(gen_inputs(cfg), cfg)
    (o1, *_), M1 = _decode(cfg, d, 1)
    (o2, *_), M2 = _decode(cfg, d, 1)
    assert np.array_equal(o1, o2) and np.array_equal(M1, M2)


def test_step_refuses_unserved_sizes():
    """n_sub = 2048 is beyond the kernel's 1024 scores per half-row: the library
    returns SDM_ERR_UNSUPPORTED (the binding's shape checks all pass)."""
    cfg = config(2).with_(B=1, H=1, T=2, n_sub=4, d_v=4)
    d = to_device(gen_inputs(cfg), cfg)
    C = torch.zeros(1, 2048, cfg.d_h, dtype=torch.bfloat16, device="cuda")
    M = torch.zeros(1, 1, 2048 * 2048, cfg.d_v, device="cuda")
    with pytest.raises(sdm.SDMError) as e:
        sdm.step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], C, C, M, topk=64, W=64, R=64)
    assert e.value.code == 5
