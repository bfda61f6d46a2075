"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
seeded synthetic workloads, element by element.

Bars: selected slot sets equal except at oracle-flagged near-ties (< 0.1% of
selections); o and M within 1e-4 relative (max abs error over max abs value,
per head); heads with a flagged selection difference are also compared after
feeding the oracle's lists to the recurrence kernel (sdm_recur), so a
legitimate tie flip is not scored as numeric error."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import sparse_memory_linear_scoring_b200 as sdm
from gpu_util import (READ_BITS, REL_TOL, WRITE_BITS, compare_lists, elem_rel_err, gpu_forward,
                      gpu_select, head_rel_err, np_inputs, oracle_full, report, to_device)
from synth import config, gen_inputs

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _status_clean():
    st, info = sdm.device_status()
    assert st == 0, "device status %d (info %d)" % (st, info)


def _check_forward(cfg, inp, ref, d=None):
    d = d if d is not None else to_device(inp, cfg)
    o, M = gpu_forward(d, cfg)
    iw, ww, ir, wr = gpu_select(d, cfg)
    torch.cuda.synchronize()
    _status_clean()
    _, same_w = compare_lists(iw.cpu().numpy(), ww.cpu().numpy(), ref["idx_w"], ref["w_w"],
                              ref["flags"], WRITE_BITS, "write lists")
    _, same_r = compare_lists(ir.cpu().numpy(), wr.cpu().numpy(), ref["idx_r"], ref["w_r"],
                              ref["flags"], READ_BITS, "read lists")
    clean = same_w.all(axis=-1) & same_r.all(axis=-1)          # [B,H]
    og, Mg = o.cpu().numpy(), M.cpu().numpy()
    eo = head_rel_err(og, ref["o"])
    eM = head_rel_err(Mg, ref["M"])
    # reported for the heads whose selections all agree (the others are
    # checked through the recurrence fed the oracle's lists, below)
    if clean.any():
        report("o %s" % cfg.name, eo[clean], elem_rel_err(og, ref["o"])[clean])
        report("M %s" % cfg.name, eM[clean], elem_rel_err(Mg, ref["M"])[clean])
    assert (eo[clean] <= REL_TOL).all(), eo
    assert (eM[clean] <= REL_TOL).all(), eM
    # the recurrence alone, fed the oracle's lists
    M2 = d["M"].clone()
    o2 = sdm.recur(d["v"], d["alpha"], d["beta"],
                   torch.from_numpy(ref["idx_w"].astype(np.int32)).cuda(),
                   torch.from_numpy(ref["w_w"].astype(np.float32)).cuda(),
                   torch.from_numpy(ref["idx_r"].astype(np.int32)).cuda(),
                   torch.from_numpy(ref["w_r"].astype(np.float32)).cuda(), M2,
                   d_qk=cfg.d_qk, n_sub=cfg.n_sub, topk=cfg.k)
    torch.cuda.synchronize()
    _status_clean()
    assert (head_rel_err(o2.cpu().numpy(), ref["o"], "o fed oracle lists %s" % cfg.name)
            <= REL_TOL).all()
    assert (head_rel_err(M2.cpu().numpy(), ref["M"], "M fed oracle lists %s" % cfg.name)
            <= REL_TOL).all()
    return o, M


def test_golden_hand_example():
    with open(os.path.join(GOLDEN, "hand_two_steps.json")) as f:
        g = json.load(f)
    dm = g["dims"]
    dev = "cuda"
    f32 = dict(dtype=torch.float32, device=dev)
    # d_v = 2 is below the kernels' 4-float row granule: pad rows with zeros
    pad = lambda a: torch.nn.functional.pad(torch.tensor(a, **f32), (0, 2))
    q = torch.tensor(g["q"], **f32)[None, None].contiguous()
    k = torch.tensor(g["k"], **f32)[None, None].contiguous()
    v = pad(g["v"])[None, None].contiguous()
    al = torch.tensor(g["alpha"], **f32)[None, None].contiguous()
    be = torch.tensor(g["beta"], **f32)[None, None].contiguous()
    C1 = torch.tensor(g["C1"], **f32)[None].contiguous()
    C2 = torch.tensor(g["C2"], **f32)[None].contiguous()
    M = pad(g["M0"])[None, None].contiguous()
    o = sdm.forward(q, k, v, al, be, C1, C2, M, topk=dm["k"], W=dm["W"], R=dm["R"])
    iw, ww, ir, wr = sdm.select(q, k, C1, C2, topk=dm["k"], W=dm["W"], R=dm["R"])
    torch.cuda.synchronize()
    _status_clean()
    e = g["expect"]
    assert iw[0, 0].cpu().tolist() == e["idx_w"]
    assert ir[0, 0].cpu().tolist() == e["idx_r"]
    np.testing.assert_allclose(ww[0, 0].cpu().numpy(), np.array(e["w_w"]), rtol=1e-6)
    np.testing.assert_allclose(o[0, 0, :, :2].cpu().numpy(), np.array(e["o"]), rtol=1e-6)
    np.testing.assert_allclose(M[0, 0, :, :2].cpu().numpy(), np.array(e["M"]), rtol=1e-6)
    assert (o[0, 0, :, 2:] == 0).all() and (M[0, 0, :, 2:] == 0).all()


@pytest.mark.parametrize("ci", [0, 1, 2])
def test_forward_parity_full(ci):
    cfg = config(ci)
    inp = gen_inputs(cfg)
    ref = oracle_full(inp, cfg, lists=True)
    o, M = _check_forward(cfg, inp, ref)
    # the unselected rows are bit-identical to M_0
    written = np.zeros((cfg.B, cfg.H, cfg.N), dtype=bool)
    for b in range(cfg.B):
        for h in range(cfg.H):
            written[b, h, np.unique(ref["idx_w"][b, h])] = True
    M0 = inp["M0"].numpy()
    Mg = M.cpu().numpy()
    assert np.array_equal(Mg[~written], M0[~written])


@pytest.mark.parametrize("shape", [
    dict(T=1), dict(T=2), dict(T=97), dict(T=1000), dict(W=1, R=1), dict(k=2, W=4, R=3),
    dict(W=64, R=1), dict(n_sub=8, k=8, W=64, R=64, T=64),
])
def test_forward_parity_shapes(shape):
    """Ragged blocks, single steps, W = k^2 (every candidate), W = R = 1."""
    base = config(1).with_(B=1, H=2, T=300, n_sub=64, k=16, W=32, R=32, m0_sd=0.5)
    cfg = base.with_(**shape)
    inp = gen_inputs(cfg)
    ref = oracle_full(inp, cfg, lists=True)
    _check_forward(cfg, inp, ref)


@pytest.mark.parametrize("shape", [
    dict(T=300), dict(T=1), dict(T=129), dict(k=8, W=16, R=8), dict(W=64, R=64, k=64, T=257),
    dict(n_sub=512, T=200), dict(B=3, H=1, T=140),
])
def test_tensor_core_scoring_shapes(shape):
    """bf16 shapes served by the tcgen05 scoring kernel: ragged 128-token tiles,
    several codebook tiles, small and large k."""
    import sparse_memory_linear_scoring_b200 as s
    base = config(1).with_(B=1, H=2, T=300, n_sub=256, k=32, W=64, R=64, m0_sd=0.5)
    cfg = base.with_(**shape)
    assert s.query_plan(s.make_dims(**cfg.dims()))["tensor_core_scoring"] == 1
    inp = gen_inputs(cfg)
    ref = oracle_full(inp, cfg, lists=True)
    _check_forward(cfg, inp, ref)


@pytest.mark.parametrize("shape", [
    dict(), dict(T=1), dict(T=129), dict(T=300, B=2, H=1),
    dict(d_qk=128, d_v=64, n_sub=512, k=128, W=128, R=128, T=200),
    dict(d_qk=128, d_v=64, n_sub=384, k=32, W=64, R=64, T=200),
    dict(d_qk=128, d_v=64, n_sub=128, k=16, W=32, R=32, T=200),
    dict(d_qk=256, d_v=32, n_sub=256, k=64, W=100, R=37, T=150),
])
def test_tensor_core_filter_shapes(shape):
    """bf16 shapes served by the tensor-core threshold filter and the survivor
    top-k (scoring mode 2): the long-context shape (d_h = 128, k = W = R = 128,
    recurring keys) with ragged and single steps, k = 128 at d_h = 64, and
    codebooks of 128 and 384 rows."""
    base = config(3).with_(B=1, H=2, T=300, m0_sd=0.5)
    cfg = base.with_(**shape)
    assert sdm.query_plan(sdm.make_dims(**cfg.dims()))["scoring_mode"] == 2
    inp = gen_inputs(cfg)
    ref = oracle_full(inp, cfg, lists=True)
    _check_forward(cfg, inp, ref)


@pytest.mark.parametrize("base", [
    config(1).with_(B=1, H=2, T=200, n_sub=256, k=32, W=64, R=64, m0_sd=0.5),
    config(3).with_(B=1, H=2, T=120, m0_sd=0.5),
    config(0).with_(B=1, H=2, T=150, m0_sd=0.5),
], ids=["bf16-tensor-core", "bf16-tensor-core-filter", "fp32"])
def test_duplicate_codebook_rows(base):
    """Duplicated codebook rows make exact score ties at every rank: the lower
    index must win in each half and among slots, on the GPU as in the oracle."""
    inp = gen_inputs(base)
    for name in ("C1", "C2"):
        c = inp[name].clone()
        c[:, 1::2] = c[:, 0::2]
        inp[name] = c
    ref = oracle_full(inp, base, lists=True)
    _check_forward(base, inp, ref)


@pytest.mark.parametrize("base", [
    config(2).with_(B=1, H=2, T=200, m0_sd=0.5),
    config(3).with_(B=1, H=2, T=120, m0_sd=0.5),
], ids=["bf16-tensor-core", "bf16-tensor-core-filter"])
def test_outlier_codebook_row(base):
    """One codebook row per half scaled by 64 (a power of two: exact in bf16), in a
    column past the 512 the threshold statistics read: every token whose score
    on row 0 is positive gets one score far above the rest.  The kept scores then
    crowd into the lowest buckets of their key range, which sends the in-kernel
    top-k to its bitwise-search path, gives the survivor top-k one large bucket,
    and crowds the merge's candidate buckets (its quickselect path)."""
    import sparse_memory_linear_scoring_b200 as s
    mode = s.query_plan(s.make_dims(**base.dims()))["scoring_mode"]
    assert mode == (1 if base.d_qk == 128 else 2)
    inp = gen_inputs(base)
    j = base.n_sub - 3
    assert j >= 512
    for name in ("C1", "C2"):
        c = inp[name].clone()
        c[:, j] = c[:, 0] * 64
        inp[name] = c
    ref = oracle_full(inp, base, lists=True)
    _check_forward(base, inp, ref)


def test_forward_run_to_run():
    """Two calls on the same inputs: M is each slot's float32 updates applied in
    time order by one stream, so its bits repeat; o sums each step's reads with
    float reductions from many streams in no fixed order, so it may differ in
    its last bits -- by float32 rounding of the sum, max |o1 - o2| / max |o| at
    most 1e-6 (the parity bar against the oracle is 1e-4)."""
    cfg = config(2).with_(B=1, H=4, T=1024)
    d = to_device(gen_inputs(cfg, device="cuda"), cfg)
    o1, M1 = gpu_forward(d, cfg)
    o2, M2 = gpu_forward(d, cfg)
    torch.cuda.synchronize()
    assert torch.equal(M1, M2)
    spread = float((o1 - o2).abs().max() / o1.abs().max())
    report("o run-to-run spread, pages-scale shape T=1024", [spread],
           [float(((o1 - o2).abs() / (o1.abs() + 1e-6 * o1.abs().max())).max())])
    assert spread <= 1e-6


def test_fp32_wide_rows():
    cfg = config(0).with_(B=2, H=3, T=200, d_v=128, d_qk=24, n_sub=16, k=6, W=20, R=12,
                          m0_sd=1.0)
    inp = gen_inputs(cfg)
    ref = oracle_full(inp, cfg, lists=True)
    _check_forward(cfg, inp, ref)


def test_empty_sequence():
    cfg = config(0).with_(T=0)
    inp = gen_inputs(cfg)
    d = to_device(inp, cfg)
    M = d["M"].clone()
    o = sdm.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["C1"], d["C2"], M,
                    topk=cfg.k, W=cfg.W, R=cfg.R)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(M, d["M"])


def test_recur_flags_bad_lists():
    """sdm_recur records out-of-range and repeated slots in the device status."""
    cfg = config(0).with_(T=8)
    inp = gen_inputs(cfg)
    d = to_device(inp, cfg)
    ref = oracle_full(inp, cfg, lists=True)
    iw = torch.from_numpy(ref["idx_w"].astype(np.int32)).cuda()
    ww = torch.from_numpy(ref["w_w"].astype(np.float32)).cuda()
    ir = torch.from_numpy(ref["idx_r"].astype(np.int32)).cuda()
    wr = torch.from_numpy(ref["w_r"].astype(np.float32)).cuda()
    bad = iw.clone()
    bad[0, 0, 3, 1] = cfg.N + 5
    M = d["M"].clone()
    sdm.recur(d["v"], d["alpha"], d["beta"], bad, ww, ir, wr, M, d_qk=cfg.d_qk, n_sub=cfg.n_sub,
              topk=cfg.k)
    st, info = sdm.device_status()
    assert st & 1 and info == 3
    rep = iw.clone()
    rep[0, 0, 5, 2] = rep[0, 0, 5, 1]
    sdm.recur(d["v"], d["alpha"], d["beta"], rep, ww, ir, wr, d["M"].clone(), d_qk=cfg.d_qk,
              n_sub=cfg.n_sub, topk=cfg.k)
    st, info = sdm.device_status()
    assert st & 8 and info == 5


def test_probe_random_rows():
    """The benchmark's random-row bandwidth probe (its own library): gathers
    leave the table unchanged, read-modify-writes add to it; bad arguments are
    rejected."""
    from sparse_memory_linear_scoring_b200.probe import probe_random_rows
    table = torch.zeros(4096, 64, dtype=torch.float32, device="cuda")
    probe_random_rows(table, rmw=False, rows_in_flight=4, ctas=2, iters=2)
    torch.cuda.synchronize()
    assert int((table != 0).sum()) == 0
    probe_random_rows(table, rmw=True, rows_in_flight=8, ctas=2, iters=2)
    torch.cuda.synchronize()
    assert float(table.sum()) > 0
    with pytest.raises(ValueError):
        probe_random_rows(table, rmw=True, rows_in_flight=3, ctas=2, iters=2)


def _repeat_inputs(cfg, period, share_qk):
    """Keys (and queries, with share_qk) that repeat with the given period, so
    the same slots come back every few steps: long runs of one slot inside a
    plan block, runs crossing chunk and block edges."""
    inp = gen_inputs(cfg)
    T = cfg.T
    idx = torch.arange(T) % period
    inp["k"] = inp["k"][:, :, idx].contiguous()
    if share_qk:
        inp["q"] = inp["k"].clone()
    return inp


@pytest.mark.parametrize("period,share", [(1, True), (3, False), (5, True), (64, True)])
def test_repeated_slots(period, share):
    cfg = config(1).with_(B=1, H=2, T=300, n_sub=64, k=16, W=32, R=32, m0_sd=0.5,
                          in_dtype="f32")
    inp = _repeat_inputs(cfg, period, share)
    ref = oracle_full(inp, cfg, lists=True)
    _check_forward(cfg, inp, ref)


@pytest.mark.parametrize("base", [
    config(1).with_(B=1, H=2, T=200, n_sub=64, k=16, W=24, R=16, m0_sd=0.5),
    config(3).with_(B=1, H=1, T=100, m0_sd=0.5),
], ids=["cuda-cores", "tensor-core-filter"])
def test_all_zero_keys_and_queries(base):
    """Every score is 0: every step selects the lowest slots (ties go to the
    lower index), so each plan block holds the same few slots P times over (on
    the tensor-core filter path every row is re-scored exactly)."""
    cfg = base
    inp = gen_inputs(cfg)
    inp["q"] = torch.zeros_like(inp["q"])
    inp["k"] = torch.zeros_like(inp["k"])
    ref = oracle_full(inp, cfg, lists=True)
    assert (ref["idx_w"] == np.sort(ref["idx_w"][0, 0, 0])).all()
    _check_forward(cfg, inp, ref)


@pytest.mark.parametrize("split", [1, 77, 128, 299])
def test_streaming_split(split):
    """Two calls over [0, s) and [s, T) with M carried equal one call over
    [0, T): M bit for bit (the same updates in the same order per slot), o
    within float32 reduction-order rounding."""
    cfg = config(1).with_(B=1, H=2, T=300, n_sub=256, k=32, W=64, R=64, m0_sd=0.5)
    inp = gen_inputs(cfg)
    d = to_device(inp, cfg)
    o1, M1 = gpu_forward(d, cfg)
    M2 = d["M"].clone()
    parts = []
    for lo, hi in ((0, split), (split, cfg.T)):
        sl = {n: (d[n][:, :, lo:hi].contiguous() if n in ("q", "k", "v", "alpha", "beta")
                  else d[n]) for n in d}
        parts.append(sdm.forward(sl["q"], sl["k"], sl["v"], sl["alpha"], sl["beta"], sl["C1"],
                                 sl["C2"], M2, topk=cfg.k, W=cfg.W, R=cfg.R))
    torch.cuda.synchronize()
    _status_clean()
    o2 = torch.cat(parts, dim=2)
    assert torch.equal(M1, M2)
    err = (o1 - o2).abs().max().item() / max(o1.abs().max().item(), 1e-30)
    assert err <= 1e-6, err
