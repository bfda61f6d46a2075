"""Helpers of the GPU parity tests: device copies of the synthetic inputs and
the comparisons against the CPU oracle (tolerances stated where used)."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
import sparse_memory_linear_scoring_b200 as sdm

# o and M: max |gpu - oracle| / max |oracle| per (b,h) head (the workload's
# "max relative error <= 1e-4", read per head so that near-zero elements do not
# blow it up).  The elementwise figure max |gpu - oracle| / (|oracle| + 1e-6 max
# |oracle|) is also computed and, when SDM_PARITY_REPORT names a file, appended
# there per check (it is reported, not asserted: its floor makes it large for
# elements that are tiny next to the head's largest).
REL_TOL = 1e-4
# softmax weights: float32 exp/sum on the GPU vs float64 in the oracle
W_TOL = 2e-5
# at most this fraction of selections may differ, and only where the oracle
# flagged a near-tie (float64 gap below 1e-5 relative at a selection boundary)
FLAGGED_FRAC = 1e-3

WRITE_BITS = 0b000111
READ_BITS = 0b111000


def ncpu() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count())


def to_device(inp, cfg, device="cuda"):
    dt = torch.bfloat16 if cfg.in_dtype == "bf16" else torch.float32
    out = {}
    for name in ("q", "k", "v", "C1", "C2"):
        out[name] = inp[name].to(device=device, dtype=dt).contiguous()
    for name in ("alpha", "beta"):
        out[name] = inp[name].to(device=device, dtype=torch.float32).contiguous()
    if "M0" in inp:
        out["M"] = inp["M0"].to(device=device, dtype=torch.float32).contiguous()
    return out


def gpu_forward(d, cfg):
    M = d["M"].clone()
    o = sdm.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["C1"], d["C2"], M,
                    topk=cfg.k, W=cfg.W, R=cfg.R)
    return o, M


def gpu_select(d, cfg):
    return sdm.select(d["q"], d["k"], d["C1"], d["C2"], topk=cfg.k, W=cfg.W, R=cfg.R,
                      d_v=cfg.d_v)


def np_inputs(inp):
    return {k: v.numpy() if hasattr(v, "numpy") else v for k, v in inp.items()}


def compare_lists(g_idx, g_w, o_idx, o_w, flags, bits, what):
    """Sets equal per step except at flagged near-ties; weights matched by slot."""
    g_idx = np.asarray(g_idx).astype(np.int64)
    gs = np.sort(g_idx, axis=-1)
    os_ = np.sort(o_idx, axis=-1)
    same = (gs == os_).all(axis=-1)
    flagged = (flags & bits) != 0
    bad = ~same & ~flagged
    n_mis = int((~same).sum())
    assert not bad.any(), "%s: %d unflagged selection mismatches, first at %s" % (
        what, int(bad.sum()), np.argwhere(bad)[:3].tolist())
    assert n_mis <= FLAGGED_FRAC * same.size, "%s: %d flagged mismatches of %d" % (
        what, n_mis, same.size)
    # weights aligned by slot where the sets agree
    go = np.argsort(g_idx, axis=-1)
    oo = np.argsort(o_idx, axis=-1)
    gw = np.take_along_axis(np.asarray(g_w, dtype=np.float64), go, axis=-1)
    ow = np.take_along_axis(o_w, oo, axis=-1)
    err = np.abs(gw - ow)[same]
    if err.size:
        assert err.max() <= W_TOL, "%s: weight error %g" % (what, err.max())
    return n_mis, same


def head_rel_err(g, ref, what=None):
    g = np.asarray(g, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    axes = tuple(range(2, ref.ndim))
    den = np.abs(ref).max(axis=axes)
    den = np.where(den == 0, 1.0, den)
    err = np.abs(g - ref).max(axis=axes) / den
    if what is not None:
        report(what, err, elem_rel_err(g, ref))
    return err


def elem_rel_err(g, ref):
    """Per head: max over elements of |g - ref| / (|ref| + 1e-6 * max |ref|)."""
    g = np.asarray(g, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    axes = tuple(range(2, ref.ndim))
    floor = 1e-6 * np.abs(ref).max(axis=axes, keepdims=True)
    floor = np.where(floor == 0, 1e-300, floor)
    return (np.abs(g - ref) / (np.abs(ref) + floor)).max(axis=axes)


def report(what, head_err, elem_err):
    path = os.environ.get("SDM_PARITY_REPORT")
    if not path:
        return
    import json
    with open(path, "a") as f:
        f.write(json.dumps({"check": what, "head_rel_max": float(np.max(head_err)),
                            "elem_rel_max": float(np.max(elem_err))}) + "\n")


def oracle_full(inp, cfg, **kw):
    return oracle.forward(np_inputs(inp), cfg.dims(), nthreads=ncpu(), **kw)
