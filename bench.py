#!/usr/bin/env python
"""Benchmark of the SDM forward pass: token-heads/s at N = 2^20 slots per head.

Workload (default): the pages-scale workload -- B=2, H=4, T=8192, d_qk=128
(halves of 64), codebooks 1024 x 64 per head (N = 2^20), d_v=64, k=64, W=R=64,
bf16 inputs, float32 state.  One step = one full forward pass (scoring,
selection, gated delta recurrence, reads) over the batch.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sdm|reference]
                  [--config 0..4] [--T steps] [--decode] [--probe-rows]

Prints one JSON line (rank 0).  Under torchrun each rank owns a contiguous
range of the flat (b,h) heads of a world-times-larger head grid (weak scaling,
no collective on the data path) and runs it as rectangular pieces of the grid;
time is the max over ranks of the summed per-step CUDA-event times, with L2
flushed between steps.  The line also carries: the roofline of the dominant
kernel and of the scoring contraction; the random-row ceiling of the
recurrence's access pattern, measured in the same run; an end-to-end rate
through the public API with pinned host inputs and outputs copied every step
(pipelined with the compute, as a serving loop would); the oracle timed on the
host cores (all of them, and one); and a parity sample: the GPU's selections
against the oracle's on the oracle's sample, with the rate of near-ties the
oracle flagged.  --impl reference times the oracle alone.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SDM forward token-heads/s at N=2^20; slot-traffic HBM GB/s vs B200 peak"
UNIT = "token-heads/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["sdm", "reference"], default="sdm")
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--T", type=int, default=0,
                    help="override the number of steps (small profiling captures only)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-probe", action="store_true",
                    help="skip the random-row probe of the recurrence's access pattern")
    ap.add_argument("--decode", action="store_true",
                    help="time single-step calls (T = 1, M carried), eagerly and as one CUDA "
                         "graph of --steps steps, on the workload's heads, and exit")
    ap.add_argument("--gdn", action="store_true",
                    help="time the dense Gated DeltaNet baseline at the matched size (d_k = W, "
                         "same B, H, T, d_v, gates) beside the SDM forward pass, and exit")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (sdm_backward) beside the forward pass on the "
                         "workload, and exit")
    ap.add_argument("--probe-rows", action="store_true",
                    help="measure the HBM ceiling of random 256-byte row gathers and "
                         "read-modify-writes (the recurrence's access pattern) and exit")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one k_recur
# launch per token-head, measured by ncu on the pages-scale workload at
# T = 1024 (8192 token-heads): 271.6 MB read + 90.4 MB written.  Valid only for
# the recurrence source it was taken on (its SHA-256 below).
RECUR_DRAM_BYTES_PER_TOKEN_HEAD = (271587584 + 90435072) / 8192.0
RECUR_DRAM_SOURCE_SHA256 = "0ee48857b052a60d68bbc1fd1273470b53448c57b4d0531cd578677d51ee9fc9"


def recur_traffic(token_heads: int):
    """Per-launch DRAM traffic of k_recur scaled from the capture, or None when
    the recurrence source changed since the counters were taken."""
    import hashlib
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                       "sparse_memory_linear_scoring_b200", "csrc", "recur.cu")
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    if sha != RECUR_DRAM_SOURCE_SHA256:
        return None
    return RECUR_DRAM_BYTES_PER_TOKEN_HEAD * token_heads


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def workload_desc(cfg):
    return ("%s: B=%d H=%d T=%d d_qk=%d d_v=%d n_sub=%d (N=%d) k=%d W=%d R=%d %s inputs, f32 state"
            % (cfg.name, cfg.B, cfg.H, cfg.T, cfg.d_qk, cfg.d_v, cfg.n_sub, cfg.N, cfg.k, cfg.W,
               cfg.R, cfg.in_dtype))


# ----------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.proc = None
        self.path = None
        self.uuid = uuid

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="sdm_clocks_", suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                   "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------- cpu baseline
def cpu_baseline(cfg, target_s: float, b0: int = 0):
    """The oracle, as it stands, on a bounded sample of the workload: the first
    min(B*H, host threads) heads over a prefix of T_s steps, on all host threads;
    then one head on one thread.  Returns the baseline and the oracle's lists of
    the sample (for the parity sample)."""
    import oracle
    from synth import gen_inputs

    nthr = host_threads()
    nheads = min(cfg.BH, nthr)
    sub = cfg.with_(B=1, H=1)
    # calibrate on one head: the marginal cost of a step (the difference of a
    # 16- and a 64-step run; the fixed cost of a call is the table's copy)
    def run_one(steps):
        one = gen_inputs(sub, t_end=steps, b0=b0)
        npi = {k: v.numpy() for k, v in one.items()}
        d = dict(cfg.dims(), B=1, H=1, T=steps)
        t = time.perf_counter()
        oracle.forward(npi, d)
        return time.perf_counter() - t
    t16, t64 = run_one(16), run_one(64)
    per_step = max((t64 - t16) / 48, t64 / 64 / 10)
    waves = (nheads + nthr - 1) // nthr
    T_s = int(max(16, min(cfg.T, target_s / max(per_step * waves, 1e-9))))
    heads = [(hh // cfg.H, hh % cfg.H) for hh in range(nheads)]
    Bs = cfg.with_(B=max(b for b, _ in heads) + 1)
    inp = gen_inputs(Bs, t_end=T_s, b0=b0)
    npi = {k: v.numpy() for k, v in inp.items()}
    dd = dict(Bs.dims(), T=T_s)
    flat = [b * cfg.H + h for b, h in heads]
    t = time.perf_counter()
    ref = oracle.forward(npi, dd, heads=flat, nthreads=nthr, lists=True)
    el = time.perf_counter() - t
    # one head, one thread, a quarter of the time
    T_1 = int(max(16, min(cfg.T, target_s / 4 / max(per_step, 1e-9))))
    one = gen_inputs(sub, t_end=T_1, b0=b0)
    t = time.perf_counter()
    oracle.forward({k: v.numpy() for k, v in one.items()}, dict(cfg.dims(), B=1, H=1, T=T_1),
                   nthreads=1)
    el1 = time.perf_counter() - t
    base = {"value": nheads * T_s / el, "unit": UNIT, "cores": min(nthr, nheads), "kind": "oracle",
            "sample": "%d heads x first %d steps of %s (oracle C, float64, %d threads, %.1f s)"
                      % (nheads, T_s, cfg.name, min(nthr, nheads), el),
            "value_1thread": T_1 / el1,
            "sample_1thread": "1 head x first %d steps, 1 thread, %.1f s" % (T_1, el1)}
    return base, {"ref": ref, "heads": heads, "T": T_s}


def parity_sample(lists, sample):
    """GPU selections (sdm_select lists of the first batch rows) against the
    oracle's on the CPU baseline's sample: mismatched sets, and how many of them
    and of all selections the oracle flagged as near-ties."""
    import numpy as np
    ref, T = sample["ref"], sample["T"]
    n_sel = mism = unflagged = flagged = 0
    for (b, h) in sample["heads"]:
        fl = ref["flags"][b, h, :T]
        for gi, oi, bits in ((lists[0], ref["idx_w"], 0b000111), (lists[2], ref["idx_r"], 0b111000)):
            g = np.sort(gi[b, h, :T].cpu().numpy().astype(np.int64), -1)
            o = np.sort(oi[b, h, :T], -1)
            same = (g == o).all(-1)
            f = (fl & bits) != 0
            n_sel += same.size
            mism += int((~same).sum())
            unflagged += int((~same & ~f).sum())
            flagged += int(f.sum())
    return {"selections": n_sel, "mismatched": mism, "unflagged_mismatched": unflagged,
            "flagged_near_ties": flagged, "flagged_rate": flagged / max(1, n_sel),
            "sample": "the CPU baseline's heads and steps"}


# ---------------------------------------------------------------------- sdm arm
def _device_uuid(torch, dev):
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        return None


def run_sdm(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import sparse_memory_linear_scoring_b200 as sdm
    from sparse_memory_linear_scoring_b200.parallel import head_pieces, max_over_ranks, shard_heads
    from synth import gen_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    # weak scaling: the head grid is (world * B) x H; rank r owns the flat heads
    # [r*B*H, (r+1)*B*H), run as rectangular pieces of the grid (here one piece
    # of B batch rows, since B*H is a whole number of rows)
    f0, nh = shard_heads(world * cfg.BH, world, rank)
    pieces = head_pieces(f0, nh, cfg.H)
    dt = torch.bfloat16 if cfg.in_dtype == "bf16" else torch.float32
    runs = []
    for pc in pieces:
        pcfg = cfg.with_(B=pc.b1 - pc.b0, H=pc.h1 - pc.h0)
        # inputs made on the device by the seeded generator, one batch row at a
        # time (the high-batch table is 64 GiB)
        d = {}
        M = torch.empty(pcfg.B, pcfg.H, cfg.N, cfg.d_v, dtype=torch.float32, device=dev)
        for i in range(pcfg.B):
            part = gen_inputs(cfg.with_(B=1), device=str(dev), b0=pc.b0 + i, h0=pc.h0, h1=pc.h1)
            for n in ("q", "k", "v", "alpha", "beta"):
                if n not in d:
                    shape = (pcfg.B,) + tuple(part[n].shape[1:])
                    d[n] = torch.empty(shape, dtype=dt if n in ("q", "k", "v") else torch.float32,
                                       device=dev)
                d[n][i] = part[n][0]
            M[i] = part["M0"][0]
            if i == 0:
                d["C1"] = part["C1"].to(dt).contiguous()
                d["C2"] = part["C2"].to(dt).contiguous()
            del part
        d["M"] = M
        d["o"] = torch.empty(pcfg.B, pcfg.H, cfg.T, cfg.d_v, dtype=torch.float32, device=dev)
        runs.append((pcfg, d, sdm.query_plan(sdm.make_dims(**pcfg.dims()))))
    plan = runs[0][2]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    # phase events of the first piece (the only one unless heads split rows)
    nph = 5 * plan["chunks"]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(nph)]
    for e in ev:          # torch creates the CUDA event on its first record
        e.record()
    torch.cuda.synchronize(dev)

    def step(events=None):
        for i, (pcfg, d, _) in enumerate(runs):
            sdm.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["C1"], d["C2"], d["M"],
                        topk=cfg.k, W=cfg.W, R=cfg.R, o=d["o"],
                        events=events if i == 0 else None)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st, info = sdm.device_status()
    if st != 0:
        raise RuntimeError("device status %d (info %d) after warm-up" % (st, info))

    clocks = ClockSampler(_device_uuid(torch, dev))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    total = 0.0
    phase = [0.0, 0.0, 0.0, 0.0]
    for _ in range(args.steps):
        flush.zero_()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record()
        step(ev)
        s1.record()
        s1.synchronize()
        total += s0.elapsed_time(s1)
        for c in range(plan["chunks"]):
            for j in range(4):
                phase[j] += ev[5 * c + j].elapsed_time(ev[5 * c + j + 1])
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    st, info = sdm.device_status()
    if st != 0:
        raise RuntimeError("device status %d (info %d) after timing" % (st, info))
    t_max = max_over_ranks(total, dev)
    phase = [max_over_ranks(x, dev) for x in phase]

    # ---- end to end through the public API: pinned host inputs -> device ->
    # forward -> o back to pinned host memory, every step.  The steps run as a
    # pipeline, as a serving loop would: step i+1's inputs are copied in on one
    # stream and step i-1's o is copied out on another while step i computes
    # (two device buffers each; M carries from step to step on the compute
    # stream).  Timed from the first copy to the last, divided by the steps.
    e2e = None
    if not args.no_e2e:
        names = ("q", "k", "v", "alpha", "beta")
        comp = torch.cuda.current_stream(dev)
        cin = torch.cuda.Stream(dev)
        cout = torch.cuda.Stream(dev)
        pipes = []
        h2d = d2h = 0
        for pcfg, d, _ in runs:
            host = {n: torch.empty_like(d[n], device="cpu").pin_memory() for n in names}
            for n in names:
                host[n].copy_(d[n])
            o_host = [torch.empty(d["o"].shape, dtype=d["o"].dtype).pin_memory()
                      for _ in range(2)]
            dbuf = [{n: torch.empty_like(d[n]) for n in names} for _ in range(2)]
            obuf = [torch.empty_like(d["o"]) for _ in range(2)]
            h2d += sum(host[n].numel() * host[n].element_size() for n in names)
            d2h += o_host[0].numel() * o_host[0].element_size()
            pipes.append((d, host, o_host, dbuf, obuf))

        def run_pipeline(nsteps, start=None):
            if start is not None:
                cin.wait_event(start)                    # no copy before the timer starts
            ev_in = [torch.cuda.Event() for _ in range(nsteps)]
            ev_done = [torch.cuda.Event() for _ in range(nsteps)]
            ev_out = [torch.cuda.Event() for _ in range(nsteps)]
            for i in range(nsteps):
                j = i & 1
                with torch.cuda.stream(cin):
                    if i >= 2:
                        cin.wait_event(ev_done[i - 2])   # buffer j is free again
                    for (_, host, _, dbuf, _) in pipes:
                        for n in names:
                            dbuf[j][n].copy_(host[n], non_blocking=True)
                    ev_in[i].record(cin)
                comp.wait_event(ev_in[i])
                if i >= 2:
                    comp.wait_event(ev_out[i - 2])       # o buffer j was copied out
                for (d, _, _, dbuf, obuf) in pipes:
                    sdm.forward(dbuf[j]["q"], dbuf[j]["k"], dbuf[j]["v"], dbuf[j]["alpha"],
                                dbuf[j]["beta"], d["C1"], d["C2"], d["M"], topk=cfg.k, W=cfg.W,
                                R=cfg.R, o=obuf[j])
                ev_done[i].record(comp)
                with torch.cuda.stream(cout):
                    cout.wait_event(ev_done[i])
                    for (_, _, o_host, _, obuf) in pipes:
                        o_host[j].copy_(obuf[j], non_blocking=True)
                    ev_out[i].record(cout)
            comp.wait_stream(cout)
            comp.wait_stream(cin)

        run_pipeline(max(2, args.warmup))
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(comp)
        run_pipeline(args.steps, s0)
        s1.record(comp)
        s1.synchronize()
        et = max_over_ranks(s0.elapsed_time(s1), dev)
        e2e = {"value": world * cfg.BH * cfg.T * args.steps / (et / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": et / args.steps,
               "pipelined": "copies of steps i+1 (in) and i-1 (out) overlap step i",
               "l2": "not flushed: the state is larger than L2"}
        del pipes

    # the selection lists of the first piece, for the parity sample
    lists = None
    if rank == 0 and not args.no_cpu_baseline:
        pcfg, d, _ = runs[0]
        lists = sdm.select(d["q"], d["k"], d["C1"], d["C2"], topk=cfg.k, W=cfg.W, R=cfg.R,
                           d_v=cfg.d_v)
        torch.cuda.synchronize(dev)

    # the random-row ceiling of the recurrence's access pattern, this run
    pat = None
    if not args.no_probe:
        del flush
        pat = pattern_ceiling(cfg.W, cfg.R)
    if rank != 0:
        return None, None
    pk, src = peaks()
    K = args.steps
    th = cfg.BH * cfg.T
    value = world * th * K / (t_max / 1e3)
    names = ["score", "merge", "plan", "recur"]
    shares = {n: phase[i] / max(1e-12, sum(phase)) for i, n in enumerate(names)}
    per = {n: phase[i] / K for i, n in enumerate(names)}
    dom = max(names, key=lambda n: per[n])
    th0 = runs[0][0].BH * cfg.T                 # token-heads of the timed piece
    slot_bytes = th0 * (2 * cfg.W + cfg.R) * cfg.d_v * 4
    score_flops = th0 * 4 * cfg.n_sub * cfg.d_qk
    fp32_peak = 148 * 128 * 2 * float(pk.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
    rec_gbs = slot_bytes / (per["recur"] / 1e3) / 1e9
    if plan["tensor_core_scoring"]:
        roof_s = {"kernel": "k_score_tc", "bound": "tensor",
                  "achieved": score_flops / (per["score"] / 1e3) / 1e12,
                  "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "peak_kind": "bf16 burst"}
    else:
        roof_s = {"kernel": "k_score_warp", "bound": "alu",
                  "achieved": score_flops / (per["score"] / 1e3) / 1e12,
                  "peak": fp32_peak, "unit": "TFLOP/s",
                  "peak_kind": "float32 FMA, 148 SMs x 128 lanes x 2 x max clock"}
    roof_s["frac"] = roof_s["achieved"] / roof_s["peak"]
    roof_s["flops_per_launch"] = score_flops
    roof_s["peak_source"] = src
    if dom == "recur":
        roof = {"kernel": "k_recur", "bound": "hbm", "achieved": rec_gbs,
                "peak": pk["hbm_gbs"], "unit": "GB/s",
                "traffic": recur_traffic(th0) if plan["chunks"] == 1 else None,
                "bytes_per_launch": slot_bytes / plan["chunks"]}
        roof["frac"] = roof["achieved"] / roof["peak"]
    elif dom == "score":
        roof = dict(roof_s, traffic=None)
    else:
        roof = {"kernel": {"merge": "k_merge", "plan": "k_plan"}[dom], "bound": "alu",
                "achieved": None, "peak": fp32_peak, "unit": "TFLOP/s", "frac": None,
                "traffic": None}
    roof["peak_source"] = src
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": t_max / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "global_batch": cfg.B * world,
                   "heads": cfg.H, "seq_len": cfg.T,
                   "parallelism": "dp%d: (b,h) heads sharded across ranks, no collective" % world,
                   "l2": "flushed between steps (256 MiB write)"},
        "roofline": roof,
        "roofline_scoring": roof_s,
        "slot_traffic": {"bytes_per_step": slot_bytes, "recur_gbs": rec_gbs,
                         "recur_frac_of_8TBs": rec_gbs / 8000.0,
                         "recur_frac_of_measured": rec_gbs / pk["hbm_gbs"],
                         "whole_step_gbs": slot_bytes / (t_max / K / 1e3) / 1e9,
                         "pattern": pat,
                         "recur_frac_of_pattern_ceiling":
                             rec_gbs / pat["ceiling_gbs"] if pat else None},
        "phases_ms": per, "phase_share": shares, "plan": plan,
        "gpu_launches": int(sum(r[2]["launches_per_call"] for r in runs) * K),
        "clocks": clk, "e2e": e2e,
    }
    return out, lists


# ---------------------------------------------------------------- reference arm
def run_reference(args, cfg):
    """The oracle on the host cores, each step a bounded sample of the workload."""
    import oracle
    from synth import gen_inputs

    budget = 150.0 / max(1, args.steps + args.warmup)   # seconds per step
    nthr = host_threads()
    nheads = min(cfg.BH, nthr)
    sub = cfg.with_(B=1, H=1)
    one = gen_inputs(sub, t_end=16)
    npi = {k: v.numpy() for k, v in one.items()}
    t = time.perf_counter()
    oracle.forward(npi, dict(cfg.dims(), B=1, H=1, T=16))
    per_step = (time.perf_counter() - t) / 16
    T_s = int(max(8, min(cfg.T, budget / max(per_step, 1e-9))))
    heads = list(range(nheads))
    Bs = cfg.with_(B=(nheads - 1) // cfg.H + 1)
    inp = gen_inputs(Bs, t_end=T_s)
    npi = {k: v.numpy() for k, v in inp.items()}
    dd = dict(Bs.dims(), T=T_s)
    for _ in range(args.warmup):
        oracle.forward(npi, dd, heads=heads, nthreads=nthr)
    tot = 0.0
    for _ in range(args.steps):
        t = time.perf_counter()
        oracle.forward(npi, dd, heads=heads, nthreads=nthr)
        tot += time.perf_counter() - t
    th = nheads * T_s * args.steps
    value = th / tot
    sample = "%d heads x first %d steps of %s per step (oracle C, float64, %d threads)" % (
        nheads, T_s, cfg.name, min(nthr, nheads))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(cfg), "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(nthr, nheads),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def probe_rows(configs=None):
    """Random whole-row gathers / read-modify-writes on a 2 GiB table (the size of
    the pages-scale slot tables), timed with CUDA events after a warm-up launch."""
    import torch
    from sparse_memory_linear_scoring_b200.probe import probe_random_rows
    nrows = 8 << 20
    table = torch.zeros(nrows, 64, dtype=torch.float32, device="cuda")
    res = []
    if configs is None:
        configs = [(ctas, rmw, u) for ctas in (296, 444, 592) for rmw in (False, True)
                   for u in (4, 8)]
    for ctas, rmw, u in configs:
        if True:
            if True:
                iters = 64
                probe_random_rows(table, rmw=rmw, rows_in_flight=u, ctas=ctas, iters=4)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                probe_random_rows(table, rmw=rmw, rows_in_flight=u, ctas=ctas, iters=iters)
                e1.record()
                e1.synchronize()
                ms = e0.elapsed_time(e1)
                nbytes = ctas * 32 * u * iters * 256 * (2 if rmw else 1)
                res.append({"pattern": "rmw" if rmw else "gather", "rows_in_flight": u,
                            "ctas": ctas, "ms": ms, "GB/s": nbytes / ms / 1e6})
    del table
    pk, src = peaks()
    best = {pat: max(r["GB/s"] for r in res if r["pattern"] == pat) for pat in ("gather", "rmw")}
    return {"probe": "random 256-byte rows of a 2 GiB float32 table", "results": res,
            "best_GB/s": best, "copy_peak_GB/s": pk["hbm_gbs"], "peak_source": src}


def pattern_ceiling(W, R):
    """The HBM ceiling of the recurrence's own access pattern: 2W of every
    (2W + R) rows are read-modify-writes, R are gathers (best of a few launch
    shapes of the random-row probe, measured in the same run)."""
    pr = probe_rows([(592, False, 8), (296, False, 8), (592, True, 4), (296, True, 8)])
    g, m = pr["best_GB/s"]["gather"], pr["best_GB/s"]["rmw"]
    f = 2.0 * W / (2.0 * W + R)
    return {"gather_gbs": g, "rmw_gbs": m, "rmw_fraction": f,
            "ceiling_gbs": 1.0 / (f / m + (1.0 - f) / g)}


def decode(cfg, steps):
    """Streaming use, M carried from call to call, on the workload's B x H heads:
    one sdm_step call per step (the fused single-step kernel) and, for
    comparison, one sdm_forward call per step (T = 1); each eager and as one
    CUDA graph of all steps."""
    import torch
    import sparse_memory_linear_scoring_b200 as sdm
    from synth import gen_inputs
    inp = gen_inputs(cfg.with_(T=steps), device="cuda")
    dt = torch.bfloat16 if cfg.in_dtype == "bf16" else torch.float32
    per = {}
    for n in ("q", "k", "v", "alpha", "beta"):
        x = inp[n].to(dt) if n in ("q", "k", "v") else inp[n]
        x = x.unsqueeze(-1) if x.dim() == 3 else x          # [B, H, T, d]
        per[n] = x.permute(2, 0, 1, 3).contiguous().unsqueeze(3)  # [T, B, H, 1, d]
    C1, C2 = inp["C1"].to(dt).contiguous(), inp["C2"].to(dt).contiguous()
    M = inp["M0"].contiguous()
    dims = sdm.make_dims(**cfg.with_(T=1).dims())
    ws = torch.empty(sdm.workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    o = torch.empty(steps, cfg.B, cfg.H, 1, cfg.d_v, dtype=torch.float32, device="cuda")

    def one_forward(t):
        a = per["alpha"][t].squeeze(-1)
        b = per["beta"][t].squeeze(-1)
        sdm.forward(per["q"][t], per["k"][t], per["v"][t], a, b, C1, C2, M, topk=cfg.k,
                    W=cfg.W, R=cfg.R, o=o[t], workspace=ws)

    def one_step(t):
        a = per["alpha"][t].squeeze(-1)
        b = per["beta"][t].squeeze(-1)
        sdm.step(per["q"][t], per["k"][t], per["v"][t], a, b, C1, C2, M, topk=cfg.k,
                 W=cfg.W, R=cfg.R, o=o[t])

    def timed(one):
        for t in range(min(steps, 8)):
            one(t)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for t in range(steps):
            one(t)
        e1.record()
        e1.synchronize()
        eager_us = e0.elapsed_time(e1) * 1e3 / steps
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for t in range(steps):
                    one(t)
        torch.cuda.current_stream().wait_stream(s)
        g.replay()
        torch.cuda.synchronize()
        e0.record()
        g.replay()
        e1.record()
        e1.synchronize()
        graph_us = e0.elapsed_time(e1) * 1e3 / steps
        del g
        return {"eager_us_per_step": eager_us, "graph_us_per_step": graph_us,
                "graph_token_heads_per_s": cfg.BH / (graph_us * 1e-6)}

    clocks = ClockSampler(_device_uuid(torch, torch.device("cuda")))
    clocks.start()
    res = {"sdm_step": timed(one_step), "sdm_forward_T1": timed(one_forward)}
    clk = clocks.stop()
    st, info = sdm.device_status(ws)
    return {"decode": "one call per step, M carried", "workload": workload_desc(cfg),
            "steps": steps, "heads": cfg.BH, "kernels": res, "device_status": st,
            "clocks": clk}


def gdn_compare(cfg, steps, warmup):
    """The pages compare SDM with a dense Gated DeltaNet at matched FLOPs
    (W = R = the GDN query dimension): time sdm_gdn_forward at d_k = W with the
    workload's B, H, T, d_v and gates, and sdm_forward on the workload itself,
    in the same process (CUDA events, L2 flushed before each step)."""
    import torch
    import sparse_memory_linear_scoring_b200 as sdm
    from synth import gen_gdn_inputs, gen_inputs
    dt = torch.bfloat16 if cfg.in_dtype == "bf16" else torch.float32
    g = gen_gdn_inputs(cfg, device="cuda")
    g = {n: (v.to(dt) if n in ("q", "k", "v") else v).contiguous() for n, v in g.items()}
    ws = torch.empty(sdm.gdn_workspace_bytes(cfg.B, cfg.H, cfg.T, cfg.W, cfg.d_v, dt),
                     dtype=torch.uint8, device="cuda")
    og = torch.empty(cfg.B, cfg.H, cfg.T, cfg.d_v, dtype=torch.float32, device="cuda")
    S = g["S0"].clone()
    d = gen_inputs(cfg, device="cuda")
    d = {n: (v.to(dt) if n in ("q", "k", "v", "C1", "C2") else v).contiguous()
         for n, v in d.items()}
    M = d["M0"]
    osd = torch.empty(cfg.B, cfg.H, cfg.T, cfg.d_v, dtype=torch.float32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def time_it(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / steps

    clocks = ClockSampler(_device_uuid(torch, torch.device("cuda")))
    clocks.start()
    gdn_ms = time_it(lambda: sdm.gdn_forward(g["q"], g["k"], g["v"], g["alpha"], g["beta"], S,
                                             o=og, workspace=ws))
    sdm_ms = time_it(lambda: sdm.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["C1"],
                                         d["C2"], M, topk=cfg.k, W=cfg.W, R=cfg.R, o=osd))
    clk = clocks.stop()
    th = cfg.BH * cfg.T
    return {"baseline": "dense Gated DeltaNet (sdm_gdn_forward), matched d_k = W",
            "workload": workload_desc(cfg), "gdn": {"d_k": cfg.W, "d_v": cfg.d_v,
                                                    "ms_per_step": gdn_ms,
                                                    "token_heads_per_s": th / (gdn_ms / 1e3)},
            "sdm": {"ms_per_step": sdm_ms, "token_heads_per_s": th / (sdm_ms / 1e3)},
            "sdm_over_gdn_time": sdm_ms / gdn_ms,
            "pages": "SDM trains 1.49x slower than GDN at 8B (other hardware, training)",
            "steps": steps, "l2": "flushed before each step", "clocks": clk}


def backward_bench(cfg, steps, warmup):
    """sdm_backward on the workload (selections from sdm_select, random dL/do and
    dL/dM_T), timed with CUDA events beside sdm_forward in the same process
    (L2 flushed before each step)."""
    import ctypes
    import torch
    import sparse_memory_linear_scoring_b200 as sdm
    from synth import gen_inputs
    dt = torch.bfloat16 if cfg.in_dtype == "bf16" else torch.float32
    d = gen_inputs(cfg, device="cuda")
    d = {n: (v.to(dt) if n in ("q", "k", "v", "C1", "C2") else v).contiguous()
         for n, v in d.items()}
    M0 = d["M0"]
    lists = sdm.select(d["q"], d["k"], d["C1"], d["C2"], topk=cfg.k, W=cfg.W, R=cfg.R,
                       d_v=cfg.d_v)
    g = torch.Generator(device="cuda").manual_seed(0)
    d_o = torch.randn(cfg.B, cfg.H, cfg.T, cfg.d_v, device="cuda", generator=g)
    dM = torch.randn(M0.shape, device="cuda", generator=g)
    dims = sdm.make_dims(**cfg.dims())
    ws = torch.empty(int(sdm.load_library().sdm_backward_workspace_bytes(ctypes.byref(dims))),
                     dtype=torch.uint8, device="cuda")
    M = M0.clone()
    o = torch.empty_like(d_o)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def time_it(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / steps

    clocks = ClockSampler(_device_uuid(torch, torch.device("cuda")))
    clocks.start()
    bwd_ms = time_it(lambda: sdm.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                                          d["C1"], d["C2"], M0, *lists, d_o, dM, topk=cfg.k,
                                          workspace=ws))
    # dL/dM_0 accumulated in dM_T's buffer (its values change from step to step,
    # which does not change the work)
    inpl_ms = time_it(lambda: sdm.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                                           d["C1"], d["C2"], M0, *lists, d_o, dM, topk=cfg.k,
                                           workspace=ws, dM_T_inplace=True))
    fwd_ms = time_it(lambda: sdm.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["C1"],
                                         d["C2"], M, topk=cfg.k, W=cfg.W, R=cfg.R, o=o))
    clk = clocks.stop()
    th = cfg.BH * cfg.T
    return {"backward": "sdm_backward at the forward's selections (gradients of q, k, v, "
                        "alpha, beta, C1, C2, M0)",
            "workload": workload_desc(cfg), "backward_ms": bwd_ms,
            "backward_dM_in_place_ms": inpl_ms,
            "backward_token_heads_per_s": th / (bwd_ms / 1e3), "forward_ms": fwd_ms,
            "backward_over_forward_time": bwd_ms / fwd_ms, "workspace_bytes": ws.numel(),
            "steps": steps, "l2": "flushed before each step", "clocks": clk,
            "device_status": sdm.device_status(ws)[0]}


def main():
    args = parse()
    if args.decode:
        from synth import config as _config
        print(json.dumps(decode(_config(args.config), max(16, args.steps))), flush=True)
        return 0
    if args.probe_rows:
        print(json.dumps(probe_rows()), flush=True)
        return 0
    if args.backward:
        from synth import config as _config
        cfg = _config(args.config)
        if args.T > 0:
            cfg = cfg.with_(T=args.T)
        print(json.dumps(backward_bench(cfg, max(3, min(args.steps, 50)), max(2, args.warmup))),
              flush=True)
        return 0
    if args.gdn:
        from synth import config as _config
        print(json.dumps(gdn_compare(_config(args.config), max(3, min(args.steps, 200)),
                                     max(3, args.warmup))), flush=True)
        return 0
    from synth import config
    cfg = config(args.config)
    if args.T > 0:
        cfg = cfg.with_(T=args.T)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, cfg)), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    out, lists = run_sdm(args, cfg, rank, world, local_rank)
    if rank == 0:
        if not args.no_cpu_baseline:
            out["cpu_baseline"], sample = cpu_baseline(cfg, args.cpu_seconds)
            if lists is not None:
                out["parity_sample"] = parity_sample(lists, sample)
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
