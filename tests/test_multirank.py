"""The multi-rank path on CPU with gloo (world size 2): (b,h) heads sharded
across ranks as contiguous flat-head ranges, run per rank as the rectangular
pieces the product calls, with no data-path exchange, must reproduce the
single-process result exactly (computed here with the CPU oracle), and the
timing reduction must take the max over ranks."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_memory_linear_scoring_b200.parallel import (gather_heads, head_pieces,
                                                         max_over_ranks, shard_heads)
from synth import config, gen_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg(B, H):
    return config(0).with_(B=B, H=H, T=48, m0_sd=0.3)


def _worker(rank, world, port, B, H, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = _cfg(B, H)
        f0, n = shard_heads(B * H, world, rank)
        os_, Ms = [], []
        # one call per piece, each on that piece's own inputs (a rectangle of
        # the head grid, generated on its own), as a rank of the product runs
        for pc in head_pieces(f0, n, H):
            local = cfg.with_(B=pc.b1 - pc.b0, H=pc.h1 - pc.h0)
            inp = gen_inputs(cfg.with_(B=pc.b1 - pc.b0), b0=pc.b0, h0=pc.h0, h1=pc.h1)
            res = oracle.forward({k: v.numpy() for k, v in inp.items()}, local.dims())
            os_.append(torch.from_numpy(res["o"]).reshape(-1, *res["o"].shape[2:]))
            Ms.append(torch.from_numpy(res["M"]).reshape(-1, *res["M"].shape[2:]))
        o_loc = torch.cat(os_) if os_ else torch.zeros(0, cfg.T, cfg.d_v)
        M_loc = torch.cat(Ms) if Ms else torch.zeros(0, cfg.N, cfg.d_v)
        o = gather_heads(o_loc, B * H)
        M = gather_heads(M_loc, B * H)
        t = max_over_ranks(float(rank + 1))
        if rank == 0:
            torch.save({"o": o, "M": M, "tmax": t}, os.path.join(out_dir, "gathered.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B,H", [(2, 2), (3, 3), (1, 5)],
                         ids=["aligned", "crosses-a-batch-row", "single-batch-row"])
def test_sharded_heads_match_single_process(B, H):
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), B, H, d), nprocs=world,
                           join=True, start_method="spawn")
        got = torch.load(os.path.join(d, "gathered.pt"))
    cfg = _cfg(B, H)
    inp = gen_inputs(cfg)
    ref = oracle.forward({k: v.numpy() for k, v in inp.items()}, cfg.dims())
    assert np.array_equal(got["o"].numpy(), ref["o"].reshape(B * H, cfg.T, cfg.d_v))
    assert np.array_equal(got["M"].numpy(), ref["M"].reshape(B * H, cfg.N, cfg.d_v))
    assert got["tmax"] == 2.0


def test_shard_heads_cover_once():
    for BH in range(0, 30):
        for world in range(1, 9):
            heads = []
            for r in range(world):
                f0, n = shard_heads(BH, world, r)
                heads += list(range(f0, f0 + n))
            assert heads == list(range(BH))


def test_head_pieces_are_contiguous_rectangles():
    """Pieces cover the range once, in flat order, and each piece's slice of a
    [B][H] tensor is contiguous (one library call on plain pointers)."""
    for B in range(1, 5):
        for H in range(1, 6):
            grid = torch.arange(B * H).view(B, H)
            for f0 in range(B * H + 1):
                for n in range(B * H - f0 + 1):
                    pcs = head_pieces(f0, n, H)
                    assert len(pcs) <= 3
                    flat = []
                    for pc in pcs:
                        sl = grid[pc.b0:pc.b1, pc.h0:pc.h1]
                        assert sl.is_contiguous() or sl.numel() <= 1 or pc.b1 - pc.b0 == 1
                        assert pc.b1 - pc.b0 == 1 or (pc.h0 == 0 and pc.h1 == H)
                        flat += sl.reshape(-1).tolist()
                    assert flat == list(range(f0, f0 + n))


def test_generator_pieces_are_slices():
    cfg = config(0).with_(B=3, H=4, T=20)
    full = gen_inputs(cfg)
    part = gen_inputs(cfg.with_(B=1), b0=2, h0=1, h1=3)
    for name in ("q", "k", "v", "alpha", "beta", "M0"):
        assert torch.equal(full[name][2:3, 1:3], part[name])
    assert torch.equal(full["C1"][1:3], part["C1"])
