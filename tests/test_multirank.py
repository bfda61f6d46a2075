"""The multi-rank path on CPU with gloo (world size 2): heads sharded across
ranks with no data-path exchange must reproduce the single-process result
exactly (computed here with the CPU oracle), and the timing reduction must take
the max over ranks."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_memory_linear_scoring_b200.parallel import gather_batch, max_over_ranks, shard_batch
from synth import config, gen_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, B_global, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = config(0).with_(B=B_global, H=2, T=48, m0_sd=0.3)
        b0, nb = shard_batch(B_global, world, rank)
        local = cfg.with_(B=nb)
        inp = gen_inputs(local, b0=b0)
        res = oracle.forward({k: v.numpy() for k, v in inp.items()}, local.dims())
        o = gather_batch(torch.from_numpy(res["o"]), B_global)
        M = gather_batch(torch.from_numpy(res["M"]), B_global)
        t = max_over_ranks(float(rank + 1))
        if rank == 0:
            torch.save({"o": o, "M": M, "tmax": t}, os.path.join(out_dir, "gathered.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B_global", [2, 3])
def test_sharded_heads_match_single_process(B_global):
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), B_global, d), nprocs=world,
                           join=True, start_method="spawn")
        got = torch.load(os.path.join(d, "gathered.pt"))
    cfg = config(0).with_(B=B_global, H=2, T=48, m0_sd=0.3)
    inp = gen_inputs(cfg)
    ref = oracle.forward({k: v.numpy() for k, v in inp.items()}, cfg.dims())
    assert np.array_equal(got["o"].numpy(), ref["o"])
    assert np.array_equal(got["M"].numpy(), ref["M"])
    assert got["tmax"] == 2.0


def test_shard_batch_covers_once():
    for B in range(1, 20):
        for world in range(1, 6):
            rows = []
            for r in range(world):
                b0, nb = shard_batch(B, world, r)
                rows += list(range(b0, b0 + nb))
            assert rows == list(range(B))


def test_generator_shards_are_slices():
    cfg = config(0).with_(B=3, H=2, T=20)
    full = gen_inputs(cfg)
    part = gen_inputs(cfg.with_(B=1), b0=2)
    for name in ("q", "k", "v", "alpha", "beta", "M0"):
        assert torch.equal(full[name][2:3], part[name])
    assert torch.equal(full["C1"], part["C1"])
