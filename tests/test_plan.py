"""How the library lays out a call (sdm_query_plan, sdm_workspace_bytes): host
logic only, no GPU.  Checks the invariants the kernels rely on: plan blocks
fit the entry-index field, buckets are split evenly over the streams, time
chunks cover the sequence, head groups bound the table span of a launch, and
the scratch stays within its budget."""
import itertools

import pytest

import sparse_memory_linear_scoring_b200 as sdm
from sparse_memory_linear_scoring_b200 import build as sdm_build
from synth import CONFIGS

GROUP_BYTES = 8 << 30
MAX_ENTRIES = 8192


@pytest.fixture(scope="module", autouse=True)
def _lib():
    sdm_build.build()
    sdm.load_library()


SHAPES = [dict(c.dims()) for c in CONFIGS] + [
    dict(B=1, H=1, T=1, d_qk=128, d_v=64, n_sub=1024, k=64, W=64, R=64, in_dtype=1),
    dict(B=3, H=5, T=777, d_qk=64, d_v=32, n_sub=100, k=10, W=30, R=7, in_dtype=0),
    dict(B=2, H=2, T=5000, d_qk=32, d_v=4, n_sub=16, k=16, W=256, R=256, in_dtype=0),
    dict(B=128, H=16, T=64, d_qk=128, d_v=128, n_sub=512, k=64, W=64, R=64, in_dtype=1),
]


@pytest.mark.parametrize("dims", SHAPES, ids=lambda d: "B%dH%dT%dn%d" % (d["B"], d["H"], d["T"], d["n_sub"]))
def test_plan_invariants(dims):
    d = sdm.make_dims(**dims)
    plan = sdm.query_plan(d)
    P, S, NB = plan["block_steps"], plan["streams_per_head"], plan["buckets_per_head"]
    Tc, nch = plan["chunk_steps"], plan["chunks"]
    WR = dims["W"] + dims["R"]
    assert 1 <= P <= 1024 and P * WR <= MAX_ENTRIES
    assert P <= max(1, dims["T"])
    assert S >= 1 and NB >= S and NB % S == 0          # each stream owns NB / S buckets
    assert S <= max(1, P * WR // 4)                     # at least 4 records per stream and block
    assert Tc % P == 0 and Tc * nch >= dims["T"] and Tc * (nch - 1) < dims["T"]
    assert plan["survivor_capacity"] >= dims["k"]
    ws = sdm.workspace_bytes(d)
    assert 0 < ws < (9 << 29)


@pytest.mark.parametrize("dims", SHAPES, ids=lambda d: "B%dH%dT%dn%d" % (d["B"], d["H"], d["T"], d["n_sub"]))
def test_launch_count(dims):
    """Per chunk: scoring (tensor cores: filter + exact fallback, plus a reset of
    the fallback list after the first chunk, plus the survivor top-k in the
    filter-only mode; else one kernel), merge, plan, and one recurrence launch
    per head group; one status reset per call."""
    plan = sdm.query_plan(sdm.make_dims(**dims))
    BH = dims["B"] * dims["H"]
    table = dims["n_sub"] ** 2 * dims["d_v"] * 4
    HG = max(1, min(BH, GROUP_BYTES // table))
    groups = -(-BH // HG)
    tc, nch = plan["tensor_core_scoring"], plan["chunks"]
    mode = plan["scoring_mode"]
    assert (mode > 0) == (tc == 1)
    per_chunk = (4 if mode == 2 else 3 if tc else 1) + 2 + groups
    assert plan["launches_per_call"] == 1 + per_chunk * nch - (1 if tc and nch else 0)


def test_workspace_grows_with_steps_until_chunked():
    base = CONFIGS[2].dims()
    sizes = [sdm.workspace_bytes(sdm.make_dims(**dict(base, T=T))) for T in (1, 64, 1024, 8192)]
    assert sizes == sorted(sizes)
    big = sdm.workspace_bytes(sdm.make_dims(**dict(base, T=1 << 20)))
    assert big < (9 << 29)                              # long sequences run as chunks
    plan = sdm.query_plan(sdm.make_dims(**dict(base, T=1 << 20)))
    assert plan["chunks"] > 1


def test_head_groups_bound_the_table_span():
    """The high-batch workload (1024 heads of 64 MiB tables) runs its recurrence
    in groups of at most 8 GiB of tables."""
    dims = CONFIGS[4].dims()
    plan = sdm.query_plan(sdm.make_dims(**dims))
    BH = dims["B"] * dims["H"]
    table = dims["n_sub"] ** 2 * dims["d_v"] * 4
    assert plan["tensor_core_scoring"] == 1
    # launches = chunks * (3 scoring + merge + plan + groups): see test_launch_count
    groups = plan["launches_per_call"] // plan["chunks"] - 5
    assert groups * (GROUP_BYTES // table) >= BH
    assert (GROUP_BYTES // table) * table <= GROUP_BYTES


def test_scoring_choice_does_not_depend_on_T():
    """The scoring kernel follows the shape only, so a sequence split into calls
    reproduces one call's state bit for bit."""
    base = CONFIGS[2].dims()
    choices = {sdm.query_plan(sdm.make_dims(**dict(base, T=T)))["tensor_core_scoring"]
               for T in (1, 2, 31, 32, 127, 128, 8192)}
    assert len(choices) == 1
