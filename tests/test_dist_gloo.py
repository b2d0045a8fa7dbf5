"""Multi-rank host logic on CPU with gloo (world size 2): seeds, shards, max-over-ranks
timing and the whole-job throughput that the benchmark reports."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from block_sparse_long_tcgen05_b200 import dist as mdist


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    w, r, _ = mdist.init("gloo", timeout_s=60)
    try:
        mdist.barrier()
        ms = 10.0 + 5.0 * r                       # rank 1 is the slow one
        ms_max = mdist.max_over_ranks(ms)
        seeds = [None] * w
        torch.distributed.all_gather_object(seeds, mdist.rank_seed(1002, r))
        groups, hs, gs = mdist.group_slice(8, 8, w, r)
        out[r] = (w, r, ms_max, seeds, list(mdist.shard(64, w, r)),
                  mdist.job_throughput(131072, w, ms_max), list(groups), (hs.start, hs.stop))
    finally:
        mdist.shutdown()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        w, rr, ms_max, seeds, shard, value, groups, heads = res[r]
        assert (w, rr) == (world, r)
        assert ms_max == 15.0                    # the slowest rank's time, on every rank
        assert len(set(seeds)) == world          # independent sequences
        assert value == pytest.approx(world * 131072 / 15e-3)
    assert res[0][4] + res[1][4] == list(range(64))     # shards cover the batch, disjoint
    assert res[0][6] + res[1][6] == list(range(8))      # group shards cover the groups, disjoint
    assert res[0][7] == (0, 32) and res[1][7] == (32, 64)   # and own exactly their groups' heads


def test_single_rank_defaults():
    assert mdist.max_over_ranks(3.5) == 3.5
    assert list(mdist.shard(10, 3, 0)) == [0, 1, 2, 3]
    assert list(mdist.shard(10, 3, 2)) == [7, 8, 9]
    assert mdist.rank_seed(1002, 0) == 1002


def test_group_shard_computes_the_same_heads():
    """The property group sharding relies on: the oracle run on one rank's groups (their
    index heads, query heads and k/v) gives exactly those heads of the full problem."""
    from block_sparse_long_tcgen05_b200 import synth
    from oracle import msa_oracle as orc
    cfg = synth.PrefillConfig("t", N=700, Hq=8, G=4, d=32, d_idx=16, k=3, idx_range=3, hot_frac=0.1, seed=5)
    inp = synth.prefill_inputs(cfg)
    rows = [0, 127, 128, 383, 500, 699]
    ids_full, o_full = orc.prefill_rows(inp, rows, cfg.Bk, cfg.k)
    world = 2
    for r in range(world):
        part = mdist.shard_inputs_by_group(inp, cfg.G, world, r)
        groups, hs, gs = mdist.group_slice(cfg.G, cfg.R, world, r)
        ids_p, o_p = orc.prefill_rows(part, rows, cfg.Bk, cfg.k)
        assert (ids_p == ids_full[:, gs]).all()
        assert (o_p == o_full[:, hs]).all()
