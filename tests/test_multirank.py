"""Multi-rank host logic on CPU (gloo, world size 2).

Decode sequences are independent, so N GPUs run N shards of one batch with no
data-path collective (weak scaling).  What needs checking without GPUs:
each rank draws its own global sequences, the shards tile the whole batch,
the timing reduction takes the slowest rank, and a rank that leaves makes the
others' next collective end with an error instead of waiting for good.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from mla_latent_kv_35_b200 import workloads as wl  # noqa: E402


def _small(name):
    w = wl.workload(name)
    if name == "ragged":
        return w
    return wl.workload(name, B=4, ctx=(300,) * 4)


@pytest.mark.parametrize("name", ["dsv2", "ragged"])
def test_shard_zero_of_one_is_identity(name):
    w = _small(name)
    assert wl.shard(w, 0, 1) is w


@pytest.mark.parametrize("name", ["dsv2", "ragged"])
def test_rank0_shard_matches_unsharded_batch(name):
    w = _small(name)
    s0 = wl.shard(w, 0, 3)
    assert s0.ctx == w.ctx
    np.testing.assert_array_equal(wl.draw_h_new(s0), wl.draw_h_new(w))
    for b in (0, w.B - 1):
        for x, y in zip(wl.draw_prior(s0, b), wl.draw_prior(w, b)):
            np.testing.assert_array_equal(x, y)
    np.testing.assert_array_equal(wl.page_layout(s0)[0], wl.page_layout(w)[0])


def test_shards_tile_the_global_batch():
    """Rank r's sequence b is sequence r*B + b of the batch grown to world*B."""
    w = _small("dsv2")
    world = 3
    whole = wl.workload("dsv2", B=w.B * world, ctx=w.ctx * world)
    h_all = wl.draw_h_new(whole)
    for r in range(world):
        s = wl.shard(w, r, world)
        np.testing.assert_array_equal(wl.draw_h_new(s), h_all[r * w.B:(r + 1) * w.B])
        c, kr = wl.draw_prior(s, 1)
        c2, kr2 = wl.draw_prior(whole, r * w.B + 1)
        np.testing.assert_array_equal(c, c2)
        np.testing.assert_array_equal(kr, kr2)


def test_ragged_shards_take_their_slice_of_the_lengths():
    w = wl.workload("ragged")
    world = 2
    s1 = wl.shard(w, 1, world)
    whole = wl._ragged_lengths(w.B * world, 7)
    assert s1.ctx == tuple(L + 1 for L in whole[w.B:])
    assert s1.ctx != w.ctx
    table, n_pages = wl.page_layout(s1)
    used = table[table >= 0]
    assert len(np.unique(used)) == used.size == n_pages - 1


def test_shard_rejects_bad_rank():
    with pytest.raises(ValueError):
        wl.shard(_small("dsv2"), 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        w = wl.shard(_small("dsv2"), rank, world)
        # per-rank "times": the reduction must return the slowest rank's
        t = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.5 * rank])
        # every rank's sequences: gather a digest of its new hidden states
        import torch
        dig = torch.tensor([float(np.abs(wl.draw_h_new(w)).sum())], dtype=torch.float64)
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, dig)
        out[rank] = (t, [float(g) for g in gathered],
                     bench.whole_job_rate(w.T, world, max(t[0], 1e-9)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_gloo_reduction_and_sharding():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 0], codes
    for r in range(world):
        t, digests, rate = res[r]
        assert t == [2.0, 5.0, 0.5]
        assert digests[0] != digests[1]
        # 4 tokens per rank, 2 ranks, slowest rank 2 ms
        assert rate == pytest.approx(4 * 2 / 2e-3)
    assert res[0][1] == res[1][1]


def _failing_rank_main(rank, world, port, out):
    import datetime
    import time
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    import bench
    if rank == 1:
        # this rank fails between steps and never reaches the collective
        out[rank] = "left"
        time.sleep(8)
        os._exit(3)
    t0 = time.time()
    try:
        bench.max_over_ranks([1.0])
        out[rank] = "returned"
    except Exception as e:  # the collective must end with an error, not hang
        out[rank] = ("error", type(e).__name__, time.time() - t0)
    os._exit(0)


def test_rank_that_leaves_ends_the_others_collective_with_an_error():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_failing_rank_main, args=(r, world, port, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(60)
        alive = [p.is_alive() for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        res = dict(out)
    assert alive == [False, False]
    assert res[1] == "left"
    assert res[0][0] == "error" and res[0][2] < 30, res[0]
