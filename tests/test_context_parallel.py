"""Context parallelism, host side (CPU): the page-aligned split of a
sequence's tokens over ranks, and the exchange of per-rank parts over a
gloo process group, merged with the oracle's log-sum-exp combine, against the
oracle's attention over the whole sequence."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from mla_latent_kv_35_b200.context_parallel import gather_parts, token_ranges  # noqa: E402


@pytest.mark.parametrize("L,world", [(0, 3), (1, 2), (64, 2), (65, 2), (1000, 3), (130, 5),
                                     (131072, 8), (200, 1)])
def test_token_ranges_partition_the_sequence(L, world):
    rs = token_ranges(L, world)
    assert len(rs) == world
    pos = 0
    for first, n, tail in rs:
        assert n >= 0 and first == pos and first + n + tail == L
        if n and first + n < L:
            assert (first + n) % 64 == 0          # whole pages except the last range
        assert first % 64 == 0 or n == 0
        pos += n
    assert pos == L


def _problem(seed, S_q=2, H=3, L=300, d_c=8, d_r=4):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((S_q, H, d_c + d_r)), rng.standard_normal((L, d_c)),
            rng.standard_normal((L, d_r)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, L, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, C, KR = _problem(5, L=L)
        first, n, _ = token_ranges(L, world, page_size=16)[rank]
        part = oracle.latent_attention_range(q, C[first:first + n], KR[first:first + n], 0.3,
                                             first, L)
        o_parts, l_parts = gather_parts(torch.from_numpy(part["o_lat"]),
                                        torch.from_numpy(part["lse"]))
        o, lse = oracle.combine_splits(o_parts.numpy(), l_parts.numpy())
        out[rank] = (o, lse)
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L", [(2, 300), (3, 33)])
def test_parts_exchanged_over_gloo_merge_to_full_attention(world, L):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, L, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0] * world, codes
    q, C, KR = _problem(5, L=L)
    full = oracle.latent_attention(q, C, KR, 0.3)
    for r in range(world):
        np.testing.assert_allclose(res[r][0], full["o_lat"], atol=1e-12)
        np.testing.assert_allclose(res[r][1], full["lse"], atol=1e-12)
