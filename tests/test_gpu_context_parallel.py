"""Context parallelism on the GPU: each rank's token range decoded with
mla_decode_partial and the parts merged with mla_combine_parts, against the
oracle's attention over the whole sequence and against mla_decode on the
whole cache.  Ranks are emulated on one GPU as per-rank page tables over one
pool (each rank's kernels finish before the next starts: nothing waits on
another rank); the exchange itself goes through a one-rank NCCL group."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch

from mla_latent_kv_35_b200 import binding as B
from mla_latent_kv_35_b200.context_parallel import decode_context_parallel, token_ranges
from gpu_util import DEV, check, ensure_lib, status, to_dev, to_np
from test_gpu_kernels import _decode_case, _decode_ref

gpu = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if torch.cuda.is_available():
        ensure_lib()
        B.mla_get_device_status()


def _rank_tables(c, lens, world):
    """Per emulated rank: local page table, local lengths and tails."""
    out = []
    for r in range(world):
        tab = np.full_like(c["table"], -1)
        n_loc = np.zeros(len(lens), np.int32)
        tail = np.zeros(len(lens), np.int32)
        for b, L in enumerate(lens):
            first, n, t = token_ranges(L, world)[r]
            pages = -(-n // 64)
            tab[b, :pages] = c["table"][b, first // 64:first // 64 + pages]
            n_loc[b], tail[b] = n, t
        out.append((tab, n_loc, tail))
    return out


def _partials(d, c, lens, S_q, world):
    Bn, H, dc = len(lens), d.n_heads, d.d_latent
    o_parts = torch.empty((world, Bn, S_q, H, dc), device=DEV)
    l_parts = torch.empty((world, Bn, S_q, H), device=DEV)
    ws = torch.empty((B.mla_decode_workspace_size(d, Bn, S_q, 0),), dtype=torch.uint8, device=DEV)
    qb = to_dev(c["qb"], d.dtype)
    for r, (tab, n_loc, tail) in enumerate(_rank_tables(c, lens, world)):
        B.mla_decode_partial(d, qb, c["pool_d"], c["n_pages"], torch.from_numpy(tab).to(DEV),
                             c["maxp"], torch.from_numpy(n_loc).to(DEV),
                             torch.from_numpy(tail).to(DEV), Bn, S_q, 0, ws, o_parts[r],
                             l_parts[r])
    assert status() == 0
    return o_parts, l_parts


@gpu
@pytest.mark.parametrize("dtype,H,S_q,lens,world", [
    ("bf16", 128, 2, [3000, 130], 3),
    ("bf16", 128, 1, [5000, 64, 200], 2),
    ("bf16", 128, 2, [129, 65], 5),        # empty ranks; last rank holds a single query token
    ("f32", 8, 2, [300, 65], 3),
])
def test_partials_merge_to_whole_sequence(dtype, H, S_q, lens, world):
    dc, dr = (64, 16) if dtype == "f32" else (512, 64)
    d, c = _decode_case(dtype, H, lens, S_q, seed=21, dc=dc, dr=dr)
    o_parts, l_parts = _partials(d, c, lens, S_q, world)
    rows = len(lens) * S_q * H
    o = torch.empty((len(lens), S_q, H, dc), device=DEV)
    lse = torch.empty((len(lens), S_q, H), device=DEV)
    B.mla_combine_parts(d, o_parts, l_parts, world, rows, o, lse)
    assert status() == 0
    o_np, l_np = to_np(o), to_np(lse)
    for b in range(len(lens)):
        ref = _decode_ref(d, c, b)
        check(o_np[b], ref["o_lat"], dtype, f"o_lat b={b}")
        check(l_np[b], ref["lse"], dtype, f"lse b={b}")


@gpu
def test_partial_with_zero_tail_is_decode():
    lens, S_q = [700, 129], 2
    d, c = _decode_case("bf16", 128, lens, S_q, seed=22)
    Bn = len(lens)
    ws = torch.empty((B.mla_decode_workspace_size(d, Bn, S_q, 0),), dtype=torch.uint8, device=DEV)
    outs = []
    for partial in (False, True):
        o = torch.empty((Bn, S_q, 128, 512), device=DEV)
        lse = torch.empty((Bn, S_q, 128), device=DEV)
        args = (d, to_dev(c["qb"], "bf16"), c["pool_d"], c["n_pages"],
                torch.from_numpy(c["table"]).to(DEV), c["maxp"],
                torch.from_numpy(c["lens"]).to(DEV))
        if partial:
            B.mla_decode_partial(*args, torch.zeros(Bn, dtype=torch.int32, device=DEV), Bn, S_q,
                                 0, ws, o, lse)
        else:
            B.mla_decode(*args, Bn, S_q, 0, ws, o, lse)
        outs.append((o, lse))
    assert status() == 0
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@gpu
def test_decode_context_parallel_through_nccl_one_rank():
    """The product call (partial decode, NCCL all-gather, merge) in a one-rank
    group: the merge of a single part is that part."""
    import torch.distributed as dist
    lens, S_q = [2000, 300], 1
    d, c = _decode_case("bf16", 128, lens, S_q, seed=23)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        Bn = len(lens)
        ws = torch.empty((B.mla_decode_workspace_size(d, Bn, S_q, 0),), dtype=torch.uint8,
                         device=DEV)
        o = torch.empty((Bn, S_q, 128, 512), device=DEV)
        lse = torch.empty((Bn, S_q, 128), device=DEV)
        decode_context_parallel(d, to_dev(c["qb"], "bf16"), c["pool_d"], c["n_pages"],
                                torch.from_numpy(c["table"]).to(DEV), c["maxp"],
                                torch.from_numpy(c["lens"]).to(DEV),
                                torch.zeros(Bn, dtype=torch.int32, device=DEV), Bn, S_q, ws, o,
                                lse)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert status() == 0
    for b in range(Bn):
        ref = _decode_ref(d, c, b)
        check(to_np(o)[b], ref["o_lat"], "bf16", f"o_lat b={b}")
        check(to_np(lse)[b], ref["lse"], "bf16", f"lse b={b}")


@gpu
def test_full_size_context_over_eight_ranks():
    """Two 131072-token sequences (two speculative query tokens) split over 8
    emulated ranks, merged, against mla_decode on the whole cache."""
    rng = torch.Generator(device="cpu").manual_seed(31)
    d = B.MLADims(128, 128, 512, 64, 128, 5120, 64, 192 ** -0.5, 10000.0, "bf16")
    lens, S_q, world, Bn = [131072, 131071], 2, 8, 2
    maxp = 131072 // 64
    n_pages = Bn * maxp + 1
    perm = torch.randperm(Bn * maxp, generator=rng).to(torch.int32).reshape(Bn, maxp)
    pool = torch.randn((n_pages, 64, 576), generator=rng).to(DEV, torch.bfloat16)
    qb = torch.randn((Bn, S_q, 128, 576), generator=rng).to(DEV, torch.bfloat16)
    table = perm.numpy()
    c = {"table": table, "qb": None, "pool_d": pool, "n_pages": n_pages, "maxp": maxp}
    ws = torch.empty((B.mla_decode_workspace_size(d, Bn, S_q, 0),), dtype=torch.uint8, device=DEV)
    o_parts = torch.empty((world, Bn, S_q, 128, 512), device=DEV)
    l_parts = torch.empty((world, Bn, S_q, 128), device=DEV)
    for r, (tab, n_loc, tail) in enumerate(_rank_tables(c, lens, world)):
        B.mla_decode_partial(d, qb, pool, n_pages, torch.from_numpy(tab).to(DEV), maxp,
                             torch.from_numpy(n_loc).to(DEV), torch.from_numpy(tail).to(DEV),
                             Bn, S_q, 0, ws, o_parts[r], l_parts[r])
    o = torch.empty((Bn, S_q, 128, 512), device=DEV)
    lse = torch.empty((Bn, S_q, 128), device=DEV)
    B.mla_combine_parts(d, o_parts, l_parts, world, Bn * S_q * 128, o, lse)
    o_full = torch.empty_like(o)
    l_full = torch.empty_like(lse)
    B.mla_decode(d, qb, pool, n_pages, torch.from_numpy(table).to(DEV), maxp,
                 torch.tensor(lens, dtype=torch.int32, device=DEV), Bn, S_q, 0, ws, o_full, l_full)
    assert status() == 0
    # both are bf16-P decodes of the same data with different splits
    check(to_np(o), to_np(o_full).astype(np.float64), "bf16", "o_lat vs whole-cache decode")
    check(to_np(lse), to_np(l_full).astype(np.float64), "bf16", "lse vs whole-cache decode")
