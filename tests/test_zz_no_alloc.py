"""The allocation-free decode entry point against the regular one.

mla_decode_noalloc serves callers that cannot allocate device memory (their
host framework owns all device memory, or their loop must not call
cudaMalloc/cudaFree, which can synchronise the device).  It keeps its
workspace in a fixed array inside the library.  These tests call it through
the C ABI twice in a row and compare each result with mla_decode run on a
caller-provided workspace, at the tolerance the decode parity tests use, and
check that oversized problems are refused before anything is launched.
This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from mla_latent_kv_35_b200 import binding as B
from mla_latent_kv_35_b200 import workloads as wl
from gpu_util import DEV, check, dims, ensure_lib, q, to_dev, to_np

gpu = pytest.mark.gpu


def _case(lens, S_q, H=128, seed=21):
    rng = np.random.default_rng(seed)
    d = dims("bf16", H=H)
    P, D = d.page_size, d.d_latent + d.d_rope
    npg = [-(-L // P) for L in lens]
    n_pages = sum(npg) + 1
    perm = rng.permutation(n_pages - 1).astype(np.int32)
    table = np.full((len(lens), max(npg)), -1, np.int32)
    o = 0
    for b, n in enumerate(npg):
        table[b, :n] = perm[o:o + n]
        o += n
    pool = np.full((n_pages, P, D), 0xFFFF, np.uint16)
    for b, L in enumerate(lens):
        rows = wl.bf16_bits(rng.standard_normal((L, D)).astype(np.float32))
        for t in range(L):
            pool[table[b, t // P], t % P] = rows[t]
    qb = q(rng.standard_normal((len(lens), S_q, H, D)), "bf16")
    return d, dict(qb=to_dev(qb, "bf16"),
                   pool=torch.from_numpy(pool.view(np.int16)).to(DEV).view(torch.bfloat16),
                   n_pages=n_pages, table=torch.from_numpy(table).to(DEV),
                   maxp=table.shape[1], lens=torch.tensor(lens, dtype=torch.int32, device=DEV))


def _outs(n, S_q, H, dc=512):
    return (torch.full((n, S_q, H, dc), float("nan"), device=DEV),
            torch.full((n, S_q, H), float("nan"), device=DEV))


@gpu
@pytest.mark.parametrize("lens,S_q", [([300, 1000, 65, 4096], 1), ([130, 2000], 2)])
def test_noalloc_matches_regular_decode(lens, S_q):
    ensure_lib()
    B.mla_get_device_status()
    d, c = _case(lens, S_q)
    n = len(lens)
    ws = torch.empty((B.mla_decode_workspace_size(d, n, S_q, 0),), dtype=torch.uint8, device=DEV)
    o_ref, l_ref = _outs(n, S_q, d.n_heads)
    B.mla_decode(d, c["qb"], c["pool"], c["n_pages"], c["table"], c["maxp"], c["lens"], n, S_q,
                 0, ws, o_ref, l_ref)
    assert B.mla_get_device_status() == 0
    for call in range(2):                       # two calls in a row share the scratch
        o, l = _outs(n, S_q, d.n_heads)
        B.mla_decode_noalloc(d, c["qb"], c["pool"], c["n_pages"], c["table"], c["maxp"],
                             c["lens"], n, S_q, 0, o, l)
        assert B.mla_get_device_status() == 0
        check(to_np(o), to_np(o_ref), "bf16", f"noalloc call {call} o_lat")
        check(to_np(l), to_np(l_ref), "bf16", f"noalloc call {call} lse")


@gpu
def test_noalloc_refuses_oversized_problem():
    ensure_lib()
    d = dims("bf16")
    n = 2048                                    # workspace far above the 64 MiB scratch
    assert B.mla_decode_workspace_size(d, n, 1, 0) > B.mla_decode_noalloc_scratch_bytes()
    dummy = torch.zeros(16, device=DEV)
    with pytest.raises(B.MLAError) as e:
        B.mla_decode_noalloc(d, dummy, dummy, 1, dummy, 1, dummy, n, 1, 0, dummy, dummy)
    assert e.value.code == 2                    # MLA_ERR_UNSUPPORTED, nothing launched
    assert B.mla_get_device_status() == 0
