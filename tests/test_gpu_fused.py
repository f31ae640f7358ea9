"""The fused pre-attention call and the CUDA-graph step against the separate
calls they replace, bit for bit.

mla_pre_attention must leave qbuf, the paged pool and the projection rows
exactly as mla_rope (q), mla_rope (k, in place), mla_cache_append and
mla_absorb_q do; those calls are themselves checked against the oracle in
test_gpu_kernels.py.  A replayed CUDA graph of the whole step must give the
eager step's bits up to the decode output, and its output projection to
within the reordering of atomic split-K sums.
"""

import numpy as np
import pytest
import torch

from mla_latent_kv_35_b200 import binding as B
from mla_latent_kv_35_b200 import workloads as wl
from mla_latent_kv_35_b200.engine import MLADecodeLayer, build_pool_host_drawn, pool_to_device
from gpu_util import DEV, dims, ensure_lib, status

gpu = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if torch.cuda.is_available():
        ensure_lib()
        B.mla_get_device_status()


def _case(dtype, T, n_seq, seed):
    rng = np.random.default_rng(seed)
    if dtype == "bf16":
        d = dims("bf16", H=128)
    else:
        d = dims("f32", H=8, dn=32, dc=64, dr=16, dm=256)
    H, dn, dc, dr = d.n_heads, d.d_nope, d.d_latent, d.d_rope
    Y = H * (dn + dr) + dc + dr
    tdt = d.torch_dtype
    y = torch.from_numpy(rng.standard_normal((T, Y)).astype(np.float32)).to(DEV, tdt)
    w_uk = torch.from_numpy((rng.standard_normal((H, dn, dc)) / np.sqrt(dc)).astype(np.float32))
    w_uk = w_uk.to(DEV, tdt)
    # tokens spread over n_seq sequences at distinct scattered positions
    flat = np.sort(rng.choice(n_seq * 4000, T, replace=False))
    bi = (flat // 4000).astype(np.int32)
    pos = (flat % 4000).astype(np.int32)
    max_pages = 4000 // 64 + 1
    n_pages = n_seq * max_pages + 3
    table = rng.permutation(n_seq * max_pages).astype(np.int32).reshape(n_seq, max_pages) + 1
    pool_np = rng.standard_normal((n_pages, 64, dc + dr)).astype(np.float32)
    pool = torch.from_numpy(pool_np).to(DEV, tdt)
    return d, dict(y=y, w_uk=w_uk, bi=torch.from_numpy(bi).to(DEV),
                   pos=torch.from_numpy(pos).to(DEV), table=table, n_pages=n_pages,
                   max_pages=max_pages, pool=pool, Y=Y, T=T)


def _separate(d, c, y, qbuf, pool, table):
    H, dn, dc, dr = d.n_heads, d.d_nope, d.d_latent, d.d_rope
    dqk, D, Y, T = dn + dr, dc + dr, c["Y"], c["T"]
    off_c = H * dqk
    B.mla_rope(d, y[:, dn:], Y, dqk, H, qbuf[:, :, dc:], H * D, D, c["pos"], T)
    kr = y[:, off_c + dc:]
    B.mla_rope(d, kr, Y, 0, 1, kr, Y, 0, c["pos"], T)
    B.mla_cache_append(d, y[:, off_c:], Y, kr, Y, c["bi"], c["pos"], table, c["max_pages"],
                       pool, c["n_pages"], T)
    B.mla_absorb_q(d, y, Y, c["w_uk"], qbuf, T)


def _both(d, c, table_np):
    H, D = d.n_heads, d.d_latent + d.d_rope
    table = torch.from_numpy(table_np).to(DEV)
    outs = []
    for fused in (False, True):
        y = c["y"].clone()
        pool = c["pool"].clone()
        qbuf = torch.full((c["T"], H, D), float("nan"), dtype=d.torch_dtype, device=DEV)
        if fused:
            B.mla_pre_attention(d, y, c["Y"], c["w_uk"], qbuf, c["bi"], c["pos"], table,
                                c["max_pages"], pool, c["n_pages"], c["T"])
        else:
            _separate(d, c, y, qbuf, pool, table)
        st = status()
        outs.append((y, qbuf, pool, st))
    return outs


def _same_bits(a, b, what):
    ai = a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32)
    bi = b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)
    diff = int((ai != bi).sum())
    assert diff == 0, f"{what}: {diff} elements differ"


@gpu
@pytest.mark.parametrize("dtype,T,n_seq", [("bf16", 16, 16), ("bf16", 130, 7), ("bf16", 256, 3),
                                           ("f32", 5, 2)])
def test_pre_attention_matches_separate_calls(dtype, T, n_seq):
    d, c = _case(dtype, T, n_seq, seed=T)
    (y0, q0, p0, s0), (y1, q1, p1, s1) = _both(d, c, c["table"])
    assert s0 == 0 and s1 == 0
    _same_bits(q1, q0, "qbuf")
    _same_bits(y1, y0, "projection rows (k_rope rotated in place)")
    _same_bits(p1, p0, "pool")
    # the work was done: every written slot differs from the untouched pool
    assert not torch.equal(p1, c["pool"])


@gpu
def test_pre_attention_reports_bad_page_like_append():
    d, c = _case("bf16", 40, 5, seed=3)
    table = c["table"].copy()
    b0 = int(c["bi"][0])
    table[b0, int(c["pos"][0]) // 64] = c["n_pages"] + 9     # outside the pool
    (y0, q0, p0, s0), (y1, q1, p1, s1) = _both(d, c, table)
    assert s0 == 5 and s1 == 5
    _same_bits(q1, q0, "qbuf")
    _same_bits(p1, p0, "pool")


@gpu
def test_graph_replay_matches_eager_step():
    w = wl.workload("dsv2", B=8, ctx=(1000, 64, 65, 2000, 129, 700, 4096, 3))
    d = B.MLADims.of(w)
    layer = MLADecodeLayer(d, wl.draw_weights(w), DEV)
    table, n_pages = wl.page_layout(w)
    layer.set_cache(pool_to_device(build_pool_host_drawn(w, table, n_pages), w.dtype, DEV),
                    torch.from_numpy(table).to(DEV),
                    torch.tensor(w.ctx, dtype=torch.int32, device=DEV))
    bi_np, pos_np = wl.positions(w)
    h = torch.from_numpy(wl.draw_h_new(w).reshape(w.T, w.d_model)).to(DEV, d.torch_dtype)
    bi = torch.from_numpy(bi_np).to(DEV)
    pos = torch.from_numpy(pos_np).to(DEV)
    def run_eager():
        bf = layer.step(h, bi, pos, w.B, w.S_q)
        return {k: bf[k].clone() for k in ("qbuf", "o_lat", "lse", "out")}

    def same(bf, ref):
        # everything up to the decode is deterministic; the output projection
        # adds split-K partial sums with atomics, so its last bits may vary
        for k in ("qbuf", "o_lat", "lse"):
            assert torch.equal(bf[k], ref[k]), k
        err = float((bf["out"] - ref["out"]).abs().max())
        assert err <= 1e-5 * max(1.0, float(ref["out"].abs().max())), err

    eager = run_eager()
    graph, bf, kernels = layer.capture(h, bi, pos, w.B, w.S_q)
    assert kernels >= 5
    for k in ("qbuf", "o_lat", "lse", "out"):
        bf[k].fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert status() == 0
    same(bf, eager)
    # new inputs in the same buffers: the replay follows them
    h.copy_(h.flip(0))
    eager2 = run_eager()
    bf["out"].zero_()
    graph.replay()
    torch.cuda.synchronize()
    same(bf, eager2)
    assert not torch.equal(eager2["o_lat"], eager["o_lat"])
    del graph


@gpu
def test_pipeline_matches_eager_steps():
    """DecodePipeline (two slots, uploads and downloads on side streams)
    gives every step the output the eager step gives for the same inputs."""
    from mla_latent_kv_35_b200.engine import DecodePipeline
    w = wl.workload("dsv2", B=6, ctx=(900, 64, 65, 3000, 129, 7))
    d = B.MLADims.of(w)
    layer = MLADecodeLayer(d, wl.draw_weights(w), DEV)
    table, n_pages = wl.page_layout(w)
    layer.set_cache(pool_to_device(build_pool_host_drawn(w, table, n_pages), w.dtype, DEV),
                    torch.from_numpy(table).to(DEV),
                    torch.tensor(w.ctx, dtype=torch.int32, device=DEV))
    bi_np, pos_np = wl.positions(w)
    h0 = torch.from_numpy(wl.draw_h_new(w).reshape(w.T, w.d_model)).to(d.torch_dtype)
    inputs = [(h0 * (1.0 + 0.25 * k)).to(d.torch_dtype).pin_memory() for k in range(5)]
    bi_h = torch.from_numpy(bi_np).pin_memory()
    pos_h = torch.from_numpy(pos_np).pin_memory()
    pipe = DecodePipeline(layer, w.B, w.S_q)
    outs = [torch.full((w.T, w.d_model), float("nan")).pin_memory() for _ in inputs]
    for x, o in zip(inputs, outs):
        pipe.submit(x, bi_h, pos_h, o)
    pipe.wait()
    assert status() == 0
    for k, x in enumerate(inputs):
        ref = layer.step(x.to(DEV), bi_h.to(DEV), pos_h.to(DEV), w.B, w.S_q)["out"].cpu()
        err = float((outs[k] - ref).abs().max())
        assert err <= 1e-5 * max(1.0, float(ref.abs().max())), (k, err)
    assert not torch.equal(outs[0], outs[1])
