"""Chunked prefill (non-absorbed) on the GPU against the oracle.

The oracle's decode_step with S_q = T new tokens is exactly one prefill
chunk: the T tokens are projected, rotated and appended, and each attends
causally (position L - T + j sees t <= L - T + j) over per-head keys and
values rebuilt from the cache.  Small chunks are checked whole (every query,
every head, the output projection); the benchmark's chunk (4096 new tokens
after 4096 cached ones, 128 heads) on sampled queries and heads, through the
oracle's own non-absorbed attention over the visible prefix.
"""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_35_b200 import binding as B
from mla_latent_kv_35_b200 import workloads as wl
from mla_latent_kv_35_b200.binding import MLADims
from mla_latent_kv_35_b200.engine import MLADecodeLayer, build_pool_host, pool_to_device
from gpu_util import DEV, check, ensure_lib, status, to_np

gpu = pytest.mark.gpu


def _stored_bf16_tol(ref):
    """Tolerance of an output the chunk stores in bf16 (o, out, the rebuilt
    k and v): the fp32-accumulation bounds of the decode outputs plus two
    bf16 roundings of at most 2^-9 relative each (the stored value and, for
    out, the bf16 o it is projected from), i.e. 2^-8 of |ref|."""
    a = np.abs(np.asarray(ref, np.float64))
    return dict(max_abs=2e-2 + 2.0 ** -8 * float(a.max()),
                mean_abs=2e-3 + 2.0 ** -8 * float(a.mean()))


def _run(w):
    """The chunk of workload w (one sequence) through MLADecodeLayer.prefill_chunk."""
    ensure_lib()
    assert w.B == 1
    W = wl.draw_weights(w)
    d = MLADims.of(w)
    layer = MLADecodeLayer(d, W, DEV)
    table, n_pages = wl.page_layout(w)
    prior = [wl.draw_prior_bits(w, 0)]
    pool = pool_to_device(build_pool_host(w, table, n_pages, prior), w.dtype, DEV)
    layer.set_cache(pool, torch.from_numpy(table).to(DEV),
                    torch.tensor(w.ctx, dtype=torch.int32, device=DEV))
    h = wl.draw_h_new(w)
    bi, pos = wl.positions(w)
    hd = torch.from_numpy(h.reshape(w.T, w.d_model)).to(DEV, d.torch_dtype)
    T, L = w.S_q, w.ctx[0]
    bf = layer.prefill_chunk(hd, torch.from_numpy(pos).to(DEV), torch.from_numpy(bi).to(DEV),
                             0, T, L)
    torch.cuda.synchronize()
    assert status() == 0
    return W, layer, bf, h, table


def _query_side(w, W, h):
    """The oracle's per-head queries (RoPE applied) and the new tokens' cache
    rows, through the oracle's projection and rotation."""
    T, L = w.S_q, w.ctx[0]
    pos = np.arange(L - T, L)
    dqk = w.d_nope + w.d_rope
    q = oracle.project(h[0], W["W_Q"]).reshape(T, w.H, dqk)
    q[..., w.d_nope:] = oracle.rope(q[..., w.d_nope:], pos[:, None], w.rope_base)
    c_new = oracle.project(h[0], W["W_DKV"])
    kr_new = oracle.rope(oracle.project(h[0], W["W_KR"]), pos, w.rope_base)
    return q, c_new, kr_new


@gpu
@pytest.mark.parametrize("T,L0", [(200, 300), (333, 0), (1, 0), (1, 129), (130, 126),
                                  (256, 128), (600, 77)])
def test_prefill_chunk_small(T, L0):
    """Every query and head of a 16-head chunk against the oracle's decode
    step over the same cache: T not a multiple of the 256-row pair tile, a
    chunk with no cached prefix, single-token chunks, a pair tile whose
    second CTA holds two real rows, several pair tiles; the context is never
    a multiple of the 128-token key block."""
    w = wl.workload("prefill", H=16, S_q=T, ctx=(L0 + T,))
    W, layer, bf, h, table = _run(w)
    c, kr = wl.draw_prior(w, 0)
    res = oracle.decode_step(h, [c], [kr], W["W_Q"], W["W_DKV"], W["W_KR"], W["W_UK"],
                             W["W_UV"], W["W_O"], w.scale, w.rope_base, w.H,
                             prior_kr_rotated=True)
    o = to_np(bf["o"])
    lse = to_np(bf["lse"])
    out = to_np(bf["out"])
    check(o, res["o"][0], "bf16", f"T={T} L0={L0} o", _stored_bf16_tol(res["o"][0]))
    check(lse, res["lse"][0], "bf16", f"T={T} L0={L0} lse")
    check(out, res["out"][0], "bf16", f"T={T} L0={L0} out", _stored_bf16_tol(res["out"][0]))
    # the rebuilt keys and values of the cached tokens, against the oracle's
    # per-head projections of the gathered rows
    C = np.concatenate([c.astype(np.float64), res["c_new"][0]], 0)
    k_nope = to_np(bf["k_nope"])
    v = to_np(bf["v"])
    for i in (0, w.H - 1):
        kref = oracle.project(C, W["W_UK"][i])
        vref = oracle.project(C, W["W_UV"][i])
        check(k_nope[:, i], kref, "bf16", f"k_nope head {i}", _stored_bf16_tol(kref))
        check(v[:, i], vref, "bf16", f"v head {i}", _stored_bf16_tol(vref))


@gpu
def test_prefill_chunk_full_size_sampled():
    """The benchmark's chunk (128 heads, 4096 new tokens after 4096 cached,
    permuted pages): sampled queries at tile and block edges, three heads,
    each through the oracle's non-absorbed attention over the tokens it sees;
    the output projection of sampled rows against W_O applied in fp64 to the
    kernel's own o."""
    w = wl.workload("prefill")
    W, layer, bf, h, table = _run(w)
    T, L = w.S_q, w.ctx[0]
    L0 = L - T
    o = bf["o"]
    lse = bf["lse"]
    out = bf["out"]
    rows = [0, 1, 127, 128, 255, 256, 2047, 3968, T - 1]
    heads = [0, 77, 127]
    o_s = to_np(o[rows][:, heads])
    lse_s = to_np(lse[rows][:, heads])
    o_rows = to_np(o[rows]).reshape(len(rows), -1)
    out_s = to_np(out[rows])
    del layer, bf
    torch.cuda.empty_cache()
    q, c_new, kr_new = _query_side(w, W, h)
    c, kr = wl.draw_prior(w, 0)
    C = np.concatenate([c.astype(np.float64), c_new], 0)
    KR = np.concatenate([kr.astype(np.float64), kr_new], 0)
    for n, j in enumerate(rows):
        vis = L0 + j + 1
        r = oracle.attention_nonabsorbed(q[j:j + 1, heads], C[:vis], KR[:vis],
                                         np.asarray(W["W_UK"])[heads],
                                         np.asarray(W["W_UV"])[heads], w.scale)
        check(o_s[n], r["o"][0], "bf16", f"row {j} o", _stored_bf16_tol(r["o"][0]))
        check(lse_s[n], r["lse"][0], "bf16", f"row {j} lse")
    oref = oracle.project(o_rows, W["W_O"])
    check(out_s, oref, "bf16", "out = W_O o (sampled rows)", _stored_bf16_tol(oref))


@gpu
def test_prefill_rejects_bad_arguments():
    """Host-side validation: shapes the kernels do not cover and T > L are
    refused before anything is enqueued."""
    ensure_lib()
    d = MLADims(16, 128, 512, 64, 128, 512, 64, 192 ** -0.5, 10000.0, "bf16")
    x = torch.zeros(4096, dtype=torch.bfloat16, device=DEV)
    f = torch.zeros(64, dtype=torch.float32, device=DEV)
    with pytest.raises(B.MLAError) as e:
        B.mla_prefill_attention(d, x, 16 * 192, x, x, x, 5, 4, x, f)
    assert e.value.code == 1
    d32 = MLADims(16, 128, 512, 64, 128, 512, 64, 192 ** -0.5, 10000.0, "f32")
    with pytest.raises(B.MLAError) as e:
        B.mla_prefill_attention(d32, x, 16 * 192, x, x, x, 1, 4, x, f)
    assert e.value.code == 2
    dn64 = MLADims(16, 64, 512, 64, 64, 512, 64, 128 ** -0.5, 10000.0, "bf16")
    pt = torch.zeros(4, dtype=torch.int32, device=DEV)
    with pytest.raises(B.MLAError) as e:
        B.mla_prefill_rebuild_kv(dn64, x, 1, pt, 4, x, x, x, x, x)
    assert e.value.code == 2
    torch.cuda.synchronize()
    assert status() == 0


@gpu
def test_prefill_pipeline_matches_direct_chunks():
    """PrefillPipeline (inputs copied in and outputs copied out on side
    streams, two slots) gives the bits of a direct prefill_chunk call, for
    several chunks in flight."""
    from mla_latent_kv_35_b200.engine import PrefillPipeline
    w = wl.workload("prefill", H=16, S_q=200, ctx=(500,))
    W, layer, bf, h, table = _run(w)
    ref = bf["out"].clone()
    T, L = w.S_q, w.ctx[0]
    bi, pos = wl.positions(w)
    d = MLADims.of(w)
    h_host = torch.from_numpy(h.reshape(T, -1)).to(d.torch_dtype).pin_memory()
    bi_host = torch.from_numpy(bi).pin_memory()
    pos_host = torch.from_numpy(pos).pin_memory()
    outs = [torch.empty((T, w.d_model), dtype=d.torch_dtype).pin_memory() for _ in range(3)]
    pipe = PrefillPipeline(layer, 0, T, L)
    for o in outs:
        pipe.submit(h_host, bi_host, pos_host, o)
    pipe.wait()
    torch.cuda.synchronize()
    assert status() == 0
    for o in outs:
        assert torch.equal(o, ref.cpu())


@gpu
def test_decode_after_prefill_chunk():
    """A decode step after a prefill chunk attends over the rows the chunk
    appended: the reference is the oracle's decode step over the drawn prior
    followed by the chunk's own latents and rotated RoPE keys."""
    from dataclasses import replace
    L0, T = 150, 200
    w = wl.workload("prefill", H=16, S_q=T, ctx=(L0 + T,))
    w_dec = replace(w, S_q=1, ctx=(L0 + T + 1,))
    ensure_lib()
    W = wl.draw_weights(w)
    d = MLADims.of(w)
    layer = MLADecodeLayer(d, W, DEV)
    table, n_pages = wl.page_layout(w_dec)
    pool = pool_to_device(build_pool_host(w, table, n_pages, [wl.draw_prior_bits(w, 0)]),
                          w.dtype, DEV)
    layer.set_cache(pool, torch.from_numpy(table).to(DEV),
                    torch.tensor(w_dec.ctx, dtype=torch.int32, device=DEV))
    h = wl.draw_h_new(w)
    bi, pos = wl.positions(w)
    layer.prefill_chunk(torch.from_numpy(h.reshape(T, -1)).to(DEV, d.torch_dtype),
                        torch.from_numpy(pos).to(DEV), torch.from_numpy(bi).to(DEV), 0, T,
                        L0 + T)
    h_next = wl.draw_h_new(w_dec)
    bi1, pos1 = wl.positions(w_dec)
    bf = layer.step(torch.from_numpy(h_next.reshape(1, -1)).to(DEV, d.torch_dtype),
                    torch.from_numpy(bi1).to(DEV), torch.from_numpy(pos1).to(DEV), 1, 1)
    torch.cuda.synchronize()
    assert status() == 0
    _, c_chunk, kr_chunk = _query_side(w, W, h)
    c, kr = wl.draw_prior(w, 0)
    C = np.concatenate([c.astype(np.float64), c_chunk], 0)
    KR = np.concatenate([kr.astype(np.float64), kr_chunk], 0)
    res = oracle.decode_step(h_next, [C], [KR], W["W_Q"], W["W_DKV"], W["W_KR"], W["W_UK"],
                             W["W_UV"], W["W_O"], w.scale, w.rope_base, w.H,
                             prior_kr_rotated=True)
    check(to_np(bf["o_lat"])[0], res["o_lat"][0][0], "bf16", "decode after prefill o_lat")
    check(to_np(bf["lse"])[0], res["lse"][0][0], "bf16", "decode after prefill lse")
    check(to_np(bf["out"])[0], res["out"][0][0], "bf16", "decode after prefill out")


@gpu
def test_prefill_chunk_long_context_sampled():
    """A 512-token chunk after 30000 cached tokens (16 heads, permuted
    pages): ~239 key blocks per query tile; sampled queries at tile edges
    and the last row, every head, through the oracle's non-absorbed attention
    over each query's visible prefix."""
    w = wl.workload("prefill", H=16, S_q=512, ctx=(30512,))
    W, layer, bf, h, table = _run(w)
    T, L = w.S_q, w.ctx[0]
    L0 = L - T
    rows = [0, 255, 256, 511]
    o_s = to_np(bf["o"][rows])
    lse_s = to_np(bf["lse"][rows])
    del layer, bf
    torch.cuda.empty_cache()
    q, c_new, kr_new = _query_side(w, W, h)
    c, kr = wl.draw_prior(w, 0)
    C = np.concatenate([c.astype(np.float64), c_new], 0)
    KR = np.concatenate([kr.astype(np.float64), kr_new], 0)
    for n, j in enumerate(rows):
        vis = L0 + j + 1
        r = oracle.attention_nonabsorbed(q[j:j + 1], C[:vis], KR[:vis], W["W_UK"], W["W_UV"],
                                         w.scale)
        check(o_s[n], r["o"][0], "bf16", f"long row {j} o", _stored_bf16_tol(r["o"][0]))
        check(lse_s[n], r["lse"][0], "bf16", f"long row {j} lse")
