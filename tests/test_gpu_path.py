"""Whole decode step (A0-A6) on the GPU against the oracle, per workload.

tiny: every sequence, non-absorbed oracle, fp32 tolerance.
bf16 workloads at full size, in the launch configuration the benchmark
times: every sequence of dsv2, ragged, long1 and long4, and for batch128
every sequence whose token range a split-worker boundary cuts (plus both
ends), all heads, against the oracle's absorbed formulation (pinned equal to
the non-absorbed one to 1e-10), which also gives the reference for the
output projection; a few heads of a few sequences also go through the
non-absorbed oracle (explicit per-head keys and values).
"""

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_35_b200 import workloads as wl
from mla_latent_kv_35_b200.binding import MLADims
from mla_latent_kv_35_b200.engine import MLADecodeLayer, build_pool_host, pool_to_device
import oracle_pool
from mla_latent_kv_35_b200 import binding as B
from gpu_util import (DEV, check, check_stored_bf16, ensure_lib, fp32_accumulation_bound,
                      status, to_np)

gpu = pytest.mark.gpu


def _setup(w, cache="bf16"):
    ensure_lib()
    W = wl.draw_weights(w)
    d = MLADims.of(w)
    layer = MLADecodeLayer(d, W, DEV)
    table, n_pages = wl.page_layout(w)
    if w.prior_from_h:
        prior = [np.zeros((0, w.D), np.float32) for _ in range(w.B)]
    elif w.dtype == "bf16":
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(8) as ex:
            prior = list(ex.map(lambda b: wl.draw_prior_bits(w, b), range(w.B)))
    else:
        prior = [np.concatenate(wl.draw_prior(w, b), 1) for b in range(w.B)]
    pool = pool_to_device(build_pool_host(w, table, n_pages, prior), w.dtype, DEV)
    del prior
    if cache == "fp8":
        pool8 = torch.empty((n_pages, w.page_size, B.FP8_ROW_BYTES), dtype=torch.uint8,
                            device=DEV)
        B.mla_cache_quantize_fp8(d, pool, pool8, n_pages)
        del pool
        pool = pool8
    layer.set_cache(pool, torch.from_numpy(table).to(DEV),
                    torch.tensor(w.ctx, dtype=torch.int32, device=DEV), kind=cache)
    h_ctx = None
    if w.prior_from_h:
        h_ctx = [wl.draw_h_ctx(w, b) for b in range(w.B)]
        layer.prefill_from_hidden(h_ctx)
    h = wl.draw_h_new(w)
    bi, pos = wl.positions(w)
    hd = torch.from_numpy(h.reshape(w.T, w.d_model)).to(DEV, d.torch_dtype)
    bf = layer.step(hd, torch.from_numpy(bi).to(DEV), torch.from_numpy(pos).to(DEV), w.B,
                    w.S_q)
    torch.cuda.synchronize()
    assert status() == 0
    return W, layer, bf, h, h_ctx, table


@gpu
def test_tiny_full_path_fp32():
    w = wl.workload("tiny")
    W, layer, bf, h, h_ctx, table = _setup(w)
    c_prior = [oracle.project(x, W["W_DKV"]) for x in h_ctx]
    kr_prior = [oracle.project(x, W["W_KR"]) for x in h_ctx]
    res = oracle.decode_step(h, c_prior, kr_prior, W["W_Q"], W["W_DKV"], W["W_KR"], W["W_UK"],
                             W["W_UV"], W["W_O"], w.scale, w.rope_base, w.H)
    H, dqk, dc = w.H, w.d_nope + w.d_rope, w.d_latent
    y = to_np(bf["y"])
    qbuf = to_np(bf["qbuf"])
    o_lat = to_np(bf["o_lat"])
    lse = to_np(bf["lse"])
    out = to_np(bf["out"])
    pool = to_np(layer.pool)
    for b in range(w.B):
        check(y[b, :H * dqk].reshape(H, dqk), res["q"][b][0], "f32", "A0 q")
        check(qbuf[b, :, dc:], res["q_roped"][b][0, :, w.d_nope:], "f32", "A2 q_rope")
        L = w.ctx[b]
        row = pool[table[b, (L - 1) // 64], (L - 1) % 64]
        check(row[:dc], res["c_new"][b][0], "f32", "A3 c")
        check(row[dc:], res["kr_new"][b][0], "f32", "A3 k_rope")
        check(o_lat[b], res["o_lat"][b][0], "f32", "A4 o_lat")
        check(lse[b], res["lse"][b][0], "f32", "A4 lse")
        check(out[b], res["out"][b][0], "f32", "A6 out")


def _check_bf16_workload(name, sample, nonabs_sample, nonabs_heads=(0, 77, 127)):
    """Every sequence in `sample`: all heads against the oracle's absorbed
    formulation (run in a pool of host processes); sequences in
    `nonabs_sample`: a few heads against the non-absorbed oracle too."""
    w = wl.workload(name)
    W, layer, bf, h, _, table = _setup(w)
    o_lat = to_np(bf["o_lat"]).reshape(w.B, w.S_q, w.H, w.d_latent)
    lse = to_np(bf["lse"]).reshape(w.B, w.S_q, w.H)
    out = to_np(bf["out"]).reshape(w.B, w.S_q, w.d_model)
    pool_bits = layer.pool.view(torch.int16)
    new_rows = {}
    for b in sample:
        L = w.ctx[b]
        new_rows[b] = [pool_bits[int(table[b, p // 64]), p % 64].cpu().numpy().view(np.uint16)
                       for p in range(L - w.S_q, L)]
    del layer, bf
    torch.cuda.empty_cache()
    ref = oracle_pool.workload_reference(w, W, h, sample)
    for b in sample:
        r = ref[b]
        check(o_lat[b], r["o_lat"], "bf16", f"{name} b={b} o_lat (all heads)")
        check(lse[b], r["lse"], "bf16", f"{name} b={b} lse")
        check(out[b], r["out"], "bf16", f"{name} b={b} out")
        # the appended rows hold the new tokens' latent and rotated RoPE key
        acc_c = fp32_accumulation_bound(h[b], W["W_DKV"])
        acc_k = fp32_accumulation_bound(h[b], W["W_KR"])
        for j, row in enumerate(new_rows[b]):
            rowf = wl.bf16_to_f32(row).astype(np.float64)
            check_stored_bf16(rowf[:w.d_latent], r["c_new"][j], "A3 c_new", acc=acc_c[j])
            check_stored_bf16(rowf[w.d_latent:], r["kr_new"][j], "A3 kr_new", rotated=True,
                              acc=acc_k[j])
    for b in nonabs_sample:
        c, kr = wl.draw_prior(w, b)
        na = oracle.decode_step(h[b:b + 1], [c], [kr], W["W_Q"], W["W_DKV"], W["W_KR"],
                                W["W_UK"], W["W_UV"], W["W_O"], w.scale, w.rope_base, w.H,
                                prior_kr_rotated=True, heads=list(nonabs_heads))
        check(o_lat[b][:, list(nonabs_heads)], na["o_lat"][0], "bf16",
              f"{name} b={b} o_lat vs non-absorbed")
        check(lse[b][:, list(nonabs_heads)], na["lse"][0], "bf16",
              f"{name} b={b} lse vs non-absorbed")


def boundary_sequences(w, S_q=1):
    """Sequences whose block range is cut by a split-worker boundary, from
    the planner's own rule (worker k starts at block floor(k*total/G))."""
    d = MLADims.of(w)
    _, bt, G = B.mla_decode_config(d, S_q, 0)
    R = max(1, -(-S_q * w.H // 128))
    # virtual sequence v = r * B + b: row block r of sequence b
    nb = [-(-L // bt) for _ in range(R) for L in w.ctx]
    starts = np.concatenate([[0], np.cumsum(nb)])
    total = int(starts[-1])
    out = set()
    for k in range(1, G):
        x = k * total // G
        v = int(np.searchsorted(starts, x, side="right") - 1)
        if x != starts[v]:
            out.add(v % w.B)
    return sorted(out)


@gpu
def test_dsv2_full_path():
    _check_bf16_workload("dsv2", sample=range(16), nonabs_sample=[0, 9, 15])


@gpu
def test_ragged_full_path():
    w = wl.workload("ragged")
    lens = np.array(w.ctx)
    _check_bf16_workload("ragged", sample=range(64),
                         nonabs_sample=[int(np.argmin(lens)), int(np.argmax(lens)), 5])


@gpu
def test_batch128_full_path():
    w = wl.workload("batch128")
    ensure_lib()
    seqs = sorted(set(boundary_sequences(w)) | {0, 1, 63, 64, 126, 127})
    assert len(seqs) >= 16
    _check_bf16_workload("batch128", sample=seqs, nonabs_sample=[0, seqs[len(seqs) // 2]],
                         nonabs_heads=(3, 100))


@gpu
@pytest.mark.parametrize("name", ["long1", "long4"])
def test_long_context_full_path(name):
    w = wl.workload(name)
    _check_bf16_workload(name, sample=range(w.B), nonabs_sample=[0], nonabs_heads=(64,))


def _fp8_row_values(raw):
    """(latent, RoPE key) numbers of 656-byte rows of the 8-bit cache, from
    the bit layout: E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits)
    times the fp32 row scale, and the half-precision key times the scale."""
    raw = np.asarray(raw, dtype=np.uint8)
    b = raw[..., :512].astype(np.int64)
    e, m = (b >> 3) & 0xF, b & 0x7
    c8 = np.where(b & 0x80, -1.0, 1.0) * np.where(e == 0, m / 8.0 * 2.0 ** -6,
                                                  (1 + m / 8.0) * 2.0 ** (e - 7.0))
    kr = np.ascontiguousarray(raw[..., 512:640]).view(np.float16).astype(np.float64)
    s = np.ascontiguousarray(raw[..., 640:644]).view(np.float32)[..., 0].astype(np.float64)
    return c8 * s[..., None], kr * s[..., None]


@gpu
def test_dsv2_full_path_fp8_cache():
    """The whole step over the 8-bit latent cache (bf16 workload dsv2): the
    prior rows quantized by the library (byte-exact against the oracle's
    quantizer in test_gpu_fp8.py), the new rows quantized by the append.
    Reference: the oracle over its own quantization of the same cache, prior
    and new rows."""
    name = "dsv2"
    w = wl.workload(name)
    W, layer, bf, h, _, table = _setup(w, cache="fp8")
    o_lat = to_np(bf["o_lat"]).reshape(w.B, w.S_q, w.H, w.d_latent)
    lse = to_np(bf["lse"]).reshape(w.B, w.S_q, w.H)
    out = to_np(bf["out"]).reshape(w.B, w.S_q, w.d_model)
    sample = [0, 5, 10, 15]
    new_rows = {}
    for b in sample:
        L = w.ctx[b]
        new_rows[b] = [layer.pool[int(table[b, p // 64]), p % 64].cpu().numpy()
                       for p in range(L - w.S_q, L)]
    del layer, bf
    torch.cuda.empty_cache()
    ref = oracle_pool.workload_reference(w, W, h, sample, cache="fp8")
    for b in sample:
        r = ref[b]
        check(o_lat[b], r["o_lat"], "bf16", f"{name} fp8 b={b} o_lat (all heads)")
        check(lse[b], r["lse"], "bf16", f"{name} fp8 b={b} lse")
        check(out[b], r["out"], "bf16", f"{name} fp8 b={b} out")
        # the appended rows: the new tokens' latent and rotated RoPE key, to
        # the precision of the 8-bit format (E4M3: 2^-4 relative to the row
        # scale's range, the f16 key 2^-11), over the bf16-rounded inputs
        for j, row in enumerate(new_rows[b]):
            c, kr = _fp8_row_values(row)
            c_ref, kr_ref = r["c_new"][j], r["kr_new"][j]
            assert np.abs(c - c_ref).max() <= 2.0 ** -3 * np.abs(c_ref).max() + 1e-30, "A3 c8"
            assert np.abs(kr - kr_ref).max() <= 2.0 ** -6 * np.abs(kr_ref).max() + 1e-30, "A3 kr16"
