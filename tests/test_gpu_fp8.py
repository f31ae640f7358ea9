"""The 8-bit latent cache on the GPU against the oracle (reading R16).

The quantizer's bytes are compared with the oracle's quantization exactly:
the E4M3 codes, the per-token fp32 scale, the half-precision RoPE key and the
zero padding of every row.  The decode over an 8-bit pool is compared with
the oracle's attention over the numbers the rows stand for.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_oracle as om
from mla_latent_kv_35_b200 import binding as B
from mla_latent_kv_35_b200 import workloads as wl
from gpu_util import DEV, dims, ensure_lib, status

gpu = pytest.mark.gpu
ROW = 656


def e4m3_decode(b):
    """Values of E4M3 bytes from the bit layout (sign, 4 exponent bits with
    bias 7, 3 mantissa bits; exponent field 0 is subnormal)."""
    b = np.asarray(b, dtype=np.int64)
    sgn = np.where(b & 0x80, -1.0, 1.0)
    e, m = (b >> 3) & 0xF, b & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * 2.0 ** (e - 7.0))
    assert not ((e == 0xF) & (m == 0x7)).any(), "NaN code"
    return sgn * val


def split_rows(raw):
    """raw uint8 [..., 656] -> (c8 values [..., 512], kr [..., 64] float64,
    s [...] float64, pad bytes [..., 12])."""
    c8 = e4m3_decode(raw[..., :512])
    kr = np.ascontiguousarray(raw[..., 512:640]).view(np.float16).astype(np.float64)
    s = np.ascontiguousarray(raw[..., 640:644]).view(np.float32)[..., 0].astype(np.float64)
    return c8, kr, s, raw[..., 644:656]


def _latents(rng, n):
    """bf16 latents with a spread of magnitudes per token, some tiny values
    (subnormal after scaling) and one all-zero token."""
    C = rng.standard_normal((n, 512)) * np.exp(rng.uniform(-6, 4, (n, 1)))
    C[:, :8] *= 1e-4
    C[0] = 0.0
    KR = rng.standard_normal((n, 64)) * 2
    q = lambda x: wl.bf16_to_f32(wl.bf16_bits(x.astype(np.float32)))
    return q(C), q(KR)


@gpu
def test_quantize_pool_matches_oracle_bytes():
    ensure_lib()
    rng = np.random.default_rng(50)
    d = dims("bf16")
    n_pages = 5
    C, KR = _latents(rng, n_pages * 64)
    rows = np.concatenate([C, KR], 1)
    pool = torch.from_numpy(wl.bf16_bits(rows).view(np.int16)).to(DEV).view(torch.bfloat16)
    pool8 = torch.full((n_pages * 64 * ROW,), 0xAB, dtype=torch.uint8, device=DEV)
    B.mla_cache_quantize_fp8(d, pool, pool8, n_pages)
    assert status() == 0
    raw = pool8.cpu().numpy().reshape(n_pages * 64, ROW)
    c8, kr, s, pad = split_rows(raw)
    s_ref, c8_ref, kr_ref = om.quantize_latent_fp8(C, KR)
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(c8, c8_ref)
    np.testing.assert_array_equal(kr, kr_ref)
    assert (pad == 0).all()


@gpu
def test_append_fp8_scatter_and_bounds():
    ensure_lib()
    rng = np.random.default_rng(51)
    d = dims("bf16")
    n_pages, Bn, maxp, T = 9, 3, 3, 20
    table = rng.permutation(n_pages)[:Bn * maxp].reshape(Bn, maxp).astype(np.int32)
    slots = rng.choice(Bn * maxp * 64, size=T, replace=False)
    bi = (slots // (maxp * 64)).astype(np.int32)
    pos = (slots % (maxp * 64)).astype(np.int32)
    C, KR = _latents(rng, T)
    stride = 576 + 32
    src = np.zeros((T, stride), np.float32)
    src[:, :512], src[:, 512:576] = C, KR
    src_d = torch.from_numpy(wl.bf16_bits(src).view(np.int16)).to(DEV).view(torch.bfloat16)
    pool8 = torch.full((n_pages, 64, ROW), 0xAB, dtype=torch.uint8, device=DEV)
    B.mla_cache_append_fp8(d, src_d, stride, src_d[:, 512:], stride,
                           torch.from_numpy(bi).to(DEV), torch.from_numpy(pos).to(DEV),
                           torch.from_numpy(table).to(DEV), maxp, pool8, n_pages, T)
    assert status() == 0
    raw = pool8.cpu().numpy()
    s_ref, c8_ref, kr_ref = om.quantize_latent_fp8(C, KR)
    written = np.zeros((n_pages, 64), bool)
    for t in range(T):
        pg, sl = table[bi[t], pos[t] // 64], pos[t] % 64
        c8, kr, s, pad = split_rows(raw[pg, sl])
        np.testing.assert_array_equal(c8, c8_ref[t])
        np.testing.assert_array_equal(kr, kr_ref[t])
        assert s == s_ref[t] and (pad == 0).all()
        written[pg, sl] = True
    assert (raw[~written] == 0xAB).all()                    # untouched slots intact
    bad = table.copy()
    bad[0, 0] = n_pages + 2
    before = pool8.clone()
    B.mla_cache_append_fp8(d, src_d[:1], stride, src_d[:1, 512:], stride,
                           torch.zeros(1, dtype=torch.int32, device=DEV),
                           torch.zeros(1, dtype=torch.int32, device=DEV),
                           torch.from_numpy(bad).to(DEV), maxp, pool8, n_pages, 1)
    assert status() == 5
    assert torch.equal(pool8, before)


def _fp8_case(H, lens, S_q, seed, peaky=False):
    """bf16 cache rows and queries in a permuted paged pool (unused slots
    hold NaN canaries), its 8-bit copy made by the library's quantizer, and
    the oracle's dequantized cache per sequence."""
    rng = np.random.default_rng(seed)
    d = dims("bf16", H=H)
    P, D = 64, 576
    npg = [-(-L // P) for L in lens]
    n_pages = sum(npg) + 1
    perm = rng.permutation(n_pages - 1).astype(np.int32)
    table = np.full((len(lens), max(npg) + 1), -1, np.int32)
    o = 0
    for b, n in enumerate(npg):
        table[b, :n] = perm[o:o + n]
        o += n
    q = lambda x: wl.bf16_to_f32(wl.bf16_bits(x.astype(np.float32)))
    rows = []
    for L in lens:
        r = rng.standard_normal((L, D)) * np.exp(rng.uniform(-1, 1, (L, 1)))
        if peaky:
            r[rng.integers(0, L)] *= 8
        rows.append(q(r))
    qb = q(rng.standard_normal((len(lens), S_q, H, D)) * (3.0 if peaky else 1.0))
    pool = np.full((n_pages, P, D), 0xFFFF, np.uint16)
    for b, r in enumerate(rows):
        for t in range(r.shape[0]):
            pool[table[b, t // P], t % P] = wl.bf16_bits(r[t].astype(np.float32))
    pool_d = torch.from_numpy(pool.view(np.int16)).to(DEV).view(torch.bfloat16)
    pool8 = torch.empty((n_pages, P, ROW), dtype=torch.uint8, device=DEV)
    B.mla_cache_quantize_fp8(d, pool_d, pool8, n_pages)
    deq = []
    for r in rows:
        s, c8, kr8 = om.quantize_latent_fp8(r[:, :512], r[:, 512:])
        deq.append(om.dequantize_fp8(s, c8, kr8))
    return d, dict(qb=qb, deq=deq, rows=rows, table=table, n_pages=n_pages, pool8=pool8,
                   lens=np.array(lens, np.int32))


def _run_fp8(d, c, S_q, workers=0):
    n = len(c["lens"])
    ws = torch.empty((B.mla_decode_fp8_workspace_size(d, n, S_q, workers),), dtype=torch.uint8,
                     device=DEV)
    o = torch.full((n, S_q, d.n_heads, 512), float("nan"), device=DEV)
    l = torch.full((n, S_q, d.n_heads), float("nan"), device=DEV)
    qd = torch.from_numpy(wl.bf16_bits(c["qb"].astype(np.float32)).view(np.int16)).to(DEV)
    B.mla_decode_fp8(d, qd.view(torch.bfloat16), c["pool8"], c["n_pages"],
                     torch.from_numpy(c["table"]).to(DEV), c["table"].shape[1],
                     torch.from_numpy(c["lens"]).to(DEV), n, S_q, workers, ws, o, l)
    assert status() == 0
    return o.double().cpu().numpy(), l.double().cpu().numpy()


@gpu
@pytest.mark.parametrize("H,S_q,lens", [
    (128, 1, [1, 64, 129, 300, 1000]),
    (128, 2, [2, 63, 65, 256, 700]),
    (16, 1, [40, 300]),
    (64, 2, [5, 130, 257]),
])
def test_decode_fp8_matches_oracle_on_dequantized_cache(H, S_q, lens):
    ensure_lib()
    from gpu_util import check
    d, c = _fp8_case(H, lens, S_q, seed=60 + H + S_q)
    o, l = _run_fp8(d, c, S_q)
    for b in range(len(lens)):
        C, KR = c["deq"][b]
        ref = oracle.latent_attention(c["qb"][b], C, KR, d.scale)
        check(o[b], ref["o_lat"], "bf16", f"fp8 o_lat b={b} L={lens[b]}")
        check(l[b], ref["lse"], "bf16", f"fp8 lse b={b}")


@gpu
def test_decode_fp8_split_invariance_and_peaky():
    ensure_lib()
    from gpu_util import check
    d, c = _fp8_case(128, [3000, 77, 1500], 1, seed=70, peaky=True)
    base_o, base_l = _run_fp8(d, c, 1, workers=1)
    for b in range(3):
        C, KR = c["deq"][b]
        ref = oracle.latent_attention(c["qb"][b], C, KR, d.scale)
        mag = max(1.0, float(np.abs(ref["o_lat"]).max()))
        check(base_o[b], ref["o_lat"], "bf16", f"fp8 peaky b={b}",
              tol=dict(max_abs=2e-2 * mag, mean_abs=2e-3 * mag))
        check(base_l[b], ref["lse"], "bf16", f"fp8 peaky lse b={b}")
    for workers in (2, 7, 0):
        o, l = _run_fp8(d, c, 1, workers=workers)
        mag = max(1.0, float(np.abs(base_o).max()))
        check(o, base_o, "bf16", f"fp8 workers={workers}",
              tol=dict(max_abs=4e-3 * mag, mean_abs=2e-4 * mag, rel_l2=2e-3))
