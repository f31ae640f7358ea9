"""GPU parity of each step against the oracle, element by element.

Each test calls the C ABI (through the ctypes binding) on seeded inputs whose
sizes span several tiles and end in a ragged tail, then compares with the
oracle's fp64 result at the documented tolerances.  Cache append and page
indexing are compared bit for bit.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_35_b200 import binding as B
from mla_latent_kv_35_b200 import workloads as wl
from gpu_util import DEV, check, dims, ensure_lib, q, status, to_dev, to_np

gpu = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if torch.cuda.is_available():
        ensure_lib()
        B.mla_get_device_status()


def _tiny_dims():
    return dims("f32", H=8, dn=32, dc=64, dr=16, dm=256)


# --------------------------------------------------------------------------
# A3 cache append: bit exact, canaries survive, bad page ids are reported
# --------------------------------------------------------------------------
@gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_cache_append_bit_exact(dtype):
    rng = np.random.default_rng(0)
    d = dims(dtype) if dtype == "bf16" else _tiny_dims()
    D = d.d_latent + d.d_rope
    P = d.page_size
    n_pages, Bn, maxp = 23, 4, 5
    table = np.full((Bn, maxp), -1, np.int32)
    perm = rng.permutation(n_pages - 1).astype(np.int32)
    table[:, :5] = perm[:20].reshape(4, 5)
    T = 37
    slots = rng.choice(Bn * maxp * P, size=T, replace=False)
    bi = (slots // (maxp * P)).astype(np.int32)
    pos = (slots % (maxp * P)).astype(np.int32)
    if dtype == "bf16":
        npt, tt = np.uint16, torch.int16
        canary = 0xFFFF
    else:
        npt, tt = np.uint32, torch.int32
        canary = 0xFFFFFFFF
    stride = D + 24                                     # rows inside a wider buffer
    src = rng.integers(0, np.iinfo(npt).max, size=(T, stride), dtype=npt)
    pool = np.full((n_pages, P, D), canary, npt)
    exp = oracle.cache_append(pool, src[:, :d.d_latent], src[:, d.d_latent:D], bi, pos,
                              table, P)
    src_d = torch.from_numpy(src.view(np.int16 if dtype == "bf16" else np.int32)).to(DEV)
    pool_d = torch.from_numpy(pool.view(np.int16 if dtype == "bf16" else np.int32)).to(DEV)
    B.mla_cache_append(d, src_d, stride, src_d[:, d.d_latent:], stride,
                       torch.from_numpy(bi).to(DEV), torch.from_numpy(pos).to(DEV),
                       torch.from_numpy(table).to(DEV), maxp, pool_d, n_pages, T)
    assert status() == 0
    got = pool_d.cpu().numpy().view(npt)
    np.testing.assert_array_equal(got, exp)
    assert (got == canary).sum() == pool.size - T * D
    # a page id outside the pool: the token is skipped and BOUNDS is raised
    bad = table.copy()
    bad[0, 0] = n_pages + 3
    pool2 = torch.from_numpy(pool.view(pool_d.cpu().numpy().dtype)).to(DEV)
    B.mla_cache_append(d, src_d[:1], stride, src_d[:1, d.d_latent:], stride,
                       torch.zeros(1, dtype=torch.int32, device=DEV),
                       torch.zeros(1, dtype=torch.int32, device=DEV),
                       torch.from_numpy(bad).to(DEV), maxp, pool2, n_pages, 1)
    assert status() == 5
    np.testing.assert_array_equal(pool2.cpu().numpy().view(npt), pool)


# --------------------------------------------------------------------------
# A2 RoPE
# --------------------------------------------------------------------------
@gpu
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("inplace", [False, True])
def test_rope(dtype, inplace):
    rng = np.random.default_rng(1)
    d = dims(dtype)
    T, nh, xs_head, dr = 19, 5, 192, 64
    xs_tok = nh * xs_head + 8
    x = q(rng.standard_normal((T, xs_tok)), dtype)
    pos = rng.integers(0, 131072, size=T).astype(np.int32)
    pos[0] = 0
    off = 128
    xd = to_dev(x, dtype)
    if inplace:
        yd, ys_tok, ys_head, yoff = xd, xs_tok, xs_head, off
    else:
        yd = torch.zeros((T, nh, 100), device=DEV, dtype=xd.dtype)
        ys_tok, ys_head, yoff = nh * 100, 100, 3
    B.mla_rope(d, xd[:, off:], xs_tok, xs_head, nh, yd.view(T, -1)[:, yoff:], ys_tok, ys_head,
               torch.from_numpy(pos).to(DEV), T)
    got = to_np(yd).reshape(T, -1)
    for h in range(nh):
        xin = x[:, off + h * xs_head: off + h * xs_head + dr].astype(np.float64)
        ref = oracle.rope(xin, pos.astype(np.float64), 10000.0)
        g = got[:, yoff + h * ys_head: yoff + h * ys_head + dr]
        if dtype == "f32":
            check(g, ref, "f32", f"rope head {h}", tol=dict(max_abs=2e-5))
        else:
            check(g, ref, "bf16", f"rope head {h}")
    if dtype == "f32":
        np.testing.assert_array_equal(got[0, yoff:yoff + dr], x[0, off:off + dr])  # pos 0


# --------------------------------------------------------------------------
# A0 projection (tcgen05 GEMM for bf16, SIMT for fp32)
# --------------------------------------------------------------------------
@gpu
@pytest.mark.parametrize("rows,in_f,out_f", [(1, 512, 200), (16, 5120, 640), (130, 256, 384),
                                             (300, 128, 130), (128, 5120, 25152)])
def test_project_bf16(rows, in_f, out_f):
    rng = np.random.default_rng(rows + out_f)
    d = dims("bf16")
    x = q(rng.standard_normal((rows, in_f)), "bf16")
    w = q(rng.standard_normal((out_f, in_f)) / math.sqrt(in_f), "bf16")
    y = torch.empty((rows, out_f), device=DEV, dtype=torch.bfloat16)
    B.mla_project(d, to_dev(x, "bf16"), to_dev(w, "bf16"), y, rows, in_f, out_f)
    assert status() == 0
    check(to_np(y), oracle.project(x, w), "bf16", f"project {rows}x{in_f}->{out_f}")


@gpu
def test_project_f32():
    rng = np.random.default_rng(2)
    d = _tiny_dims()
    for rows, in_f, out_f in [(2, 256, 464), (65, 256, 80), (1, 33, 7)]:
        x = rng.standard_normal((rows, in_f)).astype(np.float32)
        w = (rng.standard_normal((out_f, in_f)) / math.sqrt(in_f)).astype(np.float32)
        y = torch.empty((rows, out_f), device=DEV)
        B.mla_project(d, to_dev(x, "f32"), to_dev(w, "f32"), y, rows, in_f, out_f)
        check(to_np(y), oracle.project(x, w), "f32", "project f32")


# --------------------------------------------------------------------------
# A1 absorption
# --------------------------------------------------------------------------
@gpu
@pytest.mark.parametrize("dtype,T", [("bf16", 1), ("bf16", 16), ("bf16", 130), ("f32", 3)])
def test_absorb_q(dtype, T):
    rng = np.random.default_rng(3 + T)
    d = dims(dtype) if dtype == "bf16" else _tiny_dims()
    H, dn, dc, dr = d.n_heads, d.d_nope, d.d_latent, d.d_rope
    dqk, D = dn + dr, dc + dr
    stride = H * dqk + 64
    qsrc = q(rng.standard_normal((T, stride)), dtype)
    W = q(rng.standard_normal((H, dn, dc)) / math.sqrt(dc), dtype)
    qbuf = torch.zeros((T, H, D), device=DEV,
                       dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)
    B.mla_absorb_q(d, to_dev(qsrc, dtype), stride, to_dev(W, dtype), qbuf, T)
    assert status() == 0
    q_nope = qsrc[:, :H * dqk].reshape(T, H, dqk)[:, :, :dn]
    ref = oracle.absorb_query(q_nope, W)
    got = to_np(qbuf)
    check(got[:, :, :dc], ref, dtype, f"absorb T={T}")
    assert (got[:, :, dc:] == 0).all()                 # RoPE columns untouched


# --------------------------------------------------------------------------
# A6 output projection
# --------------------------------------------------------------------------
@gpu
@pytest.mark.parametrize("dtype,T", [("bf16", 1), ("bf16", 16), ("bf16", 130), ("f32", 2)])
def test_out_proj(dtype, T):
    rng = np.random.default_rng(4 + T)
    d = dims(dtype) if dtype == "bf16" else _tiny_dims()
    H, dc, dv, dm = d.n_heads, d.d_latent, d.d_v, d.d_model
    o_lat = (rng.standard_normal((T, H, dc)) * 0.1).astype(np.float32)
    W_UV = q(rng.standard_normal((H, dv, dc)) / math.sqrt(dc), dtype)
    W_O = q(rng.standard_normal((dm, H * dv)) / math.sqrt(H * dv), dtype)
    out = torch.empty((T, dm), device=DEV)
    sc = torch.empty((B.mla_out_proj_scratch_size(d, T),), dtype=torch.uint8, device=DEV)
    B.mla_out_proj(d, to_dev(o_lat, "f32"), to_dev(W_UV, dtype), to_dev(W_O, dtype), sc, out, T)
    assert status() == 0
    o_in = q(o_lat, dtype)                               # bf16 path rounds o_lat
    _, ref = oracle.out_proj(o_in, W_UV, W_O)
    check(to_np(out), ref, dtype, f"out_proj T={T}")


# --------------------------------------------------------------------------
# A4 + A5 decode on the paged latent cache
# --------------------------------------------------------------------------
def _decode_case(dtype, H, lens, S_q, seed=5, dc=512, dr=64, peaky=False):
    rng = np.random.default_rng(seed)
    d = dims(dtype, H=H, dc=dc, dr=dr) if dtype == "bf16" else \
        dims("f32", H=H, dn=32, dc=dc, dr=dr, dm=256)
    P = d.page_size
    D = dc + dr
    Bn = len(lens)
    npg = [-(-L // P) for L in lens]
    n_pages = sum(npg) + 2
    perm = rng.permutation(n_pages - 2).astype(np.int32) + 1   # page 0 and last unused
    maxp = max(npg) + 1
    table = np.full((Bn, maxp), -1, np.int32)
    o = 0
    for b, n in enumerate(npg):
        table[b, :n] = perm[o:o + n]
        o += n
    rows = [q(rng.standard_normal((L, D)), dtype) for L in lens]
    if peaky:
        for r in rows:
            r[rng.integers(0, r.shape[0])] *= 8
    qb = q(rng.standard_normal((Bn, S_q, H, D)) * (3.0 if peaky else 1.0), dtype)
    if dtype == "bf16":
        pool = np.full((n_pages, P, D), 0xFFFF, np.uint16)    # NaN canaries
    else:
        pool = np.full((n_pages, P, D), np.nan, np.float32)
    for b, r in enumerate(rows):
        for t in range(r.shape[0]):
            pool[table[b, t // P], t % P] = wl.bf16_bits(r[t]) if dtype == "bf16" else r[t]
    if dtype == "bf16":
        pool_d = torch.from_numpy(pool.view(np.int16)).to(DEV).view(torch.bfloat16)
    else:
        pool_d = torch.from_numpy(pool).to(DEV)
    return d, dict(qb=qb, rows=rows, table=table, n_pages=n_pages, maxp=maxp, pool_d=pool_d,
                   lens=np.array(lens, np.int32))


def _run_decode(d, c, S_q, workers=0):
    Bn = len(c["lens"])
    H, dc = d.n_heads, d.d_latent
    ws = torch.empty((B.mla_decode_workspace_size(d, Bn, S_q, workers),), dtype=torch.uint8,
                     device=DEV)
    o_lat = torch.full((Bn, S_q, H, dc), float("nan"), device=DEV)
    lse = torch.full((Bn, S_q, H), float("nan"), device=DEV)
    B.mla_decode(d, to_dev(c["qb"], d.dtype), c["pool_d"], c["n_pages"],
                 torch.from_numpy(c["table"]).to(DEV), c["maxp"],
                 torch.from_numpy(c["lens"]).to(DEV), Bn, S_q, workers, ws, o_lat, lse)
    assert status() == 0
    return to_np(o_lat), to_np(lse)


def _expected_kernel(dtype, H, S_q):
    """The split kernel mla_decode should pick: tensor cores for every bf16
    shape (query blocks under 128 rows are padded), CUDA cores for fp32."""
    return B.DECODE_KERNEL_TC if dtype == "bf16" else B.DECODE_KERNEL_SIMT


def _decode_ref(d, c, b):
    dc = d.d_latent
    r = c["rows"][b].astype(np.float64)
    return oracle.latent_attention(c["qb"][b], r[:, :dc], r[:, dc:], d.scale)


@gpu
@pytest.mark.parametrize("dtype,H,S_q,lens", [
    ("f32", 8, 1, [37, 64]),
    ("f32", 8, 2, [2, 65, 200]),
    ("bf16", 128, 1, [1, 64, 129, 300, 1000]),
    ("bf16", 128, 2, [2, 63, 64, 65, 128, 129, 700]),
    ("bf16", 64, 2, [5, 130, 257]),
    ("bf16", 16, 1, [40, 300]),
    ("bf16", 32, 1, [33, 200, 129]),
    ("bf16", 64, 1, [1, 190, 64]),
    ("bf16", 96, 2, [3, 300, 257]),
    ("bf16", 8, 2, [2, 70]),
])
def test_decode_matches_oracle(dtype, H, S_q, lens):
    dc, dr = (64, 16) if dtype == "f32" else (512, 64)
    d, c = _decode_case(dtype, H, lens, S_q, dc=dc, dr=dr)
    kind, _, _ = B.mla_decode_config(d, S_q, 0)
    assert kind == _expected_kernel(dtype, H, S_q)
    o_lat, lse = _run_decode(d, c, S_q)
    for b in range(len(lens)):
        ref = _decode_ref(d, c, b)
        check(o_lat[b], ref["o_lat"], dtype, f"o_lat b={b} L={lens[b]}")
        check(lse[b], ref["lse"], dtype, f"lse b={b}")


@gpu
@pytest.mark.parametrize("peaky", [False, True])
def test_decode_split_invariance(peaky):
    d, c = _decode_case("bf16", 128, [3000, 77, 1500], 1, seed=6, peaky=peaky)
    base_o, base_l = _run_decode(d, c, 1, workers=1)
    for b in range(3):
        ref = _decode_ref(d, c, b)
        # P is rounded to bf16 (2^-9 relative) before PV, so the absolute error
        # bound scales with the output magnitude; the planted needle makes
        # outputs O(10) in the peaky variant
        mag = max(1.0, float(np.abs(ref["o_lat"]).max()))
        check(base_o[b], ref["o_lat"], "bf16", f"workers=1 b={b}",
              tol=dict(max_abs=2e-2 * mag, mean_abs=2e-3 * mag))
        check(base_l[b], ref["lse"], "bf16", f"lse workers=1 b={b}")
    mag = max(1.0, float(np.abs(base_o).max()))
    for workers in (2, 7, 300, 0):
        o, l = _run_decode(d, c, 1, workers=workers)
        check(o, base_o, "bf16", f"workers={workers}",
              tol=dict(max_abs=4e-3 * mag, mean_abs=2e-4 * mag, rel_l2=2e-3))
        check(l, base_l, "bf16", f"lse workers={workers}", tol=dict(max_abs=1e-3))


# --------------------------------------------------------------------------
# failure path: a bounded wait that runs out returns a status, no fault
# --------------------------------------------------------------------------
@gpu
def test_timeout_selftest_reports_status():
    B.mla_selftest_wait_timeout(2_000_000)      # 2 ms
    assert status() == 4
    assert status() == 0                         # cleared by the read
    x = torch.ones(4, device=DEV)                # context still usable
    assert float((x * 2).sum()) == 8.0


@gpu
def test_decode_rejects_short_context():
    d, c = _decode_case("bf16", 128, [10, 20], 2, seed=9)
    c["lens"] = np.array([1, 20], np.int32)              # seq_len < S_q
    Bn = 2
    ws = torch.empty((B.mla_decode_workspace_size(d, Bn, 2, 0),), dtype=torch.uint8, device=DEV)
    o_lat = torch.empty((Bn, 2, 128, 512), device=DEV)
    lse = torch.empty((Bn, 2, 128), device=DEV)
    B.mla_decode(d, to_dev(c["qb"], "bf16"), c["pool_d"], c["n_pages"],
                 torch.from_numpy(c["table"]).to(DEV), c["maxp"],
                 torch.from_numpy(c["lens"]).to(DEV), Bn, 2, 0, ws, o_lat, lse)
    assert status() == 5
    assert torch.isinf(lse[0]).all() and (o_lat[0] == 0).all()
    ref = _decode_ref(d, c, 1)
    check(to_np(o_lat)[1], ref["o_lat"], "bf16", "valid sequence still correct")


@gpu
@pytest.mark.parametrize("dtype,H,S_q", [("bf16", 128, 1), ("bf16", 128, 2), ("f32", 8, 1)])
def test_decode_reports_page_outside_pool(dtype, H, S_q):
    """A page id past the pool is reported as MLA_ERR_BOUNDS and never read;
    the other sequences of the batch are unaffected."""
    dc, dr = (64, 16) if dtype == "f32" else (512, 64)
    lens = [300, 200, 90]
    d, c = _decode_case(dtype, H, lens, S_q, seed=11, dc=dc, dr=dr)
    c["table"][0, 2] = c["n_pages"] + 7
    o_lat, lse = _run_decode_status(d, c, S_q, expect=5)
    assert status() == 0                         # cleared by the first read
    for b in (1, 2):
        ref = _decode_ref(d, c, b)
        check(o_lat[b], ref["o_lat"], dtype, f"o_lat b={b}")
        check(lse[b], ref["lse"], dtype, f"lse b={b}")
    assert np.isfinite(o_lat[0]).all()


def _run_decode_status(d, c, S_q, expect):
    Bn = len(c["lens"])
    H, dc = d.n_heads, d.d_latent
    ws = torch.empty((B.mla_decode_workspace_size(d, Bn, S_q, 0),), dtype=torch.uint8,
                     device=DEV)
    o_lat = torch.full((Bn, S_q, H, dc), float("nan"), device=DEV)
    lse = torch.full((Bn, S_q, H), float("nan"), device=DEV)
    B.mla_decode(d, to_dev(c["qb"], d.dtype), c["pool_d"], c["n_pages"],
                 torch.from_numpy(c["table"]).to(DEV), c["maxp"],
                 torch.from_numpy(c["lens"]).to(DEV), Bn, S_q, 0, ws, o_lat, lse)
    assert status() == expect
    return to_np(o_lat), to_np(lse)
