"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

None of these compare the oracle with itself.  Each pin is chosen so that a
plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand) fails at least one of them:

* cache arithmetic printed on the deepforge "DeepSeek-V2" page (golden file);
* RoPE against the complex-exponential closed form, and its invariants;
* the absorption identity (deepforge §1 "Store a latent, rebuild the keys and
  values": the up-projections are linear, so W_UK folds into the query and
  W_UV into the output) to 1e-10;
* a pure-Python brute force of textbook attention on tiny inputs;
* special cases that reduce to a library routine (torch SDPA in fp64) or to
  closed forms.
"""

import cmath
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_oracle as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            kv = line.split(";", 1)[0]
            k, v = (s.strip() for s in kv.split("="))
            out[k] = float(v)
    return out


# --------------------------------------------------------------------------
# cache arithmetic
# --------------------------------------------------------------------------

def test_cache_arithmetic_matches_pages():
    g = _golden("cache_arithmetic.txt")
    assert oracle.cache_elems_per_token("mla", d_latent=512, d_rope=64) == \
        g["mla_elems_per_token"]
    assert oracle.cache_elems_per_token("mha", n_heads=128, d_head=128) == \
        g["mha_elems_per_token"]
    assert oracle.cache_elems_per_token("mha", n_heads=128, d_head=128) * 60 \
        == g["dense_numbers_60_layers"]
    dense = oracle.dense_cache_bytes(128, 128, 60, 8192)
    sparse = oracle.mla_cache_bytes(512, 64, 60, 8192)
    assert dense // sparse == g["dense_over_mla_int"]
    assert abs(dense / sparse - 32768 / 576) < 1e-12
    assert oracle.gqa_equivalent_groups(512, 64, 128) == g["gqa_groups"]
    # GQA with that many groups caches the same numbers as MLA
    assert oracle.cache_elems_per_token(
        "gqa", n_groups=g["gqa_groups"], d_head=128) == 576


# --------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------

def _rope_complex(x, pos, base):
    """Closed form: pair k is the complex number x[2k] + i x[2k+1] times
    exp(i * pos * base^(-2k/d))."""
    d = len(x)
    out = []
    for k in range(d // 2):
        z = complex(x[2 * k], x[2 * k + 1]) * cmath.exp(
            1j * pos * base ** (-2.0 * k / d))
        out += [z.real, z.imag]
    return np.array(out)


def test_rope_worked_example():
    # d=4, base 10000: theta_0 = 1 rad/pos, theta_1 = 0.01 rad/pos.
    x = np.array([1.0, 0.0, 0.0, 1.0])
    y = oracle.rope(x, 100, 10000.0)
    expect = [math.cos(100.0), math.sin(100.0), -math.sin(1.0), math.cos(1.0)]
    np.testing.assert_allclose(y, expect, rtol=0, atol=1e-12)


@pytest.mark.parametrize("d,base", [(2, 10000.0), (16, 10000.0), (64, 10000.0),
                                    (8, 500.0)])
def test_rope_closed_form(d, base):
    rng = np.random.default_rng(1)
    for pos in (0, 1, 7, 4095, 131071):
        x = rng.standard_normal(d)
        np.testing.assert_allclose(oracle.rope(x, pos, base),
                                   _rope_complex(x, pos, base),
                                   rtol=0, atol=1e-9)


def test_rope_invariants():
    rng = np.random.default_rng(2)
    q = rng.standard_normal(64)
    k = rng.standard_normal(64)
    np.testing.assert_array_equal(oracle.rope(q, 0), q)          # pos 0
    for m in (3, 1000, 131000):
        assert abs(np.linalg.norm(oracle.rope(q, m)) - np.linalg.norm(q)) < 1e-10
    # <RoPE(q,m), RoPE(k,n)> depends only on m - n
    ref = oracle.rope(q, 10) @ oracle.rope(k, 3)
    for shift in (1, 50, 9000):
        v = oracle.rope(q, 10 + shift) @ oracle.rope(k, 3 + shift)
        assert abs(v - ref) < 1e-10
    # batched call agrees with one-by-one calls
    X = rng.standard_normal((5, 3, 16))
    pos = np.arange(5)[:, None]
    Y = oracle.rope(X, pos)
    for t in range(5):
        for h in range(3):
            np.testing.assert_allclose(Y[t, h], oracle.rope(X[t, h], t),
                                       atol=1e-14)


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _rand_problem(rng, S_q=2, H=3, L=9, d_n=5, d_c=7, d_r=4, d_v=None):
    d_v = d_n if d_v is None else d_v
    return dict(
        q=rng.standard_normal((S_q, H, d_n + d_r)),
        C=rng.standard_normal((L, d_c)),
        KR=rng.standard_normal((L, d_r)),
        W_UK=rng.standard_normal((H, d_n, d_c)),
        W_UV=rng.standard_normal((H, d_v, d_c)),
        scale=1.0 / math.sqrt(d_n + d_r),
    )


def _brute_force(q, C, KR, W_UK, W_UV, scale):
    """Textbook attention with explicit keys/values, pure-Python loops."""
    S_q, H, _ = q.shape
    L, d_c = C.shape
    d_n = W_UK.shape[1]
    d_v = W_UV.shape[1]
    d_r = KR.shape[1]
    outs = {}
    for j in range(S_q):
        for i in range(H):
            vis = L - S_q + j + 1
            keys, vals = [], []
            for t in range(vis):
                k = [sum(W_UK[i][a][c] * C[t][c] for c in range(d_c))
                     for a in range(d_n)] + [KR[t][r] for r in range(d_r)]
                v = [sum(W_UV[i][a][c] * C[t][c] for c in range(d_c))
                     for a in range(d_v)]
                keys.append(k)
                vals.append(v)
            s = [scale * sum(q[j][i][a] * keys[t][a] for a in range(d_n + d_r))
                 for t in range(vis)]
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            z = sum(e)
            o = [sum(e[t] / z * vals[t][a] for t in range(vis))
                 for a in range(d_v)]
            ol = [sum(e[t] / z * C[t][c] for t in range(vis))
                  for c in range(d_c)]
            outs[(j, i)] = (o, ol, mx + math.log(z))
    return outs


def test_nonabsorbed_matches_brute_force():
    rng = np.random.default_rng(3)
    P = _rand_problem(rng)
    res = oracle.attention_nonabsorbed(**P)
    bf = _brute_force(**P)
    for (j, i), (o, ol, lse) in bf.items():
        np.testing.assert_allclose(res["o"][j, i], o, atol=1e-12)
        np.testing.assert_allclose(res["o_lat"][j, i], ol, atol=1e-12)
        assert abs(res["lse"][j, i] - lse) < 1e-12


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_absorption_identity(seed):
    rng = np.random.default_rng(seed)
    P = _rand_problem(rng, S_q=2, H=4, L=33, d_n=8, d_c=12, d_r=6)
    a = oracle.attention_nonabsorbed(**P)
    b = oracle.attention_absorbed(**P)
    for key in ("o", "o_lat", "lse"):
        np.testing.assert_allclose(a[key], b[key], rtol=0, atol=1e-10)


def test_softmax_rows_and_lse():
    rng = np.random.default_rng(4)
    P = _rand_problem(rng, S_q=2, H=3, L=20)
    res = oracle.attention_nonabsorbed(**P)
    d_n = P["W_UK"].shape[1]
    for j in range(2):
        for i in range(3):
            p = res["p"][j][i]
            assert abs(p.sum() - 1.0) < 1e-12
            assert len(p) == 20 - 2 + j + 1            # causal visibility
            # lse recomputed from raw scores
            vis = len(p)
            k = np.concatenate([P["C"][:vis] @ P["W_UK"][i].T, P["KR"][:vis]], 1)
            s = P["scale"] * k @ P["q"][j, i]
            assert abs(res["lse"][j, i] - math.log(np.exp(s).sum())) < 1e-12
            assert d_n == 5


def test_single_token_context():
    # L = 1: the only probability is 1, so o_i = W_UV[i] c_0 exactly.
    rng = np.random.default_rng(5)
    P = _rand_problem(rng, S_q=1, H=3, L=1)
    res = oracle.attention_nonabsorbed(**P)
    for i in range(3):
        np.testing.assert_allclose(res["o"][0, i], P["W_UV"][i] @ P["C"][0],
                                   atol=1e-14)
        np.testing.assert_allclose(res["o_lat"][0, i], P["C"][0], atol=1e-15)


def test_identical_tokens_ignore_query():
    rng = np.random.default_rng(6)
    P = _rand_problem(rng, S_q=1, H=2, L=10)
    P["C"][:] = P["C"][0]
    P["KR"][:] = P["KR"][0]
    r1 = oracle.attention_nonabsorbed(**P)
    P["q"] = rng.standard_normal(P["q"].shape) * 10
    r2 = oracle.attention_nonabsorbed(**P)
    np.testing.assert_allclose(r1["o"], r2["o"], atol=1e-12)
    np.testing.assert_allclose(r1["o_lat"][0, 0], P["C"][0], atol=1e-12)


def test_zero_query_is_uniform_mean():
    rng = np.random.default_rng(7)
    P = _rand_problem(rng, S_q=1, H=2, L=13)
    P["q"][:] = 0.0
    res = oracle.attention_nonabsorbed(**P)
    for i in range(2):
        np.testing.assert_allclose(res["o_lat"][0, i], P["C"].mean(0), atol=1e-13)
        np.testing.assert_allclose(res["o"][0, i],
                                   P["W_UV"][i] @ P["C"].mean(0), atol=1e-13)
        assert abs(res["lse"][0, i] - math.log(13)) < 1e-13


@pytest.mark.parametrize("S_q,L", [(1, 17), (2, 17), (3, 5)])
def test_reduces_to_library_sdpa(S_q, L):
    """H=1, d_c = d_n, W_UK = W_UV = I, no RoPE part: plain single-head
    softmax attention with a causal block at the end; torch's fp64 SDPA is
    an independent implementation of that."""
    rng = np.random.default_rng(8)
    d = 6
    P = dict(q=rng.standard_normal((S_q, 1, d)), C=rng.standard_normal((L, d)),
             KR=np.zeros((L, 0)), W_UK=np.eye(d)[None], W_UV=np.eye(d)[None],
             scale=1.0 / math.sqrt(d))
    res = oracle.attention_nonabsorbed(**P)
    q = torch.tensor(P["q"][:, 0][None, None])          # [1,1,S_q,d]
    kv = torch.tensor(P["C"][None, None])               # [1,1,L,d]
    mask = torch.ones(S_q, L, dtype=torch.bool).tril(diagonal=L - S_q)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, kv, kv, attn_mask=mask, scale=P["scale"])[0, 0].numpy()
    np.testing.assert_allclose(res["o"][:, 0], ref, atol=1e-12)


def test_combine_splits_equals_full():
    rng = np.random.default_rng(9)
    P = _rand_problem(rng, S_q=1, H=3, L=40)
    full = oracle.attention_nonabsorbed(**P)
    cuts = [0, 7, 8, 25, 40]
    o_parts, l_parts = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        sub = dict(P, C=P["C"][a:b], KR=P["KR"][a:b])
        r = oracle.attention_nonabsorbed(**sub)
        o_parts.append(r["o_lat"])
        l_parts.append(r["lse"])
    o, lse = oracle.combine_splits(o_parts, l_parts)
    np.testing.assert_allclose(o, full["o_lat"], atol=1e-12)
    np.testing.assert_allclose(lse, full["lse"], atol=1e-12)
    o1, l1 = oracle.combine_splits([full["o_lat"]], [full["lse"]])
    np.testing.assert_allclose(o1, full["o_lat"], atol=1e-15)
    # an empty split (lse = -inf) carries no weight
    o2, l2 = oracle.combine_splits([full["o_lat"], np.zeros_like(full["o_lat"])],
                                   [full["lse"], np.full_like(full["lse"], -np.inf)])
    np.testing.assert_allclose(o2, full["o_lat"], atol=1e-15)


def test_range_partition_merges_to_full():
    """Range attention of a partition of the sequence, merged, is the whole
    sequence's attention; the causal cut falls inside the last ranges."""
    rng = np.random.default_rng(17)
    S_q, H, L, d_c, d_r = 2, 3, 40, 6, 4
    q = rng.standard_normal((S_q, H, d_c + d_r))
    C = rng.standard_normal((L, d_c))
    KR = rng.standard_normal((L, d_r))
    full = oracle.latent_attention(q, C, KR, 0.4)
    for cuts in ([0, 7, 8, 39, 40], [0, 20, 38, 40], [0, 40], [0, 1, 2, 39, 40]):
        parts = [oracle.latent_attention_range(q, C[a:b], KR[a:b], 0.4, a, L)
                 for a, b in zip(cuts[:-1], cuts[1:])]
        o, lse = oracle.combine_splits([r["o_lat"] for r in parts], [r["lse"] for r in parts])
        np.testing.assert_allclose(o, full["o_lat"], atol=1e-12)
        np.testing.assert_allclose(lse, full["lse"], atol=1e-12)
    # the last token is the second query: query 0 sees nothing in [39, 40)
    last = oracle.latent_attention_range(q, C[39:], KR[39:], 0.4, 39, L)
    assert np.all(last["lse"][0] == -np.inf) and np.all(last["o_lat"][0] == 0)
    assert np.all(np.isfinite(last["lse"][1]))
    # a single visible token: its own latent, lse = its score
    np.testing.assert_allclose(last["o_lat"][1], np.broadcast_to(C[39], (H, d_c)), atol=1e-15)
    s = 0.4 * (q[1, :, :d_c] @ C[39] + q[1, :, d_c:] @ KR[39])
    np.testing.assert_allclose(last["lse"][1], s, atol=1e-12)


def test_cache_append_scatter():
    rng = np.random.default_rng(10)
    pool = np.full((6, 4, 5), 0xFFFF, dtype=np.uint16)
    table = np.array([[3, 0, -1], [5, 1, 2]], dtype=np.int32)
    c = rng.integers(0, 60000, size=(3, 3)).astype(np.uint16)
    kr = rng.integers(0, 60000, size=(3, 2)).astype(np.uint16)
    bi = np.array([0, 1, 1])
    pos = np.array([5, 3, 9])
    out = oracle.cache_append(pool, c, kr, bi, pos, table, 4)
    expect = pool.copy()
    rows = np.concatenate([c, kr], 1)
    expect[table[bi, pos // 4], pos % 4] = rows                 # fancy index
    np.testing.assert_array_equal(out, expect)
    assert (out == 0xFFFF).sum() == pool.size - 3 * 5           # canaries


def test_decode_step_composes_the_pieces():
    """decode_step vs hand composition with the absorbed formulation."""
    rng = np.random.default_rng(11)
    H, dm, dn, dc, dr, S_q = 3, 10, 4, 6, 4, 2
    W = dict(W_Q=rng.standard_normal((H * (dn + dr), dm)),
             W_DKV=rng.standard_normal((dc, dm)),
             W_KR=rng.standard_normal((dr, dm)),
             W_UK=rng.standard_normal((H, dn, dc)),
             W_UV=rng.standard_normal((H, dn, dc)),
             W_O=rng.standard_normal((dm, H * dn)))
    h = rng.standard_normal((2, S_q, dm))
    cp = [rng.standard_normal((5, dc)), rng.standard_normal((0, dc))]
    kp = [rng.standard_normal((5, dr)), rng.standard_normal((0, dr))]
    res = oracle.decode_step(h, cp, kp, scale=0.3, rope_base=100.0,
                             n_heads=H, **W)
    for b in range(2):
        Lp = cp[b].shape[0]
        pos = np.arange(Lp + S_q)
        C = np.concatenate([cp[b], h[b] @ W["W_DKV"].T])
        KR = oracle.rope(np.concatenate([kp[b], h[b] @ W["W_KR"].T]), pos, 100.0)
        q = (h[b] @ W["W_Q"].T).reshape(S_q, H, dn + dr)
        q[..., dn:] = oracle.rope(q[..., dn:], pos[Lp:, None], 100.0)
        ab = oracle.attention_absorbed(q, C, KR, W["W_UK"], W["W_UV"], 0.3)
        np.testing.assert_allclose(res["o_lat"][b], ab["o_lat"], atol=1e-10)
        out = ab["o"].reshape(S_q, -1) @ W["W_O"].T
        np.testing.assert_allclose(res["out"][b], out, atol=1e-10)


def test_planted_mistakes_are_caught(monkeypatch):
    """Each plausible slip in the oracle trips one of the pins above."""
    rng = np.random.default_rng(12)
    P = _rand_problem(rng, S_q=1, H=2, L=6, d_n=3, d_c=4, d_r=2)
    bf = _brute_force(**P)

    def disagrees():
        r = oracle.attention_nonabsorbed(**P)
        return any(abs(r["lse"][j, i] - v[2]) > 1e-9 or
                   np.abs(r["o"][j, i] - v[0]).max() > 1e-9
                   for (j, i), v in bf.items())

    assert not disagrees()
    # transposed up-projection: use W_UK[i] columns as rows
    bad = dict(P, W_UK=np.transpose(P["W_UK"], (0, 2, 1))[:, :3, :3])
    with pytest.raises(Exception):
        oracle.attention_nonabsorbed(**bad)
    # wrong softmax scale
    orig = om._softmax_attend
    monkeypatch.setattr(om, "_softmax_attend",
                        lambda s, v: orig(s * 0.5, v))
    assert disagrees()
    monkeypatch.setattr(om, "_softmax_attend", orig)
    # RoPE slips are planted inside rope in test_rope_planted_mistakes_are_caught,
    # the projection's transpose in test_project_transpose_slip_is_caught


def test_out_proj_matches_nonabsorbed_output():
    """out_proj(o_lat) equals W_O applied to the explicit per-head outputs."""
    rng = np.random.default_rng(13)
    P = _rand_problem(rng, S_q=1, H=3, L=11)
    res = oracle.attention_nonabsorbed(**P)
    W_O = rng.standard_normal((7, 3 * 5))
    o, out = oracle.out_proj(res["o_lat"], P["W_UV"], W_O)
    np.testing.assert_allclose(o, res["o"], atol=1e-12)
    np.testing.assert_allclose(out, res["o"].reshape(1, -1) @ W_O.T, atol=1e-12)


# --------------------------------------------------------------------------
# projection: pure-Python brute force, square and non-square weights
# --------------------------------------------------------------------------

def _project_brute(x, w):
    """y[r][o] = sum_i x[r][i] * w[o][i], written out with loops (w is
    [out, in]: each output feature is one row of w)."""
    return [[sum(x[r][i] * w[o][i] for i in range(len(x[r]))) for o in range(len(w))]
            for r in range(len(x))]


@pytest.mark.parametrize("rows,in_f,out_f", [(3, 4, 4), (2, 5, 3), (1, 3, 7)])
def test_project_matches_brute_force(rows, in_f, out_f):
    rng = np.random.default_rng(rows * 100 + in_f * 10 + out_f)
    x = rng.standard_normal((rows, in_f))
    w = rng.standard_normal((out_f, in_f))
    np.testing.assert_allclose(oracle.project(x, w), _project_brute(x, w), rtol=0, atol=1e-12)


def test_project_transpose_slip_is_caught(monkeypatch):
    """A transposed weight (x @ w instead of x @ w^T) planted in the oracle
    fails the brute-force pin on a square, non-symmetric weight."""
    rng = np.random.default_rng(31)
    x = rng.standard_normal((3, 4))
    w = rng.standard_normal((4, 4))
    assert np.abs(w - w.T).max() > 0.1
    monkeypatch.setattr(om, "project", lambda a, b: np.asarray(a, float) @ np.asarray(b, float))
    assert np.abs(om.project(x, w) - np.array(_project_brute(x, w))).max() > 1e-3


# --------------------------------------------------------------------------
# decode_step wiring, worked by hand
# --------------------------------------------------------------------------

def test_decode_step_hand_worked_example():
    """One sequence with two cached tokens and two new query tokens, two
    heads, every weight chosen so the step can be followed by hand.

    Sizes: d_model 2, d_nope 1, latent 1, rope 2 (one pair, theta = 1 rad per
    position whatever the base), d_v 1, scale 1/2.
    Cached before the step (reading R2): token 0 with c = 3, pre-RoPE key
    (1, 0); token 1 with c = -1, pre-RoPE key (0, 1).  The new tokens sit at
    positions 2 and 3 (L - S_q + j), with hidden states (1, 0) and (0, 1).
      W_DKV = [1 2]  -> c_2 = 1, c_3 = 2
      W_KR  = I      -> pre-RoPE keys (1, 0) and (0, 1)
    RoPE by position t rotates the key by t rad:
      k_0 = (1, 0), k_1 = (-sin 1, cos 1), k_2 = (cos 2, sin 2),
      k_3 = (-sin 3, cos 3)
    W_Q gives both heads q_nope = 1 and q_rope = h, so the rotated query
    parts are (cos 2, sin 2) at position 2 and (-sin 3, cos 3) at position 3.
    Head 0: W_UK = 2, W_UV = 1, so its key is (2 c_t ; k_t); head 1: W_UK = 0,
    W_UV = 2.  Dot products of rotated RoPE parts depend on the position
    difference: (cos 2, sin 2).(-sin 1, cos 1) = sin 1,
    (-sin 3, cos 3).(1, 0) = -sin 3, (-sin 3, cos 3).(-sin 1, cos 1) = cos 2,
    (-sin 3, cos 3).(cos 2, sin 2) = -sin 1, and a part with itself gives 1.
    Query at position 2 sees tokens 0..2; query at position 3 sees 0..3.
    Raw scores (before the scale 1/2):
      head 0, pos 2: 6 + cos 2,  -2 + sin 1,  2 + 1
      head 0, pos 3: 6 - sin 3,  -2 + cos 2,  2 - sin 1,  4 + 1
      head 1, pos 2: cos 2,  sin 1,  1
      head 1, pos 3: -sin 3,  cos 2,  -sin 1,  1
    o_lat = sum p_t c_t over c = (3, -1, 1, 2); o = W_UV o_lat;
    W_O = [[1, 0], [3, 1]] gives out = (o_0, 3 o_0 + o_1).
    """
    sin, cos, exp, log = math.sin, math.cos, math.exp, math.log
    raw = {(0, 0): [6 + cos(2), -2 + sin(1), 3.0],
           (0, 1): [6 - sin(3), -2 + cos(2), 2 - sin(1), 5.0],
           (1, 0): [cos(2), sin(1), 1.0],
           (1, 1): [-sin(3), cos(2), -sin(1), 1.0]}
    cvals = [3.0, -1.0, 1.0, 2.0]
    W_UV = [1.0, 2.0]
    expect_olat = np.zeros((2, 2, 1))
    expect_lse = np.zeros((2, 2))
    for (i, j), s in raw.items():
        s = [0.5 * v for v in s]
        z = sum(exp(v) for v in s)
        expect_olat[j, i, 0] = sum(exp(v) / z * cvals[t] for t, v in enumerate(s))
        expect_lse[j, i] = log(z)
    o = expect_olat[:, :, 0] * np.array(W_UV)           # [S_q, H]
    expect_out = np.stack([o[:, 0], 3 * o[:, 0] + o[:, 1]], axis=1)

    W = dict(W_Q=np.array([[1., 1.], [1., 0.], [0., 1.], [1., 1.], [1., 0.], [0., 1.]]),
             W_DKV=np.array([[1., 2.]]), W_KR=np.eye(2),
             W_UK=np.array([[[2.]], [[0.]]]), W_UV=np.array([[[1.]], [[2.]]]),
             W_O=np.array([[1., 0.], [3., 1.]]))
    h = np.array([[[1., 0.], [0., 1.]]])
    c_prior = [np.array([[3.], [-1.]])]
    kr_prior = [np.array([[1., 0.], [0., 1.]])]
    for form in ("nonabsorbed", "absorbed"):
        res = oracle.decode_step(h, c_prior, kr_prior, scale=0.5, rope_base=10000.0,
                                 n_heads=2, formulation=form, **W)
        np.testing.assert_allclose(res["o_lat"][0], expect_olat, rtol=0, atol=1e-12)
        np.testing.assert_allclose(res["lse"][0], expect_lse, rtol=0, atol=1e-12)
        np.testing.assert_allclose(res["out"][0], expect_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(res["c_new"][0], [[1.], [2.]], atol=0)
        np.testing.assert_allclose(res["kr_new"][0], [[cos(2), sin(2)], [-sin(3), cos(3)]],
                                   atol=1e-15)
    # the same cache given as already rotated keys
    kr_rot = [np.array([[1., 0.], [-sin(1), cos(1)]])]
    res = oracle.decode_step(h, c_prior, kr_rot, scale=0.5, rope_base=10000.0, n_heads=2,
                             prior_kr_rotated=True, **W)
    np.testing.assert_allclose(res["o_lat"][0], expect_olat, rtol=0, atol=1e-12)
    # a subset of heads: the same numbers for that head, no output projection
    res = oracle.decode_step(h, c_prior, kr_prior, scale=0.5, rope_base=10000.0, n_heads=2,
                             heads=[1], **W)
    np.testing.assert_allclose(res["o_lat"][0][:, 0], expect_olat[:, 1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["lse"][0][:, 0], expect_lse[:, 1], rtol=0, atol=1e-12)
    assert res["out"][0] is None
    # planted in the oracle: the new tokens placed at positions 0..S_q-1
    # instead of L-S_q..L-1 (decode_step builds them with a two-argument
    # arange; the one-argument calls stay correct)
    def arange(*a, **k):
        if len(a) == 2:
            return np.arange(0, a[1] - a[0], **k)
        return np.arange(*a, **k)
    orig_np = om.np
    try:
        om.np = _NumpyWith(arange=arange)
        res = oracle.decode_step(h, c_prior, kr_prior, scale=0.5, rope_base=10000.0,
                                 n_heads=2, **W)
    finally:
        om.np = orig_np
    assert np.abs(res["o_lat"][0] - expect_olat).max() > 1e-3


# --------------------------------------------------------------------------
# RoPE: mistakes planted inside the oracle's own function are caught
# --------------------------------------------------------------------------

class _NumpyWith:
    """numpy with some functions replaced, to plant a slip inside the
    oracle's rope (which reaches numpy through the module's `np`)."""

    def __init__(self, **over):
        self.__dict__.update(over)

    def __getattr__(self, name):
        return getattr(np, name)


@pytest.mark.parametrize("slip", ["sin_sign", "theta_exponent", "angle_units"])
def test_rope_planted_mistakes_are_caught(monkeypatch, slip):
    """Slips planted inside the oracle's rope (through the numpy it calls)
    make it disagree with the complex-exponential closed form."""
    rng = np.random.default_rng(32)
    x = rng.standard_normal(16)
    expect = _rope_complex(x, 37, 10000.0)
    np.testing.assert_allclose(oracle.rope(x, 37, 10000.0), expect, atol=1e-9)
    if slip == "sin_sign":                  # rotating the wrong way
        fake = _NumpyWith(sin=lambda a: -np.sin(a))
    elif slip == "theta_exponent":          # base^(-k/d) instead of base^(-2k/d)
        fake = _NumpyWith(power=lambda a, b: np.power(a, b / 2.0))
    else:                                   # angle taken in degrees
        fake = _NumpyWith(cos=lambda a: np.cos(np.deg2rad(a)),
                          sin=lambda a: np.sin(np.deg2rad(a)))
    monkeypatch.setattr(om, "np", fake)
    got = oracle.rope(x, 37, 10000.0)
    assert np.abs(got - expect).max() > 1e-3


def test_chunk_equals_consecutive_single_token_steps():
    """A prefill chunk (decode_step with S_q = T) equals T single-token steps
    in order, each appending its token's latent and rotated RoPE key to the
    cache before the next: the chunk's causal mask and positions (query j of
    the chunk at position L0 + j) agree with plain sequential decoding."""
    rng = np.random.default_rng(11)
    H, dm, dn, dc, dr, L0, T = 2, 16, 8, 16, 4, 3, 4
    W = dict(W_Q=rng.standard_normal((H * (dn + dr), dm)) / 4,
             W_DKV=rng.standard_normal((dc, dm)) / 4,
             W_KR=rng.standard_normal((dr, dm)) / 4,
             W_UK=rng.standard_normal((H, dn, dc)) / 4,
             W_UV=rng.standard_normal((H, dn, dc)) / 4,
             W_O=rng.standard_normal((dm, H * dn)) / 4)
    scale, base = (dn + dr) ** -0.5, 10000.0
    h = rng.standard_normal((1, T, dm))
    c_prior = rng.standard_normal((L0, dc))
    kr_prior = oracle.rope(rng.standard_normal((L0, dr)), np.arange(L0), base)
    args = (W["W_Q"], W["W_DKV"], W["W_KR"], W["W_UK"], W["W_UV"], W["W_O"], scale, base, H)
    chunk = oracle.decode_step(h, [c_prior], [kr_prior], *args, prior_kr_rotated=True)
    C, KR = c_prior, kr_prior
    for j in range(T):
        one = oracle.decode_step(h[:, j:j + 1], [C], [KR], *args, prior_kr_rotated=True)
        for key in ("o", "o_lat", "lse", "out", "c_new", "kr_new"):
            np.testing.assert_allclose(one[key][0][0], chunk[key][0][j], rtol=1e-12, atol=1e-12)
        C = np.concatenate([C, one["c_new"][0]], 0)
        KR = np.concatenate([KR, one["kr_new"][0]], 0)
