"""fp64 CPU oracle for one decode step of Multi-head Latent Attention (MLA).

TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
baseline leg of the benchmark use this module.  It shares no code, tables or
helpers with the CUDA path and imports nothing from it.

What it follows (page addresses as printed, with their section names):

* deepforge.srivtx.xyz "DeepSeek-V2" page, §1 "Theory from first principles",
  subsection "Store a latent, rebuild the keys and values" and the box
  "MLA: compress once, reconstruct in attention": each token stores one
  latent ``c_t = W_DKV h_t`` (512-dim) plus one 64-dim key that carries RoPE;
  keys and values are rebuilt per head by the up-projections ``k = W_UK c``
  and ``v = W_UV c``; because those maps are linear, ``W_UK`` can be folded
  into the query and ``W_UV`` into the output projection ("absorption").
* Same page, subsection "The bottleneck at inference time": to produce token
  t, the query of t is compared against the keys of all earlier tokens and
  their values are mixed -- plain softmax attention over the cache.
* crackai.dev "DeepSeek-V2" page, "How It Works": up-projections differ per
  head; a small decoupled RoPE key set carries position separately.

The primary path, :func:`attention_nonabsorbed`, does NOT use absorption: it
rebuilds per-head keys ``k_{i,t} = [W_UK,i c_t ; RoPE(k_rope_t)]`` and values
``v_{i,t} = W_UV,i c_t`` explicitly and runs textbook softmax attention.
:func:`attention_absorbed` is the independent absorbed formulation used only
to pin the absorption identity.

Readings of points the pages leave open (the readings R1-R8 of this
library, stated here in full):

* R1  the 64-dim RoPE key is one vector per token, shared by all heads
      (576 = 512 + 64 numbers per token only adds up that way).
* R2  the current query tokens are appended to the cache before attention;
      query j of S_q sits at position L - S_q + j and sees positions <= its own.
* R3  queries come from a dense ``W_Q``: per head ``[q_nope (d_n) ; q_rope (d_r)]``.
* R4  RoPE rotates consecutive pairs (x_2k, x_2k+1) by angle pos * theta_k with
      theta_k = base^(-2k/d_r).
* R6  ``W_UK[i]`` has shape [d_n, d_c] and ``W_UV[i]`` has shape [d_v, d_c]
      (k = W_UK c, v = W_UV c).
* R7  d_v = d_n.
* R8  the RoPE key is ``W_KR h_t`` followed by RoPE at the token's position.
"""

from __future__ import annotations

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------
# Cache-size arithmetic (deepforge page, §1 "The bottleneck at inference time"
# and the cache-size listing after "What the design buys"; crackai page,
# "Key Takeaways for Interviews": MHA caches 2*n_heads*d_head, GQA caches
# 2*n_groups*d_head, MLA caches d_latent plus the small RoPE part).
# ---------------------------------------------------------------------------

def cache_elems_per_token(kind: str, *, n_heads: int = 0, d_head: int = 0,
                          n_groups: int = 0, d_latent: int = 0,
                          d_rope: int = 0) -> int:
    """Numbers cached per token per layer for MHA, GQA or MLA."""
    if kind == "mha":
        return 2 * n_heads * d_head
    if kind == "gqa":
        return 2 * n_groups * d_head
    if kind == "mla":
        return d_latent + d_rope
    raise ValueError(kind)


def dense_cache_bytes(n_heads: int, d_head: int, layers: int, ctx: int,
                      bytes_per: int = 2) -> int:
    """Bytes of a full key+value cache: one key and one value per head."""
    return cache_elems_per_token("mha", n_heads=n_heads, d_head=d_head) \
        * layers * ctx * bytes_per


def mla_cache_bytes(d_latent: int, d_rope: int, layers: int, ctx: int,
                    bytes_per: int = 2) -> int:
    """Bytes of the MLA cache: one latent and one RoPE key per token."""
    return cache_elems_per_token("mla", d_latent=d_latent, d_rope=d_rope) \
        * layers * ctx * bytes_per


def gqa_equivalent_groups(d_latent: int, d_rope: int, d_head: int) -> float:
    """Number of GQA groups whose cache equals the MLA cache per token."""
    return (d_latent + d_rope) / (2.0 * d_head)


# ---------------------------------------------------------------------------
# Elementary steps
# ---------------------------------------------------------------------------

def rope(x, pos, base: float = 10000.0):
    """Rotary position embedding over consecutive pairs (reading R4).

    ``x`` has shape [..., d] with d even; ``pos`` broadcasts against
    ``x.shape[:-1]``.  Pair k, i.e. (x[2k], x[2k+1]), is rotated by the angle
    ``pos * base**(-2k/d)``.  All arithmetic in fp64.
    """
    x = np.asarray(x, dtype=F64)
    d = x.shape[-1]
    if d % 2:
        raise ValueError("RoPE width must be even")
    if d == 0:
        return x.copy()
    k = np.arange(d // 2, dtype=F64)
    theta = np.power(F64(base), -2.0 * k / d)
    ang = np.asarray(pos, dtype=F64)[..., None] * theta
    cos, sin = np.cos(ang), np.sin(ang)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    y = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)), dtype=F64)
    y[..., 0::2] = x0 * cos - x1 * sin
    y[..., 1::2] = x0 * sin + x1 * cos
    return y


def project(x, w):
    """Dense projection y = W x for every row of x (x: [..., in], w: [out, in])."""
    return np.asarray(x, dtype=F64) @ np.asarray(w, dtype=F64).T


def _softmax_attend(scores, values):
    """Textbook softmax with max subtraction; returns (p, out, lse)."""
    m = scores.max()
    e = np.exp(scores - m)
    z = e.sum()
    p = e / z
    return p, p @ values, m + np.log(z)


# ---------------------------------------------------------------------------
# Attention over one sequence's cache
# ---------------------------------------------------------------------------

def attention_nonabsorbed(q, C, KR, W_UK, W_UV, scale):
    """Non-absorbed MLA attention for the S_q query tokens of ONE sequence.

    q    [S_q, H, d_n + d_r]  per-head query, RoPE already applied to the
                              last d_r entries
    C    [L, d_c]             cached latents c_t, t = 0..L-1
    KR   [L, d_r]             cached RoPE keys (already rotated)
    W_UK [H, d_n, d_c], W_UV [H, d_v, d_c]

    For head i the keys are rebuilt as k_{i,t} = [W_UK[i] c_t ; KR_t] and the
    values as v_{i,t} = W_UV[i] c_t.  Query j (position L - S_q + j) attends to
    t <= L - S_q + j.  Returns dict with
      o     [S_q, H, d_v]  attention output per head,
      o_lat [S_q, H, d_c]  sum_t p_t c_t (latent-space output),
      lse   [S_q, H]       natural-log partition of the scaled scores,
      p     list of [S_q][H] probability rows.
    """
    q = np.asarray(q, dtype=F64)
    C = np.asarray(C, dtype=F64)
    KR = np.asarray(KR, dtype=F64)
    S_q, H, _ = q.shape
    L = C.shape[0]
    d_v = W_UV.shape[1]
    d_c = C.shape[1]
    if L < S_q:
        raise ValueError("context shorter than the query block")
    o = np.zeros((S_q, H, d_v))
    o_lat = np.zeros((S_q, H, d_c))
    lse = np.zeros((S_q, H))
    probs = [[None] * H for _ in range(S_q)]
    for i in range(H):
        K_i = np.concatenate([C @ np.asarray(W_UK[i], dtype=F64).T, KR], axis=1)
        V_i = C @ np.asarray(W_UV[i], dtype=F64).T
        for j in range(S_q):
            vis = L - S_q + j + 1
            s = scale * (K_i[:vis] @ q[j, i])
            p, o[j, i], lse[j, i] = _softmax_attend(s, V_i[:vis])
            o_lat[j, i] = p @ C[:vis]
            probs[j][i] = p
    return {"o": o, "o_lat": o_lat, "lse": lse, "p": probs}


def absorb_query(q_nope, W_UK):
    """Fold W_UK into the query: q_lat[..., i, :] = W_UK[i]^T q_nope[..., i, :].

    q_nope [..., H, d_n], W_UK [H, d_n, d_c] -> [..., H, d_c].  With
    k_{i,t} = W_UK[i] c_t, q_nope . k = q_lat . c_t (linearity).
    """
    q_nope = np.asarray(q_nope, dtype=F64)
    W = np.asarray(W_UK, dtype=F64)
    out = np.zeros(q_nope.shape[:-1] + (W.shape[2],))
    for i in range(W.shape[0]):
        out[..., i, :] = q_nope[..., i, :] @ W[i]
    return out


def latent_attention(q_abs, C, KR, scale):
    """Attention run directly on the cache with an absorbed query.

    q_abs [S_q, H, d_c + d_r] = [q_lat ; roped q_rope] per head, C [L, d_c],
    KR [L, d_r].  Score s_t = scale * (q_lat . c_t + q_rope . KR_t), causal as
    in attention_nonabsorbed.  Returns o_lat [S_q, H, d_c] = sum_t p_t c_t and
    lse [S_q, H].
    """
    q_abs = np.asarray(q_abs, dtype=F64)
    C = np.asarray(C, dtype=F64)
    KR = np.asarray(KR, dtype=F64)
    S_q, H, _ = q_abs.shape
    L, d_c = C.shape
    o_lat = np.zeros((S_q, H, d_c))
    lse = np.zeros((S_q, H))
    for j in range(S_q):
        vis = L - S_q + j + 1
        for i in range(H):
            s = scale * (C[:vis] @ q_abs[j, i, :d_c] + KR[:vis] @ q_abs[j, i, d_c:])
            _, o_lat[j, i], lse[j, i] = _softmax_attend(s, C[:vis])
    return {"o_lat": o_lat, "lse": lse}


def latent_attention_range(q_abs, C_rng, KR_rng, scale, first, total):
    """latent_attention restricted to one contiguous range of the cache.

    The sequence has ``total`` tokens (its last S_q are the queries, causal as
    in latent_attention); C_rng [n, d_c] and KR_rng [n, d_r] are its tokens
    first .. first + n - 1.  Query j sees token t when t <= total - S_q + j.
    Returns o_lat and lse over the visible tokens of the range; a row that
    sees none of them gets o_lat = 0 and lse = -inf.  Merging the ranges of a
    partition of the sequence with combine_splits gives latent_attention of
    the whole sequence (the softmax normalisation splits over disjoint token
    sets, the same identity the split-KV merge rests on).
    """
    q_abs = np.asarray(q_abs, dtype=F64)
    C_rng = np.asarray(C_rng, dtype=F64)
    KR_rng = np.asarray(KR_rng, dtype=F64)
    S_q, H, _ = q_abs.shape
    n, d_c = C_rng.shape
    o_lat = np.zeros((S_q, H, d_c))
    lse = np.full((S_q, H), -np.inf)
    for j in range(S_q):
        last_visible = total - S_q + j          # global index
        vis = min(n, max(0, last_visible - first + 1))
        if vis == 0:
            continue
        for i in range(H):
            s = scale * (C_rng[:vis] @ q_abs[j, i, :d_c] + KR_rng[:vis] @ q_abs[j, i, d_c:])
            _, o_lat[j, i], lse[j, i] = _softmax_attend(s, C_rng[:vis])
    return {"o_lat": o_lat, "lse": lse}


def out_proj(o_lat, W_UV, W_O):
    """Output side with W_UV folded in: o_i = W_UV[i] o_lat_i, then
    out = W_O [o_1; ...; o_H].  o_lat [T, H, d_c] -> (o [T, H, d_v], out [T, d_model])."""
    o_lat = np.asarray(o_lat, dtype=F64)
    W = np.asarray(W_UV, dtype=F64)
    o = np.zeros(o_lat.shape[:-1] + (W.shape[1],))
    for i in range(W.shape[0]):
        o[..., i, :] = o_lat[..., i, :] @ W[i].T
    out = project(o.reshape(o.shape[0], -1), W_O)
    return o, out


def attention_absorbed(q, C, KR, W_UK, W_UV, scale):
    """Absorbed formulation of the same attention (identity check only).

    W_UK folds into the query: q_lat_i = W_UK[i]^T q_nope_i, so the score is
    q_lat_i . c_t + q_rope_i . KR_t; W_UV folds into the output:
    o_i = W_UV[i] (sum_t p_t c_t).
    """
    q = np.asarray(q, dtype=F64)
    d_n = W_UK.shape[1]
    q_lat = absorb_query(q[..., :d_n], W_UK)
    att = latent_attention(np.concatenate([q_lat, q[..., d_n:]], axis=-1), C, KR, scale)
    o = np.zeros(att["o_lat"].shape[:-1] + (W_UV.shape[1],))
    for i in range(W_UV.shape[0]):
        o[:, i] = att["o_lat"][:, i] @ np.asarray(W_UV[i], dtype=F64).T
    return {"o": o, "o_lat": att["o_lat"], "lse": att["lse"], "q_lat": q_lat}


# ---------------------------------------------------------------------------
# One whole decode step of a batch
# ---------------------------------------------------------------------------

def decode_step(h_new, c_prior, krpre_prior, W_Q, W_DKV, W_KR, W_UK, W_UV,
                W_O, scale, rope_base, n_heads, seqs=None,
                prior_kr_rotated=False, heads=None, formulation="nonabsorbed"):
    """One MLA decode step for a batch, non-absorbed, fp64.

    h_new        [B, S_q, d_model]   hidden states of the new tokens
    c_prior      list of [L_b - S_q, d_c] latents already cached
    krpre_prior  list of [L_b - S_q, d_r] RoPE keys of those tokens BEFORE
                 rotation (rotated here by their positions 0..)
    W_Q [H*(d_n+d_r), d_model], W_DKV [d_c, d_model], W_KR [d_r, d_model],
    W_UK [H, d_n, d_c], W_UV [H, d_v, d_c], W_O [d_model, H*d_v]
    seqs         optional subset of sequence indices to evaluate
    prior_kr_rotated  the prior RoPE keys are given as cached, i.e. already
                 rotated (workloads that draw the cache directly)
    heads        optional subset of heads for the attention (the output
                 projection needs every head and is then skipped)
    formulation  "nonabsorbed" (default, the reference) or "absorbed" (the
                 pinned-equal absorbed formulation, far cheaper at long
                 context because it never rebuilds keys and values)

    Steps per sequence b (positions per reading R2):
      1. new tokens: c = W_DKV h, kr = RoPE(W_KR h, pos), pos = L-S_q .. L-1
      2. q = W_Q h split per head into [q_nope ; q_rope]; q_rope <- RoPE(q_rope, pos)
      3. non-absorbed attention over the cache (see attention_nonabsorbed)
      4. out = W_O [o_1; ...; o_H]
    Returns dict of per-sequence results keyed by stage name.
    """
    h_new = np.asarray(h_new, dtype=F64)
    B, S_q, _ = h_new.shape
    H = n_heads
    d_c = W_DKV.shape[0]
    d_r = W_KR.shape[0]
    d_qk = W_Q.shape[0] // H
    seqs = range(B) if seqs is None else seqs
    res = {k: {} for k in ("q", "q_roped", "c_new", "kr_new", "o", "o_lat",
                           "lse", "out")}
    for b in seqs:
        Lp = np.asarray(c_prior[b]).shape[0]
        L = Lp + S_q
        pos = np.arange(Lp, L)
        c_new = project(h_new[b], W_DKV)                   # [S_q, d_c]
        kr_new = rope(project(h_new[b], W_KR), pos, rope_base)
        C = np.concatenate([np.asarray(c_prior[b], dtype=F64).reshape(Lp, d_c),
                            c_new], axis=0)
        kr_prior = np.asarray(krpre_prior[b], dtype=F64).reshape(Lp, d_r)
        if not prior_kr_rotated:
            kr_prior = rope(kr_prior, np.arange(Lp), rope_base)
        KR = np.concatenate([kr_prior, kr_new], axis=0)
        q = project(h_new[b], W_Q).reshape(S_q, H, d_qk)
        q_roped = q.copy()
        q_roped[..., d_qk - d_r:] = rope(q[..., d_qk - d_r:], pos[:, None],
                                         rope_base)
        hs = list(range(H)) if heads is None else list(heads)
        attn = attention_nonabsorbed if formulation == "nonabsorbed" \
            else attention_absorbed
        att = attn(q_roped[:, hs], C, KR, np.asarray(W_UK)[hs],
                   np.asarray(W_UV)[hs], scale)
        out = project(att["o"].reshape(S_q, -1), W_O) if heads is None else None
        res["q"][b] = q
        res["q_roped"][b] = q_roped
        res["c_new"][b] = c_new
        res["kr_new"][b] = kr_new
        res["o"][b] = att["o"]
        res["o_lat"][b] = att["o_lat"]
        res["lse"][b] = att["lse"]
        res["out"][b] = out
    return res


# ---------------------------------------------------------------------------
# Paged cache append (deepforge page, §1 box: only c_t and the small RoPE key
# are ever written to memory).  Layout: pool[page, slot, 0:d_c] = c,
# pool[page, slot, d_c:d_c+d_r] = rotated RoPE key; token at position p of
# sequence b lives in page page_table[b][p // page_size], slot p % page_size.
# ---------------------------------------------------------------------------

def cache_append(pool, c, kr, batch_idx, pos, page_table, page_size):
    """Return a copy of ``pool`` with each new token's row written, one by one.

    Works on any dtype (raw bf16 bit patterns as uint16 included); copies the
    values unchanged.
    """
    out = np.array(pool, copy=True)
    d_c = c.shape[1]
    for t in range(c.shape[0]):
        b = int(batch_idx[t])
        p = int(pos[t])
        page = int(page_table[b][p // page_size])
        slot = p % page_size
        out[page, slot, :d_c] = c[t]
        out[page, slot, d_c:] = kr[t]
    return out


def combine_splits(o_parts, lse_parts):
    """Merge per-split attention results by log-sum-exp weighting.

    o_parts [S, ...D] (each split's normalised output), lse_parts [S, ...];
    returns (o, lse) of attention over the union of the splits' tokens.
    Splits whose lse is -inf (no tokens) carry zero weight.
    """
    o_parts = np.asarray(o_parts, dtype=F64)
    lse_parts = np.asarray(lse_parts, dtype=F64)
    m = lse_parts.max(axis=0)
    w = np.exp(lse_parts - m)
    z = w.sum(axis=0)
    o = (w[..., None] * o_parts).sum(axis=0) / z[..., None]
    return o, m + np.log(z)


# ---------------------------------------------------------------------------
# 8-bit latent cache (deepforge page, §4 "Build it yourself", stretch goals:
# quantize the latent to 8 bits and measure the extra error a production
# cache would pay).  The pages fix neither the format nor the scale; the
# reading used here (R16): each token's 512-number latent is stored in the
# 8-bit float format E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa
# bits, largest finite value 448, no infinities) after division by one
# per-token scale s (max|c| / 448, or more when the RoPE key needs it); the
# 64-number RoPE key, divided by the same s, is kept in half precision.  The
# scale and the divisions are single-precision steps (the precision the GPU
# quantizer takes the decision in), so both sides produce the same codes.
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def round_to_grid(x, mant_bits: int, emin: int, max_value: float):
    """Round x to the nearest number of a binary floating-point format with
    `mant_bits` stored mantissa bits and smallest normal exponent `emin`
    (subnormals below 2^emin), ties to even, saturating at +-max_value.

    Inside binade [2^e, 2^(e+1)) the representable numbers are multiples of
    2^(e - mant_bits); below 2^emin they are multiples of 2^(emin - mant_bits).
    """
    x = np.asarray(x, dtype=F64)
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)
    quantum = np.exp2(e - mant_bits)
    q = np.round(a / quantum) * quantum          # numpy rounds halves to even
    q = np.minimum(q, max_value)
    return np.sign(x) * q


def e4m3_round(x):
    """Nearest E4M3 value (3 mantissa bits, normals from 2^-6, max 448)."""
    return round_to_grid(x, 3, -6, E4M3_MAX)


def bf16_round(x):
    """Nearest bfloat16 value (7 stored mantissa bits, 8 exponent bits)."""
    return round_to_grid(x, 7, -126, 3.3895313892515355e38)


def f16_round(x):
    """Nearest IEEE half-precision value (10 stored mantissa bits, normals
    from 2^-14, largest finite 65504)."""
    return round_to_grid(x, 10, -14, 65504.0)


F16_MAX = 65504.0


def quantize_latent_fp8(C, KR):
    """8-bit cache rows of tokens C [L, d_c], KR [L, d_r] (reading R16).

    Per token t, in single precision: one scale for the whole row,
    s_t = max(max_k |C[t, k]| / 448, max_r |KR[t, r]| / 65504) (1 for an
    all-zero row), so that both parts divided by it fit their formats; then
    c8_t = E4M3(C[t] / s_t) and the RoPE key is stored as the half-precision
    number kr8_t = f16(KR[t] / s_t).  Returns (s [L], c8 [L, d_c] E4M3
    values, kr8 [L, d_r] half values); the cache the attention sees is
    s_t [c8_t ; kr8_t] (dequantize_fp8).
    """
    C32 = np.asarray(C, dtype=np.float32)
    K32 = np.asarray(KR, dtype=np.float32)
    mc = np.abs(C32).max(axis=1) if C32.shape[1] else np.zeros(C32.shape[0], np.float32)
    mk = np.abs(K32).max(axis=1) if K32.shape[1] else np.zeros(K32.shape[0], np.float32)
    s = np.maximum(mc / np.float32(E4M3_MAX), mk / np.float32(F16_MAX)).astype(np.float32)
    s = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    c8 = e4m3_round((C32 / s[:, None]).astype(np.float32).astype(F64))
    kr8 = f16_round((K32 / s[:, None]).astype(np.float32).astype(F64))
    return s.astype(F64), c8, kr8


def dequantize_fp8(s, c8, kr8):
    """The cache numbers an 8-bit row stands for: (s c8, s kr8)."""
    s = np.asarray(s, dtype=F64)[:, None]
    return s * np.asarray(c8, dtype=F64), s * np.asarray(kr8, dtype=F64)
