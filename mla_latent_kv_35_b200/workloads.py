"""Seeded synthetic inputs for the MLA decode workloads.

This module only draws random numbers and lays out pages; it holds none of
the attention arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from it.  Every array is float32 on the host.  For bf16
workloads the values are rounded to the nearest bf16 (ties to even) here,
once, so both sides consume exactly the same numbers.

Shapes follow DeepSeek-V2's attention (deepforge "DeepSeek-V2" page, §1 "Store
a latent, rebuild the keys and values": 128 heads of width 128, a 512-dim
latent and a 64-dim RoPE key per token).  Seven workloads:

  tiny       fp32: B=2, H=8, d_model 256, d_nope 32, latent 64, rope 16,
             contexts {37, 64}, prior cache built from hidden states
  dsv2       bf16: B=16, H=128, d_model 5120, L=4096, sequential pages
  batch128   bf16: B=128, L=32768, 64-token pages in a permuted pool
  ragged     bf16: B=64, prior lengths log-uniform in [128, 65536] (seed 7),
             one new token appended per sequence, permuted pages
  long1/long4 bf16: B=1 / B=4, L=131072 including 2 speculative query tokens
  prefill    bf16: one sequence, a chunk of 4096 new tokens after 4096 cached
             ones (the chunk's tokens are the S_q query tokens)

Random streams: every array has its own stream,
``default_rng(SeedSequence([seed, stream, index]))``, so one sequence's
cache can be regenerated alone (the oracle's sampled checks rely on this).
"""

from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

PAGE_SIZE = 64

# stream ids
_S_H, _S_WDKV, _S_WUK, _S_WUV, _S_WQ, _S_WO, _S_LAT, _S_KR, _S_PERM, \
    _S_LEN, _S_HCTX, _S_PEAK = range(12)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S_q: int
    H: int
    d_model: int
    d_nope: int
    d_latent: int
    d_rope: int
    ctx: tuple            # total context per sequence, new tokens included
    dtype: str            # "f32" or "bf16"
    seed: int = 0
    permute_pages: bool = False
    prior_from_h: bool = False   # tiny: prior cache comes from hidden states
    rope_base: float = 10000.0
    page_size: int = PAGE_SIZE
    peaky: bool = False
    seq_offset: int = 0          # global index of this batch's sequence 0
    global_B: int = 0            # sequences in the whole (sharded) batch; 0 = B
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def d_v(self) -> int:          # value head width = d_nope (reading R7)
        return self.d_nope

    @property
    def D(self) -> int:            # cached numbers per token
        return self.d_latent + self.d_rope

    @property
    def scale(self) -> float:      # 1/sqrt(d_nope + d_rope)
        return 1.0 / math.sqrt(self.d_nope + self.d_rope)

    @property
    def T(self) -> int:
        return self.B * self.S_q

    @property
    def prior(self) -> list:
        return [L - self.S_q for L in self.ctx]

    @property
    def pages_per_seq(self) -> list:
        return [-(-L // self.page_size) for L in self.ctx]


def _ragged_lengths(B, seed):
    rng = np.random.default_rng(np.random.SeedSequence([seed, _S_LEN]))
    u = rng.uniform(math.log(128.0), math.log(65536.0), size=B)
    return [int(math.floor(math.exp(x))) for x in u]


def workload(name: str, **over) -> Workload:
    """Return one of the named workloads (optionally with fields replaced)."""
    big = dict(H=128, d_model=5120, d_nope=128, d_latent=512, d_rope=64,
               dtype="bf16")
    if name == "tiny":
        w = Workload("tiny", B=2, S_q=1, H=8, d_model=256, d_nope=32,
                     d_latent=64, d_rope=16, ctx=(37, 64), dtype="f32",
                     prior_from_h=True)
    elif name == "dsv2":
        w = Workload("dsv2", B=16, S_q=1, ctx=(4096,) * 16, **big)
    elif name == "batch128":
        w = Workload("batch128", B=128, S_q=1, ctx=(32768,) * 128,
                     permute_pages=True, **big)
    elif name == "ragged":
        lens = _ragged_lengths(64, 7)
        w = Workload("ragged", B=64, S_q=1, ctx=tuple(L + 1 for L in lens),
                     permute_pages=True, extra={"len_seed": 7}, **big)
    elif name in ("long1", "long4"):
        B = 1 if name == "long1" else 4
        w = Workload(name, B=B, S_q=2, ctx=(131072,) * B,
                     permute_pages=True, **big)
    elif name == "prefill":
        # one sequence: 4096 cached tokens, then a chunk of 4096 new ones
        w = Workload("prefill", B=1, S_q=4096, ctx=(8192,), permute_pages=True, **big)
    else:
        raise KeyError(name)
    return replace(w, **over) if over else w


WORKLOADS = ("tiny", "dsv2", "batch128", "ragged", "long1", "long4", "prefill")


def shard(w: Workload, rank: int, world: int) -> Workload:
    """Rank `rank`'s share of a batch of world * w.B sequences (weak scaling).

    The whole batch is the named workload grown to world * B sequences; rank r
    takes global sequences [r * B, r * B + B).  Each sequence's cache and
    hidden state come from streams keyed by its global index, so a shard's
    sequences are the same numbers wherever they run, rank 0's shard is the
    unsharded workload, and the ranks' sequences differ.  Weights are shared.
    """
    if world <= 1:
        return w
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    ctx = w.ctx
    if "len_seed" in w.extra:
        lens = _ragged_lengths(world * w.B, w.extra["len_seed"])
        ctx = tuple(L + w.S_q for L in lens[rank * w.B:(rank + 1) * w.B])
    return replace(w, ctx=ctx, seq_offset=rank * w.B, global_B=world * w.B,
                   name=f"{w.name}[rank {rank} of {world}]")


# ---------------------------------------------------------------------------
# bf16 rounding of inputs (ties to even), done once on the host
# ---------------------------------------------------------------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 array -> uint16 bf16 bit patterns, round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def _quant(w: Workload, x: np.ndarray) -> np.ndarray:
    return bf16_to_f32(bf16_bits(x)) if w.dtype == "bf16" else \
        np.asarray(x, dtype=np.float32)


def _rng(w: Workload, stream: int, idx: int = 0):
    return np.random.default_rng(np.random.SeedSequence([w.seed, stream, idx]))


def _normal(w, stream, shape, std=1.0, idx=0):
    x = _rng(w, stream, idx).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


# ---------------------------------------------------------------------------
# Draws
# ---------------------------------------------------------------------------

def draw_weights(w: Workload) -> dict:
    """All projection weights, each ~ N(0, 1/fan_in) (reading R6/R8).

    W_Q [H*(d_n+d_r), d_model]; W_DKV [d_c, d_model] and W_KR [d_r, d_model]
    come from one [(d_c+d_r), d_model] draw; W_UK [H, d_n, d_c];
    W_UV [H, d_v, d_c]; W_O [d_model, H*d_v].
    """
    H, dm, dn, dc, dr = w.H, w.d_model, w.d_nope, w.d_latent, w.d_rope
    wdkr = _normal(w, _S_WDKV, (dc + dr, dm), 1.0 / math.sqrt(dm))
    out = {
        "W_DKV": wdkr[:dc],
        "W_KR": wdkr[dc:],
        "W_UK": _normal(w, _S_WUK, (H, dn, dc), 1.0 / math.sqrt(dc)),
        "W_UV": _normal(w, _S_WUV, (H, w.d_v, dc), 1.0 / math.sqrt(dc)),
        "W_Q": _normal(w, _S_WQ, (H * (dn + dr), dm), 1.0 / math.sqrt(dm)),
        "W_O": _normal(w, _S_WO, (dm, H * w.d_v), 1.0 / math.sqrt(H * w.d_v)),
    }
    return {k: _quant(w, v) for k, v in out.items()}


def draw_h_new(w: Workload) -> np.ndarray:
    """Hidden states of the new tokens, [B, S_q, d_model] ~ N(0, 1)."""
    gB = w.global_B or w.B
    h = _normal(w, _S_H, (gB, w.S_q, w.d_model))[w.seq_offset:w.seq_offset + w.B]
    if w.peaky:
        h *= np.float32(4.0)
    return _quant(w, h)


def draw_h_ctx(w: Workload, b: int) -> np.ndarray:
    """Hidden states of sequence b's prior tokens (tiny workload only)."""
    return _quant(w, _normal(w, _S_HCTX, (w.prior[b], w.d_model), idx=w.seq_offset + b))


def draw_prior(w: Workload, b: int):
    """Sequence b's prior cache drawn directly: (latents [Lp, d_c],
    pre-RoPE keys [Lp, d_r]), both ~ N(0, 1), rounded for bf16."""
    Lp = w.prior[b]
    g = w.seq_offset + b
    c = _normal(w, _S_LAT, (Lp, w.d_latent), idx=g)
    kr = _normal(w, _S_KR, (Lp, w.d_rope), idx=g)
    if w.peaky and Lp > 0:
        t = int(_rng(w, _S_PEAK, g).integers(0, Lp))
        c[t] *= np.float32(6.0)
    return _quant(w, c), _quant(w, kr)


def draw_prior_bits(w: Workload, b: int) -> np.ndarray:
    """Sequence b's prior cache rows [Lp, d_c + d_r] as bf16 bit patterns
    (uint16), same values as draw_prior."""
    c, kr = draw_prior(w, b)
    return bf16_bits(np.concatenate([c, kr], axis=1))


def draw_prior_all(w: Workload, seqs=None, threads: int = 8):
    """draw_prior for many sequences, in parallel threads."""
    seqs = list(range(w.B)) if seqs is None else list(seqs)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(lambda b: draw_prior(w, b), seqs))


def page_layout(w: Workload):
    """Page table [B, max_pages] int32 and pool size.

    Sequence b's k-th 64-token page is pool page ``table[b, k]``.  Pages of all
    sequences are distinct; with ``permute_pages`` their order in the pool is
    a seeded random permutation.  One extra page at the end of the pool is
    never referenced (canary slack).  Unused table entries hold -1.
    """
    n = w.pages_per_seq
    total = int(sum(n))
    if w.permute_pages:
        perm = _rng(w, _S_PERM, w.seq_offset).permutation(total).astype(np.int32)
    else:
        perm = np.arange(total, dtype=np.int32)
    table = np.full((w.B, max(n)), -1, dtype=np.int32)
    off = 0
    for b, nb in enumerate(n):
        table[b, :nb] = perm[off:off + nb]
        off += nb
    return table, total + 1


def positions(w: Workload):
    """(batch_idx [T], pos [T]) of the new query tokens, b-major."""
    bi = np.repeat(np.arange(w.B, dtype=np.int32), w.S_q)
    pos = np.concatenate([np.arange(L - w.S_q, L, dtype=np.int32)
                          for L in w.ctx])
    return bi, pos
