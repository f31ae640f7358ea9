"""Oracle checks of whole workloads, spread over host processes.

The full-size parity tests compare every sequence (or many) of a workload
with the fp64 oracle.  One sequence of 131072 tokens costs the oracle tens of
seconds per query token, so the work is split into (sequence, head range)
tasks run in a pool of `spawn`ed processes (never forked: the parent holds a
CUDA context).  Each task regenerates its sequence's cache from the seeded
generator and runs the oracle's absorbed attention (pinned equal to the
non-absorbed one to 1e-10) on it.  Nothing here imports the CUDA path.
"""

from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

import oracle
from mla_latent_kv_35_b200 import workloads as wl


def _task(args):
    """Oracle attention of one sequence for a range of heads.

    args = (workload, b, heads, q_roped [S_q, H', d_n + d_r], c_new
    [S_q, d_c], kr_new [S_q, d_r], W_UK [H', d_n, d_c], W_UV [H', d_v, d_c],
    cache); the cache is sequence b's drawn prior followed by its new tokens,
    for cache "fp8" quantized to the 8-bit rows and read back
    (oracle.quantize_latent_fp8 / dequantize_fp8).
    Returns (b, heads, o_lat [S_q, H', d_c], lse [S_q, H'], o [S_q, H', d_v]).
    """
    w, b, heads, q_roped, c_new, kr_new, W_UK, W_UV, cache = args
    c, kr = wl.draw_prior(w, b)
    C = np.concatenate([c.astype(np.float64), c_new], 0)
    KR = np.concatenate([kr.astype(np.float64), kr_new], 0)
    if cache == "fp8":
        C, KR = oracle.dequantize_fp8(*oracle.quantize_latent_fp8(C, KR))
    r = oracle.attention_absorbed(q_roped, C, KR, W_UK, W_UV, w.scale)
    return b, heads, r["o_lat"], r["lse"], r["o"]


def n_procs() -> int:
    return max(1, min(16, len(os.sched_getaffinity(0)) - 1))


def workload_reference(w, W, h, seqs, head_chunk=32, cache="bf16"):
    """Oracle o_lat, lse and out of sequences `seqs` of workload w, all heads.

    W: the workload's weights (workloads.draw_weights), h: its new hidden
    states [B, S_q, d_model].  The query side of each sequence (projection,
    RoPE at positions L - S_q .. L - 1, the new tokens' latent and RoPE key)
    comes from the oracle's decode_step on an empty-headed call; the
    attention over the cache runs in the pool.  Returns {b: dict(o_lat, lse,
    out, c_new, kr_new)}.
    """
    seqs = list(seqs)
    per = {}
    tasks = []
    for b in seqs:
        Lp = w.prior[b]
        # decode_step's query side and new-token rows do not depend on the
        # prior's values, only on its length (the positions); a zero prior of
        # that length gives them without drawing the cache here
        z = oracle.decode_step(h[b:b + 1], [np.zeros((Lp, w.d_latent))],
                               [np.zeros((Lp, w.d_rope))], W["W_Q"], W["W_DKV"], W["W_KR"],
                               W["W_UK"], W["W_UV"], W["W_O"], w.scale, w.rope_base, w.H,
                               prior_kr_rotated=True, heads=[0], formulation="absorbed")
        q_roped = z["q_roped"][0]
        per[b] = dict(c_new=z["c_new"][0], kr_new=z["kr_new"][0],
                      o_lat=np.zeros((w.S_q, w.H, w.d_latent)),
                      lse=np.zeros((w.S_q, w.H)), o=np.zeros((w.S_q, w.H, w.d_v)))
        for h0 in range(0, w.H, head_chunk):
            hs = list(range(h0, min(w.H, h0 + head_chunk)))
            tasks.append((w, b, hs, q_roped[:, hs], per[b]["c_new"], per[b]["kr_new"],
                          np.asarray(W["W_UK"])[hs], np.asarray(W["W_UV"])[hs], cache))
    ctx = mp.get_context("spawn")
    with ctx.Pool(n_procs()) as pool:
        for b, hs, o_lat, lse, o in pool.imap_unordered(_task, tasks):
            per[b]["o_lat"][:, hs] = o_lat
            per[b]["lse"][:, hs] = lse
            per[b]["o"][:, hs] = o
    for b in seqs:
        _, out = oracle.out_proj(per[b]["o_lat"], W["W_UV"], W["W_O"])
        per[b]["out"] = out
    return per
