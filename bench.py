"""Benchmark of one MLA decode step (A0-A6) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

A step is one pass of the whole hot path over one batch: projection (A0),
RoPE (A2), cache append (A3), query absorption (A1), split-KV decode on the
paged latent cache with LSE combine (A4+A5) and the output projection (A6),
enqueued through the C ABI on one stream.  Inputs are seeded synthetic data of
the DeepSeek-V2 attention shapes (workloads.py); the default workload is
`batch128` (B=128, 128 heads, latent 512 + RoPE 64, context 32768 in 64-token
pages scattered by a seeded permutation): its 4.83 GB cache is far larger
than the 126 MB L2, so no flush is needed between steps.

Prints ONE JSON line (rank 0).  `value` is decode tokens per second of the
whole step (B*S_q query tokens per step, summed over ranks); `roofline`
describes the decode call (split kernel + combine); `e2e` repeats the
measurement through the same public API with host buffers (inputs copied in
from pinned memory and the output copied back inside the timed region).
With --gpus N > 1 every rank runs its own batch (independent sequences, no
data-path collective: weak scaling).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


FP8_ROW_BYTES = 656   # E4M3 latent, f16 RoPE key, fp32 scale, padding


def _workload_bytes(w, cache_kind="bf16"):
    """Algorithmic bytes and FLOPs of the decode call (A4+A5) per step.  The
    cache is read once: D bf16 numbers per token, or one 656-byte row of the
    8-bit cache."""
    D = w.D
    vis = []
    for L in w.ctx:
        for j in range(w.S_q):
            vis.append(L - w.S_q + j + 1)
    cache = sum(w.ctx) * (FP8_ROW_BYTES if cache_kind == "fp8" else D * 2)
    q = w.T * w.H * D * 2
    out = w.T * w.H * (w.d_latent + 1) * 4
    flops = 2 * w.H * (D + w.d_latent) * sum(vis)
    return cache + q + out, flops, cache


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running.
    Entering waits for nvidia-smi's first sample; summary() keeps only the
    samples taken after mark(), i.e. during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.t_mark = 0.0

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "25"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t0 = time.perf_counter()
            while not self.lines and time.perf_counter() - t0 < 3.0:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def mark(self):
        self.t_mark = time.perf_counter()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, ln in self.lines:
            if t < self.t_mark:
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def code_digest(paths):
    """sha256 of the sources with comments and blank lines removed, so an
    edit to comments alone does not count as a kernel change."""
    import re
    h = hashlib.sha256()
    for p in paths:
        with open(p) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for line in src.split("\n"):
            line = line.strip()
            if line:
                h.update(line.encode() + b"\n")
    return h.hexdigest()


def _traffic_for(kernel_src_paths, record="decode_tc_traffic.json"):
    """ncu DRAM bytes per call recorded in profiles/, if the kernel code is
    unchanged since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", record)
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("code_sha256") != code_digest(kernel_src_paths):
        return None
    return rec.get("dram_bytes_per_call")


L2_BYTES = 126 * 1024 * 1024
L2_FLUSH_BYTES = 2 * L2_BYTES


def flush_needed(w, cache_kind="bf16"):
    """The decode call reads only the cache (plus small q and outputs): when
    the cache is under twice the L2 size, repeated calls would be served
    partly from L2, so the bench flushes L2 between timed calls."""
    _, _, cache_bytes = _workload_bytes(w, cache_kind)
    return cache_bytes < 2 * L2_BYTES


def run_config(w, workload_name, world, flush=None, cache_kind="bf16"):
    """The JSON line's `config`, shared by both arms."""
    _, _, cache_bytes = _workload_bytes(w, cache_kind)
    flush = flush_needed(w, cache_kind) if flush is None else flush
    l2 = ("L2 flushed (%d MB write) before every timed call; cache %.3f GB"
          % (L2_FLUSH_BYTES >> 20, cache_bytes / 1e9) if flush else
          "inputs larger than L2 (cache %.2f GB), no flush" % (cache_bytes / 1e9))
    return {"workload": workload_name, "batch_per_gpu": w.B, "global_batch": w.B * world,
            "heads": w.H, "context": w.ctx[0] if len(set(w.ctx)) == 1 else "ragged",
            "S_q": w.S_q, "latent": w.d_latent, "rope": w.d_rope, "page": w.page_size,
            "d_model": w.d_model,
            "cache": ("8-bit latent cache: E4M3 latent, f16 RoPE key, fp32 row scale, 656 B "
                      "per token" if cache_kind == "fp8" else "bf16, 1152 B per token"),
            "l2": l2,
            "parallelism": (f"dp{world}: independent sequence shards, no collective"
                            if world > 1 else "single GPU")}


def max_over_ranks(vals, device=None):
    """Element-wise maximum of `vals` over all ranks of the default process
    group (the values themselves when there is no group or one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank, world, ms):
    """Units per second of the whole job: every rank's units over the
    slowest rank's time (ms)."""
    return units_per_rank * world / (ms * 1e-3)


# ---------------------------------------------------------------------------
# CPU oracle arm
# ---------------------------------------------------------------------------
def _oracle_sample(w, budget_s=25.0):
    """Time the oracle's decode step on whole sequences of the workload until
    about budget_s seconds of CPU work; returns (tokens/s, sample text, cores)."""
    import oracle
    from mla_latent_kv_35_b200 import workloads as wl
    W = wl.draw_weights(w)
    h = wl.draw_h_new(w)
    cores = len(os.sched_getaffinity(0))
    t_total, toks, seqs = 0.0, 0, 0
    for b in range(w.B):
        c, kr = wl.draw_prior(w, b)
        t0 = time.perf_counter()
        oracle.decode_step(h[b:b + 1], [c], [kr], W["W_Q"], W["W_DKV"], W["W_KR"], W["W_UK"],
                           W["W_UV"], W["W_O"], w.scale, w.rope_base, w.H,
                           prior_kr_rotated=True)
        t_total += time.perf_counter() - t0
        toks += w.S_q
        seqs += 1
        if t_total >= budget_s:
            break
    sample = (f"{seqs} of {w.B} sequences of {w.name} (context {w.ctx[0]}), all {w.H} heads, "
              f"fp64 non-absorbed oracle, {t_total:.1f} s")
    return toks / t_total, sample, cores, t_total


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    tps = []
    sample = ""
    cores = len(os.sched_getaffinity(0))
    budget = max(5.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        v, sample, cores, _ = _oracle_sample(w, budget_s=budget)
        if i >= args.warmup:
            tps.append(v)
    value = statistics.mean(tps)
    line = {
        "impl": "reference",
        "metric": "MLA decode tokens/s (one attention layer, whole step A0-A6)",
        "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * w.T / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": run_config(w, w.name, args.gpus, cache_kind=args.cache),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_gpu(args, w):
    import torch
    import torch.distributed as dist
    from mla_latent_kv_35_b200 import binding as B
    from mla_latent_kv_35_b200 import build as _build
    from mla_latent_kv_35_b200 import workloads as wl
    from mla_latent_kv_35_b200.engine import (DecodePipeline, MLADecodeLayer, build_pool_host,
                                               build_pool_host_drawn, pool_to_device)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    # launched by torchrun (any world size): one NCCL process group
    distributed = "WORLD_SIZE" in os.environ
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if distributed:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    # weak scaling: this rank's own sequences of a world * B batch
    workload_name = w.name
    w = wl.shard(w, rank, world)
    if rank == 0:
        _build.build()
    if distributed:
        dist.barrier()
    B.lib()

    d = B.MLADims.of(w)
    W = wl.draw_weights(w)
    layer = MLADecodeLayer(d, W, dev)
    table, n_pages = wl.page_layout(w)
    if w.prior_from_h:
        host = build_pool_host(w, table, n_pages, [np.zeros((0, w.D), np.float32)] * w.B)
    else:
        host = build_pool_host_drawn(w, table, n_pages)
    pool = pool_to_device(host, w.dtype, dev)
    del host
    if args.cache == "fp8":
        # the 8-bit cache: the same rows, quantized on the GPU
        pool8 = torch.empty((n_pages, w.page_size, FP8_ROW_BYTES), dtype=torch.uint8, device=dev)
        B.mla_cache_quantize_fp8(d, pool, pool8, n_pages)
        del pool
        pool = pool8
    layer.set_cache(pool, torch.from_numpy(table).to(dev),
                    torch.tensor(w.ctx, dtype=torch.int32, device=dev), kind=args.cache)
    if w.prior_from_h:
        layer.prefill_from_hidden([wl.draw_h_ctx(w, b) for b in range(w.B)])
    h_np = wl.draw_h_new(w).reshape(w.T, w.d_model)
    bi_np, pos_np = wl.positions(w)
    h = torch.from_numpy(h_np).to(dev, d.torch_dtype)
    bi = torch.from_numpy(bi_np).to(dev)
    pos = torch.from_numpy(pos_np).to(dev)
    stream = torch.cuda.current_stream(dev)

    def eager_step():
        layer.step(h, bi, pos, w.B, w.S_q)

    # the decode call alone, with events on the launching stream
    bf = layer.buffers(w.B, w.S_q)

    decode_call = B.mla_decode_fp8 if args.cache == "fp8" else B.mla_decode

    def decode_only():
        decode_call(d, bf["qbuf"], layer.pool, layer.n_pages, layer.page_table,
                    layer.max_pages, layer.seq_lens, w.B, w.S_q, 0, bf["ws"], bf["o_lat"],
                    bf["lse"])

    for _ in range(args.warmup):
        eager_step()
    torch.cuda.synchronize(dev)
    st = B.mla_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {B.mla_status_string(st)}")
    # the timed step is a CUDA graph of the whole step (captured once, replayed)
    graph, gbuf, kernels_per_step = layer.capture(h, bi, pos, w.B, w.S_q)

    def step():
        graph.replay()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    # L2 flush between timed calls when the decode's inputs fit in L2: a
    # write of twice the L2 size, outside every timed region
    flush = args.flush_l2 == "on" or (args.flush_l2 == "auto" and flush_needed(w, args.cache))
    flush_buf = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.int32, device=dev) \
        if flush else None

    def timed(fn, K, end=None):
        """K calls timed with CUDA events on the launching stream (barrier +
        synchronize on both sides); `end` makes that stream wait for work the
        calls left on other streams.  Without a flush the K calls run back to
        back between one pair of events; with it, each call has its own pair
        and an L2 flush runs before it, outside the pair.  Returns the mean ms
        per call, the wall time and this process's kernel launches."""
        if distributed:
            dist.barrier()
        torch.cuda.synchronize(dev)
        l0 = B.mla_launch_count()
        t0 = time.perf_counter()
        if flush_buf is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(K):
                fn()
            if end is not None:
                end()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1)
        else:
            pairs = []
            for _ in range(K):
                flush_buf.add_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                if end is not None:
                    end()
                e1.record(stream)
                pairs.append((e0, e1))
            torch.cuda.synchronize(dev)
            ms = sum(a.elapsed_time(b) for a, b in pairs)
        wall = time.perf_counter() - t0
        launches = B.mla_launch_count() - l0
        if distributed:
            dist.barrier()
        return ms / K, wall, launches

    # end to end through the public API with host buffers
    h_host = torch.from_numpy(h_np).to(d.torch_dtype).pin_memory()
    bi_host = torch.from_numpy(bi_np).pin_memory()
    pos_host = torch.from_numpy(pos_np).pin_memory()
    out_host = torch.empty((w.T, w.d_model), dtype=torch.float32).pin_memory()

    # every step copies its inputs in and its output out; DecodePipeline
    # overlaps those transfers with the neighbouring steps' compute
    pipe = DecodePipeline(layer, w.B, w.S_q)
    out_hosts = [out_host, torch.empty_like(out_host).pin_memory()]
    n_e2e = [0]

    def e2e_step():
        pipe.submit(h_host, bi_host, pos_host, out_hosts[n_e2e[0] % 2])
        n_e2e[0] += 1

    def e2e_end():
        pipe.drain(stream)

    for _ in range(4):
        e2e_step()
    pipe.wait()
    torch.cuda.synchronize(dev)

    with ClockSampler(local) as clk:
        clk.mark()
        step_ms, wall, _ = timed(step, args.steps)
        launches = kernels_per_step * args.steps
        n_eager = max(3, args.steps // 4)
        eager_ms, _, eager_launches = timed(eager_step, n_eager)
        dec_ms, _, dec_launches = timed(decode_only, max(args.steps, 5))
        e2e_ms, _, _ = timed(e2e_step, args.steps, end=e2e_end)
    clocks = clk.summary()
    st = B.mla_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {B.mla_status_string(st)}")
    h2d = h_host.numel() * h_host.element_size() + bi_host.numel() * 4 + pos_host.numel() * 4
    d2h = out_host.numel() * 4

    # max over ranks
    t_step, t_dec, t_e2e, t_eager = step_ms, dec_ms, e2e_ms, eager_ms
    t_step, t_dec, t_e2e, t_eager = max_over_ranks([t_step, t_dec, t_e2e, t_eager], dev)

    hbm_peak, tf_peak, peak_kind = _peaks()
    alg_bytes, flops, cache_bytes = _workload_bytes(w, args.cache)
    achieved = alg_bytes / (t_dec * 1e-3) / 1e9
    roof_t = max(alg_bytes / (hbm_peak * 1e9), flops / (tf_peak * 1e12))
    csrc = os.path.join(ROOT, "mla_latent_kv_35_b200", "csrc")
    # the record holds the batch128 call's DRAM bytes (an 8-sequence capture
    # scaled by 16): valid for that workload and kernel only
    traffic = (_traffic_for([os.path.join(csrc, "decode_tc.cuh")])
               if args.cache == "bf16" and workload_name == "batch128" and w.B == 128
               and world == 1 else None)
    line = {
        "metric": "MLA decode tokens/s (one attention layer, whole step A0-A6)",
        "value": whole_job_rate(w.T, world, t_step),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("bf16 (E4M3 cache, f16 decode MMAs)" if args.cache == "fp8" else
                  "bf16" if w.dtype == "bf16" else "f32"),
        "data": "synthetic",
        "config": run_config(w, workload_name, world, flush, args.cache),
        "decode": {"ms": t_dec, "tokens_per_s": whole_job_rate(w.T, world, t_dec),
                   "cache_gb_per_s": cache_bytes / (t_dec * 1e-3) / 1e9,
                   "tflops": flops / (t_dec * 1e-3) / 1e12,
                   "roofline_ms": roof_t * 1e3, "frac_of_roofline": roof_t / (t_dec * 1e-3)},
        "roofline": {"kernel": ("mla_decode_fp8 (decode_fp8_kernel + combine)"
                                if args.cache == "fp8" else
                                "mla_decode (decode_tc_kernel + combine)"), "bound": "hbm",
                     "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_source": peak_kind,
                     "alg_bytes_per_launch": alg_bytes, "traffic": traffic},
        "e2e": {"value": whole_job_rate(w.T, world, t_e2e), "unit": "tokens/s",
                "ms_per_step": t_e2e, "pipelined": True,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "step": {"cuda_graph": True, "kernels_per_step": kernels_per_step,
                 "eager_ms_per_step": t_eager,
                 "eager_launches_per_step": eager_launches / n_eager},
        "clocks": clocks,
        "wall_s_timed": wall,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, cores, _ = _oracle_sample(w, budget_s=20.0)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, pipe
    if distributed:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# Chunked prefill (non-absorbed): one chunk of T new tokens of one sequence
# ---------------------------------------------------------------------------
def prefill_flops(w):
    """Algorithmic FLOPs of one chunk per stage (multiply-add = 2): the A0
    projection, the K/V rebuild of all L tokens, the causal attention (query
    j sees L - T + j + 1 tokens; QK over d_nope + d_rope, PV over d_v) and
    the W_O projection."""
    T, L, H = w.S_q, w.ctx[0], w.H
    Y = H * (w.d_nope + w.d_rope) + w.D
    pairs = sum(L - T + j + 1 for j in range(T))
    return {"a0": 2.0 * T * w.d_model * Y,
            "rebuild": 2.0 * L * H * (w.d_nope + w.d_v) * w.d_latent,
            "attention": 2.0 * pairs * H * (w.d_nope + w.d_rope + w.d_v),
            "w_o": 2.0 * T * H * w.d_v * w.d_model}


def prefill_config(w, world):
    return {"workload": w.name, "chunk_tokens": w.S_q, "cached_before": w.ctx[0] - w.S_q,
            "context_after": w.ctx[0], "heads": w.H, "d_nope": w.d_nope, "d_rope": w.d_rope,
            "d_v": w.d_v, "latent": w.d_latent, "d_model": w.d_model, "page": w.page_size,
            "form": "non-absorbed: K/V rebuilt per head from the latent cache",
            "l2": "inputs larger than L2 (rebuilt K/V %.0f MB, weights %.0f MB), no flush"
                  % (w.ctx[0] * w.H * (w.d_nope + w.d_v) * 2 / 1e6,
                     2 * (w.H * (w.d_nope + w.d_rope) * w.d_model + w.D * w.d_model
                          + 2 * w.H * 128 * w.d_latent + w.d_model * w.H * w.d_v) / 1e6),
            "parallelism": (f"dp{world}: one sequence per rank, no collective"
                            if world > 1 else "single GPU")}


def _oracle_prefill_sample(w, n=128):
    """The oracle on the first n tokens of the chunk: by causality they are
    computed exactly as in the whole chunk (same prior, same positions).
    Returns (tokens/s, sample text, cores, seconds)."""
    import oracle
    from mla_latent_kv_35_b200 import workloads as wl
    W = wl.draw_weights(w)
    h = wl.draw_h_new(w)[:, :n]
    c, kr = wl.draw_prior(w, 0)
    cores = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    oracle.decode_step(h, [c], [kr], W["W_Q"], W["W_DKV"], W["W_KR"], W["W_UK"], W["W_UV"],
                       W["W_O"], w.scale, w.rope_base, w.H, prior_kr_rotated=True)
    t = time.perf_counter() - t0
    sample = (f"first {n} of {w.S_q} chunk tokens of {w.name} (causally identical to the whole "
              f"chunk's), all {w.H} heads, fp64 non-absorbed oracle, {t:.1f} s; the oracle "
              f"rebuilds every head's keys and values for this sample alone, which the whole "
              f"chunk would share")
    return n / t, sample, cores, t


def run_reference_prefill(args, w):
    if int(os.environ.get("RANK", "0")) != 0:
        return
    tps = []
    sample, cores = "", len(os.sched_getaffinity(0))
    for i in range(args.warmup + args.steps):
        v, sample, cores, _ = _oracle_prefill_sample(w, n=32)
        if i >= args.warmup:
            tps.append(v)
    value = statistics.mean(tps)
    line = {
        "impl": "reference",
        "metric": "MLA chunked-prefill tokens/s (one attention layer, whole chunk P0-P3)",
        "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * w.S_q / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": prefill_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_gpu_prefill(args, w):
    import torch
    import torch.distributed as dist
    from mla_latent_kv_35_b200 import binding as B
    from mla_latent_kv_35_b200 import build as _build
    from mla_latent_kv_35_b200 import workloads as wl
    from mla_latent_kv_35_b200.engine import (MLADecodeLayer, PrefillPipeline, build_pool_host,
                                               pool_to_device)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    distributed = "WORLD_SIZE" in os.environ
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if distributed:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    # weak scaling: every rank prefills its own sequence (global index rank)
    w = wl.shard(w, rank, world)
    if rank == 0:
        _build.build()
    if distributed:
        dist.barrier()
    B.lib()
    d = B.MLADims.of(w)
    W = wl.draw_weights(w)
    layer = MLADecodeLayer(d, W, dev)
    table, n_pages = wl.page_layout(w)
    pool = pool_to_device(build_pool_host(w, table, n_pages, [wl.draw_prior_bits(w, 0)]),
                          w.dtype, dev)
    layer.set_cache(pool, torch.from_numpy(table).to(dev),
                    torch.tensor(w.ctx, dtype=torch.int32, device=dev))
    T, L = w.S_q, w.ctx[0]
    h_np = wl.draw_h_new(w).reshape(T, w.d_model)
    bi_np, pos_np = wl.positions(w)
    h = torch.from_numpy(h_np).to(dev, d.torch_dtype)
    bi = torch.from_numpy(bi_np).to(dev)
    pos = torch.from_numpy(pos_np).to(dev)
    stream = torch.cuda.current_stream(dev)
    bf = layer.prefill_buffers(T, L)

    def step():
        layer.prefill_chunk(h, pos, bi, 0, T, L)

    def attention_only():
        B.mla_prefill_attention(d, bf["y"], layer.Y, bf["ctx"], bf["k_nope"], bf["v"], T, L,
                                bf["o"], bf["lse"])

    h_host = torch.from_numpy(h_np).to(d.torch_dtype).pin_memory()
    bi_host = torch.from_numpy(bi_np).pin_memory()
    pos_host = torch.from_numpy(pos_np).pin_memory()
    out_host = torch.empty((T, w.d_model), dtype=d.torch_dtype).pin_memory()
    # every chunk copies its inputs in and its output out; PrefillPipeline
    # overlaps those transfers with the neighbouring chunks' compute
    pipe = PrefillPipeline(layer, 0, T, L)
    out_hosts = [out_host, torch.empty_like(out_host).pin_memory()]
    n_e2e = [0]

    def e2e_step():
        pipe.submit(h_host, bi_host, pos_host, out_hosts[n_e2e[0] % 2])
        n_e2e[0] += 1

    def e2e_end():
        pipe.drain(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = B.mla_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {B.mla_status_string(st)}")

    for _ in range(4):
        e2e_step()
    pipe.wait()
    torch.cuda.synchronize(dev)

    def timed(fn, K, end=None):
        if distributed:
            dist.barrier()
        torch.cuda.synchronize(dev)
        l0 = B.mla_launch_count()
        t0 = time.perf_counter()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            fn()
        if end is not None:
            end()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - t0
        launches = B.mla_launch_count() - l0
        if distributed:
            dist.barrier()
        return e0.elapsed_time(e1) / K, wall, launches

    with ClockSampler(local) as clk:
        clk.mark()
        step_ms, wall, launches = timed(step, args.steps)
        att_ms, _, _ = timed(attention_only, max(args.steps, 5))
        e2e_ms, _, _ = timed(e2e_step, args.steps, end=e2e_end)
    clocks = clk.summary()
    st = B.mla_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {B.mla_status_string(st)}")
    t_step, t_att, t_e2e = max_over_ranks([step_ms, att_ms, e2e_ms], dev)
    _, tf_peak, peak_kind = _peaks()
    fl = prefill_flops(w)
    achieved = fl["attention"] / (t_att * 1e-3) / 1e12
    h2d = h_host.numel() * h_host.element_size() + bi_host.numel() * 4 + pos_host.numel() * 4
    d2h = out_host.numel() * out_host.element_size()
    line = {
        "metric": "MLA chunked-prefill tokens/s (one attention layer, whole chunk P0-P3)",
        "value": whole_job_rate(T, world, t_step),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": prefill_config(w, world),
        "step_tflops": sum(fl.values()) / (t_step * 1e-3) / 1e12,
        "roofline": {"kernel": "mla_prefill_attention (prefill_attn_kernel)", "bound": "tensor",
                     "achieved": achieved, "peak": tf_peak, "unit": "TFLOP/s",
                     "frac": achieved / tf_peak, "peak_source": peak_kind + " (bf16 burst)",
                     "alg_flops_per_launch": fl["attention"], "kernel_ms": t_att,
                     "traffic": _traffic_for([os.path.join(ROOT, "mla_latent_kv_35_b200", "csrc",
                                                           "prefill_tc.cuh")],
                                             "prefill_attn_traffic.json")
                     if w.H == 128 else None},
        "e2e": {"value": whole_job_rate(T, world, t_e2e), "unit": "tokens/s",
                "ms_per_step": t_e2e, "pipelined": True,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clocks,
        "wall_s_timed": wall,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, cores, _ = _oracle_prefill_sample(w)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del pipe
    if distributed:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="batch128")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flush-l2", default="auto", choices=["auto", "on", "off"],
                    help="flush L2 before every timed call (auto: when the cache is "
                         "under twice the L2 size)")
    ap.add_argument("--batch", type=int, default=0,
                    help="use only the first N sequences of the workload")
    ap.add_argument("--heads", type=int, default=0,
                    help="use N heads instead of the workload's (small profiling case)")
    ap.add_argument("--cache", default="bf16", choices=["bf16", "fp8"],
                    help="latent cache format (fp8: the 8-bit cache, bf16 workloads only)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from mla_latent_kv_35_b200 import workloads as wl
    w = wl.workload(args.workload)
    if args.batch:
        # same shapes with fewer sequences (small profiling case)
        from dataclasses import replace
        w = replace(w, B=args.batch, ctx=w.ctx[:args.batch], name=f"{w.name}[B={args.batch}]")
    if args.heads:
        from dataclasses import replace
        w = replace(w, H=args.heads, name=f"{w.name}[H={args.heads}]")
    if w.name.startswith("prefill"):
        if args.impl == "reference":
            run_reference_prefill(args, w)
        else:
            run_gpu_prefill(args, w)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
