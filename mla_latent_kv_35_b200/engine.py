"""One MLA decode layer driven through the C ABI (device buffers + call order).

``MLADecodeLayer.step`` enqueues the whole hot path on the current stream:

  A0  mla_project       y = [W_Q; W_DKV; W_KR] h           (one GEMM)
  A2  mla_rope          q_rope -> qbuf[..., d_c:],  k_rope rotated in place
  A3  mla_cache_append  [c ; k_rope] of the new tokens -> paged pool
  A1  mla_absorb_q      q_nope . W_UK -> qbuf[..., :d_c]
  A4+A5 mla_decode      split-KV attention on the latent cache + LSE combine
  A6  mla_out_proj      W_UV per head, then W_O

Torch only provides device memory and the stream; every step runs in the
library's kernels.
"""

from __future__ import annotations

import numpy as np
import torch

from . import binding as _b
from .binding import MLADims


def _to_dev(x: np.ndarray, dtype, device):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)


class MLADecodeLayer:
    """Weights and cache of one MLA layer on one GPU."""

    def __init__(self, dims: MLADims, weights: dict, device="cuda"):
        self.dims = dims
        self.device = torch.device(device)
        dt = dims.torch_dtype
        H, dn, dr, dc = dims.n_heads, dims.d_nope, dims.d_rope, dims.d_latent
        self.dqk = dn + dr
        self.D = dc + dr
        self.Y = H * self.dqk + self.D      # row width of the A0 output
        w_a0 = np.concatenate([weights["W_Q"], weights["W_DKV"], weights["W_KR"]], 0)
        self.W_A0 = _to_dev(w_a0, dt, self.device)
        self.W_UK = _to_dev(weights["W_UK"], dt, self.device)
        self.W_UV = _to_dev(weights["W_UV"], dt, self.device)
        self.W_O = _to_dev(weights["W_O"], dt, self.device)
        self._bufs = {}
        self.pool = None
        self.cache_kind = "bf16"

    # ------------------------------------------------------------------
    # cache
    # ------------------------------------------------------------------
    def set_cache(self, pool, page_table, seq_lens, kind: str = "bf16"):
        """pool [n_pages, page_size, D] (dims dtype), page_table int32
        [B, max_pages], seq_lens int32 [B] (context after this step's append).

        kind "fp8": pool is the 8-bit latent cache, uint8 [n_pages,
        page_size, 656] (E4M3 latent, half-precision RoPE key, fp32 row
        scale; mla_cache_quantize_fp8 converts a bf16 pool): steps append by
        quantizing and attend with mla_decode_fp8."""
        if kind not in ("bf16", "fp8"):
            raise ValueError(f"cache kind {kind!r}")
        if kind == "fp8" and self.dims.dtype != "bf16":
            raise ValueError("the 8-bit cache is for bf16 layers")
        self.cache_kind = kind
        self.pool = pool
        self.page_table = page_table
        self.seq_lens = seq_lens
        self.n_pages = pool.shape[0]
        self.max_pages = page_table.shape[1]

    def prefill_from_hidden(self, h_ctx_list):
        """Fill each sequence's prior tokens from hidden states: project with
        [W_DKV; W_KR], rotate the RoPE keys at positions 0.., append."""
        d = self.dims
        H = d.n_heads
        w_ckv = self.W_A0[H * self.dqk:]
        for b, h in enumerate(h_ctx_list):
            n = h.shape[0]
            if n == 0:
                continue
            hd = _to_dev(h, d.torch_dtype, self.device)
            y = torch.empty((n, self.D), dtype=d.torch_dtype, device=self.device)
            _b.mla_project(d, hd, w_ckv, y, n, d.d_model, self.D)
            pos = torch.arange(n, dtype=torch.int32, device=self.device)
            kr = y[:, d.d_latent:]
            _b.mla_rope(d, kr, self.D, 0, 1, kr, self.D, 0, pos, n)
            bi = torch.full((n,), b, dtype=torch.int32, device=self.device)
            append = _b.mla_cache_append_fp8 if self.cache_kind == "fp8" else _b.mla_cache_append
            append(d, y, self.D, kr, self.D, bi, pos, self.page_table, self.max_pages, self.pool,
                   self.n_pages, n)

    # ------------------------------------------------------------------
    # step buffers
    # ------------------------------------------------------------------
    def buffers(self, B: int, S_q: int, num_workers: int = 0, slot: int = 0):
        """Device buffers of one step (slot: an independent second set, for
        steps that overlap in DecodePipeline)."""
        key = (B, S_q, num_workers, slot, self.cache_kind)
        if key not in self._bufs:
            d = self.dims
            T = B * S_q
            dev, dt = self.device, d.torch_dtype
            ws = (_b.mla_decode_fp8_workspace_size if self.cache_kind == "fp8"
                  else _b.mla_decode_workspace_size)(d, B, S_q, num_workers)
            sc = _b.mla_out_proj_scratch_size(d, T)
            self._bufs[key] = dict(
                y=torch.empty((T, self.Y), dtype=dt, device=dev),
                qbuf=torch.empty((T, d.n_heads, self.D), dtype=dt, device=dev),
                o_lat=torch.empty((T, d.n_heads, d.d_latent), dtype=torch.float32, device=dev),
                lse=torch.empty((T, d.n_heads), dtype=torch.float32, device=dev),
                out=torch.empty((T, d.d_model), dtype=torch.float32, device=dev),
                ws=torch.empty((max(ws, 256),), dtype=torch.uint8, device=dev),
                scratch=torch.empty((max(sc, 256),), dtype=torch.uint8, device=dev),
            )
        return self._bufs[key]

    # ------------------------------------------------------------------
    # the hot path
    # ------------------------------------------------------------------
    def step(self, h, batch_idx, pos, B: int, S_q: int, num_workers: int = 0,
             fused: bool = True, slot: int = 0):
        """h [T, d_model] device (dims dtype), batch_idx/pos int32 [T] device,
        T = B*S_q tokens b-major.  Returns the dict of step buffers.

        fused: A1-A3 through mla_pre_attention (one launch for bf16) instead
        of the four separate calls; both write the same bits.  An 8-bit
        cache always takes the separate calls, its append quantizing the new
        rows (mla_cache_append_fp8)."""
        d = self.dims
        H, dn, dc, dr = d.n_heads, d.d_nope, d.d_latent, d.d_rope
        T = B * S_q
        bf = self.buffers(B, S_q, num_workers, slot)
        y, qbuf = bf["y"], bf["qbuf"]
        Y, D, dqk = self.Y, self.D, self.dqk
        _b.mla_project(d, h, self.W_A0, y, T, d.d_model, Y)                        # A0
        fp8 = self.cache_kind == "fp8"
        if fused and not fp8:
            _b.mla_pre_attention(d, y, Y, self.W_UK, qbuf, batch_idx, pos,          # A1-A3
                                 self.page_table, self.max_pages, self.pool, self.n_pages, T)
        else:
            off_c = H * dqk
            _b.mla_rope(d, y[:, dn:], Y, dqk, H, qbuf[:, :, dc:], H * D, D, pos, T)  # A2 q
            kr = y[:, off_c + dc:]
            _b.mla_rope(d, kr, Y, 0, 1, kr, Y, 0, pos, T)                             # A2 k
            append = _b.mla_cache_append_fp8 if fp8 else _b.mla_cache_append
            append(d, y[:, off_c:], Y, kr, Y, batch_idx, pos,                         # A3
                   self.page_table, self.max_pages, self.pool, self.n_pages, T)
            _b.mla_absorb_q(d, y, Y, self.W_UK, qbuf, T)                               # A1
        decode = _b.mla_decode_fp8 if fp8 else _b.mla_decode
        decode(d, qbuf, self.pool, self.n_pages, self.page_table,                     # A4+A5
               self.max_pages, self.seq_lens, B, S_q, num_workers, bf["ws"],
               bf["o_lat"], bf["lse"])
        _b.mla_out_proj(d, bf["o_lat"], self.W_UV, self.W_O, bf["scratch"],         # A6
                        bf["out"], T)
        return bf

    # ------------------------------------------------------------------
    # chunked prefill (non-absorbed)
    # ------------------------------------------------------------------
    def prefill_buffers(self, T: int, L: int, slot: int = 0):
        """Device buffers of one prefill chunk of T tokens ending at context L
        (slot: an independent second set, for chunks that overlap in
        PrefillPipeline)."""
        key = ("prefill", T, L, slot)
        if key not in self._bufs:
            d = self.dims
            dev, dt = self.device, d.torch_dtype
            H = d.n_heads
            self._bufs[key] = dict(
                y=torch.empty((T, self.Y), dtype=dt, device=dev),
                ctx=torch.empty((L, self.D), dtype=dt, device=dev),
                k_nope=torch.empty((L, H, d.d_nope), dtype=dt, device=dev),
                v=torch.empty((L, H, d.d_v), dtype=dt, device=dev),
                o=torch.empty((T, H, d.d_v), dtype=dt, device=dev),
                lse=torch.empty((T, H), dtype=torch.float32, device=dev),
                out=torch.empty((T, d.d_model), dtype=dt, device=dev),
            )
        return self._bufs[key]

    def prefill_chunk(self, h, pos, batch_idx, b: int, T: int, L: int, slot: int = 0):
        """Prefill T new tokens of sequence b, at positions L - T .. L - 1.

        h [T, d_model] device; pos int32 [T] = L - T .. L - 1 and batch_idx
        int32 [T] = b, both on the device.  The chunk takes the non-absorbed
        form: the new tokens' latents and RoPE keys go into the cache, then
        every head's keys and values of all L tokens are rebuilt once
        (W_UK c, W_UV c) and the T queries attend causally over them.

          P0  mla_project            y = [W_Q; W_DKV; W_KR] h
          P0  mla_rope (x2)          q_rope and k_rope rotated in place in y
          P0  mla_cache_append       [c ; k_rope] -> paged pool
          P1  mla_prefill_rebuild_kv ctx rows, k_nope, v of the L tokens
          P2  mla_prefill_attention  o [T, H, d_v], lse [T, H]
          P3  mla_project            out = W_O o  (bf16 [T, d_model])

        Returns the dict of chunk buffers.  bf16 layers with a bf16 cache."""
        d = self.dims
        if d.dtype != "bf16" or self.cache_kind != "bf16":
            raise ValueError("chunked prefill needs a bf16 layer and a bf16 cache")
        if not 0 < T <= L:
            raise ValueError("need 0 < T <= L")
        H, dn, dc = d.n_heads, d.d_nope, d.d_latent
        Y, dqk = self.Y, self.dqk
        off_c = H * dqk
        bf = self.prefill_buffers(T, L, slot)
        y = bf["y"]
        _b.mla_project(d, h, self.W_A0, y, T, d.d_model, Y)
        _b.mla_rope(d, y[:, dn:], Y, dqk, H, y[:, dn:], Y, dqk, pos, T)
        kr = y[:, off_c + dc:]
        _b.mla_rope(d, kr, Y, 0, 1, kr, Y, 0, pos, T)
        _b.mla_cache_append(d, y[:, off_c:], Y, kr, Y, batch_idx, pos, self.page_table,
                            self.max_pages, self.pool, self.n_pages, T)
        _b.mla_prefill_rebuild_kv(d, self.pool, self.n_pages, self.page_table[b], L, self.W_UK,
                                  self.W_UV, bf["ctx"], bf["k_nope"], bf["v"])
        _b.mla_prefill_attention(d, y, Y, bf["ctx"], bf["k_nope"], bf["v"], T, L, bf["o"],
                                 bf["lse"])
        _b.mla_project(d, bf["o"], self.W_O, bf["out"], T, H * d.d_v, d.d_model)
        return bf

    def capture(self, h, batch_idx, pos, B: int, S_q: int, num_workers: int = 0,
                fused: bool = True, slot: int = 0):
        """Capture one step on these input buffers into a CUDA graph.

        Returns (graph, buffers, kernels): graph.replay() reruns the whole
        step (projection through output projection) on whatever h,
        batch_idx and pos hold at that time, writing the same buffers;
        kernels is the number of kernel launches the graph contains.  The
        step's buffers are allocated before capture, so the graph holds no
        memory of its own.
        """
        bf = self.buffers(B, S_q, num_workers, slot)
        torch.cuda.synchronize(self.device)
        graph = torch.cuda.CUDAGraph()
        l0 = _b.mla_launch_count()
        with torch.cuda.graph(graph):
            self.step(h, batch_idx, pos, B, S_q, num_workers, fused, slot)
        kernels = _b.mla_launch_count() - l0
        return graph, bf, kernels



class DecodePipeline:
    """A decode loop that overlaps each step's host transfers with compute.

    Two slots, each with its own input buffers, step buffers and CUDA graph
    of the whole step.  submit() enqueues step i in slot i % 2: the inputs
    are copied from pinned host memory on an upload stream while the
    previous step computes, the graph replays on the current stream once its
    inputs are in (and the slot's previous output has left), and the output
    is copied back on a download stream while the next step computes.  Every
    step still moves its own inputs in and its own output out.
    """

    def __init__(self, layer: MLADecodeLayer, B: int, S_q: int, num_workers: int = 0,
                 fused: bool = True):
        d = layer.dims
        dev = layer.device
        T = B * S_q
        self.layer = layer
        self.up = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        self.slots = []
        for s in range(2):
            h = torch.zeros((T, d.d_model), dtype=d.torch_dtype, device=dev)
            bi = torch.zeros((T,), dtype=torch.int32, device=dev)
            pos = torch.zeros((T,), dtype=torch.int32, device=dev)
            graph, bf, kernels = layer.capture(h, bi, pos, B, S_q, num_workers, fused, slot=s)
            self.slots.append(dict(h=h, bi=bi, pos=pos, graph=graph, out=bf["out"],
                                   inputs_in=torch.cuda.Event(), done=torch.cuda.Event(),
                                   out_read=torch.cuda.Event()))
        self.kernels_per_step = kernels
        self.i = 0

    def submit(self, h_host, bi_host, pos_host, out_host):
        """Enqueue one step: h_host [T, d_model], bi_host/pos_host int32 [T]
        and out_host fp32 [T, d_model] are pinned host tensors; out_host
        holds the step's output once the step's `out_read` event has
        completed (after wait(), at the latest)."""
        sl = self.slots[self.i % 2]
        self.i += 1
        compute = torch.cuda.current_stream(self.layer.device)
        # the slot's inputs are free once its previous step has run
        self.up.wait_event(sl["done"])
        with torch.cuda.stream(self.up):
            sl["h"].copy_(h_host, non_blocking=True)
            sl["bi"].copy_(bi_host, non_blocking=True)
            sl["pos"].copy_(pos_host, non_blocking=True)
            sl["inputs_in"].record(self.up)
        compute.wait_event(sl["inputs_in"])
        compute.wait_event(sl["out_read"])
        sl["graph"].replay()
        sl["done"].record(compute)
        self.down.wait_event(sl["done"])
        with torch.cuda.stream(self.down):
            out_host.copy_(sl["out"], non_blocking=True)
            sl["out_read"].record(self.down)
        return sl["out_read"]

    def drain(self, stream=None):
        """Make `stream` (default: the current one) wait for every submitted
        step's output transfer."""
        stream = stream or torch.cuda.current_stream(self.layer.device)
        for sl in self.slots:
            stream.wait_event(sl["out_read"])

    def wait(self):
        """Block the host until every submitted step's output is on the host."""
        for sl in self.slots:
            sl["out_read"].synchronize()


class PrefillPipeline:
    """Chunked prefill that overlaps each chunk's host transfers with compute.

    Two slots, each with its own input buffers and chunk buffers.  submit()
    enqueues chunk i in slot i % 2: h, positions and batch indices are copied
    from pinned host memory on an upload stream while the previous chunk
    computes; the chunk runs on the current stream once its inputs are in
    (and the slot's previous output has left); its `out` goes back on a
    download stream while the next chunk computes.  Chunks of one sequence
    still run in order on the compute stream, so each sees the cache rows the
    previous one appended.
    """

    def __init__(self, layer: MLADecodeLayer, b: int, T: int, L: int):
        d = layer.dims
        dev = layer.device
        self.layer, self.b, self.T, self.L = layer, b, T, L
        self.up = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        self.slots = []
        for s in range(2):
            layer.prefill_buffers(T, L, slot=s)
            self.slots.append(dict(
                h=torch.empty((T, d.d_model), dtype=d.torch_dtype, device=dev),
                bi=torch.empty((T,), dtype=torch.int32, device=dev),
                pos=torch.empty((T,), dtype=torch.int32, device=dev),
                inputs_in=torch.cuda.Event(), done=torch.cuda.Event(),
                out_read=torch.cuda.Event()))
        self.i = 0

    def submit(self, h_host, bi_host, pos_host, out_host):
        """Enqueue one chunk: h_host [T, d_model] (layer dtype), bi_host and
        pos_host int32 [T] and out_host [T, d_model] (layer dtype) are pinned
        host tensors; out_host holds the chunk's output once its `out_read`
        event (returned) has completed."""
        s = self.i % 2
        sl = self.slots[s]
        self.i += 1
        compute = torch.cuda.current_stream(self.layer.device)
        self.up.wait_event(sl["done"])
        with torch.cuda.stream(self.up):
            sl["h"].copy_(h_host, non_blocking=True)
            sl["bi"].copy_(bi_host, non_blocking=True)
            sl["pos"].copy_(pos_host, non_blocking=True)
            sl["inputs_in"].record(self.up)
        compute.wait_event(sl["inputs_in"])
        compute.wait_event(sl["out_read"])
        bf = self.layer.prefill_chunk(sl["h"], sl["pos"], sl["bi"], self.b, self.T, self.L,
                                      slot=s)
        sl["done"].record(compute)
        self.down.wait_event(sl["done"])
        with torch.cuda.stream(self.down):
            out_host.copy_(bf["out"], non_blocking=True)
            sl["out_read"].record(self.down)
        return sl["out_read"]

    def drain(self, stream=None):
        """Make `stream` (default: the current one) wait for every submitted
        chunk's output transfer."""
        stream = stream or torch.cuda.current_stream(self.layer.device)
        for sl in self.slots:
            stream.wait_event(sl["out_read"])

    def wait(self):
        for sl in self.slots:
            sl["out_read"].synchronize()


def build_pool_host(w, page_table, n_pages, prior_bits, canary=0xFFFF):
    """Host image of the paged pool for workload ``w``: prior rows of each
    sequence scattered into its pages, every other slot set to ``canary``.

    prior_bits: list of [Lp_b, D] uint16 (bf16) or float32 arrays.
    """
    D = w.D
    if w.dtype == "bf16":
        pool = np.full((n_pages, w.page_size, D), canary, dtype=np.uint16)
    else:
        pool = np.full((n_pages, w.page_size, D), np.nan, dtype=np.float32)
    for b, rows in enumerate(prior_bits):
        Lp = rows.shape[0]
        npg = -(-Lp // w.page_size)
        if npg == 0:
            continue
        full = Lp // w.page_size
        pages = page_table[b, :npg]
        if full:
            pool[pages[:full]] = rows[:full * w.page_size].reshape(full, w.page_size, D)
        rem = Lp - full * w.page_size
        if rem:
            pool[pages[full], :rem] = rows[full * w.page_size:]
    return pool


def build_pool_host_drawn(w, page_table, n_pages, canary=0xFFFF, threads=8):
    """Like build_pool_host, drawing each sequence's prior rows from the
    seeded generator inside worker threads (no full copy of the priors)."""
    from concurrent.futures import ThreadPoolExecutor

    from . import workloads as wl
    D = w.D
    if w.dtype == "bf16":
        pool = np.full((n_pages, w.page_size, D), canary, dtype=np.uint16)
    else:
        pool = np.full((n_pages, w.page_size, D), np.nan, dtype=np.float32)

    def fill(b):
        if w.dtype == "bf16":
            rows = wl.draw_prior_bits(w, b)
        else:
            rows = np.concatenate(wl.draw_prior(w, b), 1)
        Lp = rows.shape[0]
        full = Lp // w.page_size
        npg = -(-Lp // w.page_size)
        pages = page_table[b, :npg]
        if full:
            pool[pages[:full]] = rows[:full * w.page_size].reshape(full, w.page_size, D)
        rem = Lp - full * w.page_size
        if rem:
            pool[pages[full], :rem] = rows[full * w.page_size:]

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(fill, range(w.B)))
    return pool


def pool_to_device(pool_host: np.ndarray, dtype: str, device="cuda"):
    if dtype == "bf16":
        return torch.from_numpy(pool_host.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(pool_host).to(device)
