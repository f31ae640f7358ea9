"""ctypes binding of libmla_b200.so: argument marshalling only.

Every function takes torch tensors (device memory owned by the caller), turns
them into raw pointers plus sizes and calls the C entry point of the same
name on the current CUDA stream.  Nothing is computed here; if the library is
missing, loading fails loudly (there is no fallback).
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")

MLA_F32, MLA_BF16 = 0, 1
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED",
          3: "MLA_ERR_CUDA", 4: "MLA_ERR_TIMEOUT", 5: "MLA_ERR_BOUNDS"}

# Every symbol include/mla.h declares.
EXPORTS = ("mla_project", "mla_absorb_q", "mla_rope", "mla_cache_append",
           "mla_decode_workspace_size", "mla_decode", "mla_out_proj_scratch_size",
           "mla_out_proj", "mla_get_device_status", "mla_status_string",
           "mla_launch_count", "mla_selftest_wait_timeout", "mla_get_wait_diag",
           "mla_decode_noalloc", "mla_pre_attention", "mla_decode_partial",
           "mla_combine_parts", "mla_decode_config", "mla_decode_noalloc_scratch_bytes",
           "mla_cache_append_fp8", "mla_cache_quantize_fp8", "mla_decode_fp8",
           "mla_decode_fp8_workspace_size", "mla_prefill_rebuild_kv", "mla_prefill_attention")


class MLAError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")


class Dims(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int), ("d_nope", ctypes.c_int),
                ("d_latent", ctypes.c_int), ("d_rope", ctypes.c_int),
                ("d_v", ctypes.c_int), ("d_model", ctypes.c_int),
                ("page_size", ctypes.c_int), ("scale", ctypes.c_float),
                ("rope_base", ctypes.c_float), ("dtype", ctypes.c_int)]


@dataclass(frozen=True)
class MLADims:
    n_heads: int
    d_nope: int
    d_latent: int
    d_rope: int
    d_v: int
    d_model: int
    page_size: int
    scale: float
    rope_base: float
    dtype: str  # "f32" | "bf16"

    def c(self) -> Dims:
        return Dims(self.n_heads, self.d_nope, self.d_latent, self.d_rope,
                    self.d_v, self.d_model, self.page_size, self.scale,
                    self.rope_base, MLA_BF16 if self.dtype == "bf16" else MLA_F32)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @staticmethod
    def of(w) -> "MLADims":
        """Dims of a workloads.Workload."""
        return MLADims(w.H, w.d_nope, w.d_latent, w.d_rope, w.d_v, w.d_model,
                       w.page_size, w.scale, w.rope_base, w.dtype)


_lib = None

_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "mla_project": ([ctypes.POINTER(Dims), _P, _P, _P, _I, _I, _I, _P], _I),
    "mla_absorb_q": ([ctypes.POINTER(Dims), _P, _I, _P, _P, _I, _P], _I),
    "mla_rope": ([ctypes.POINTER(Dims), _P, _I, _I, _I, _P, _I, _I, _P, _I, _P], _I),
    "mla_cache_append": ([ctypes.POINTER(Dims), _P, _I, _P, _I, _P, _P, _P, _I, _P,
                          _I, _I, _P], _I),
    "mla_decode_workspace_size": ([ctypes.POINTER(Dims), _I, _I, _I], _Z),
    "mla_decode": ([ctypes.POINTER(Dims), _P, _P, _I, _P, _I, _P, _I, _I, _I, _P, _Z,
                    _P, _P, _P], _I),
    "mla_out_proj_scratch_size": ([ctypes.POINTER(Dims), _I], _Z),
    "mla_out_proj": ([ctypes.POINTER(Dims), _P, _P, _P, _P, _Z, _P, _I, _P], _I),
    "mla_get_device_status": ([_P], _I),
    "mla_status_string": ([_I], ctypes.c_char_p),
    "mla_launch_count": ([], ctypes.c_uint64),
    "mla_selftest_wait_timeout": ([ctypes.c_ulonglong, _P], _I),
    "mla_get_wait_diag": ([ctypes.POINTER(ctypes.c_uint32)], _I),
    "mla_decode_noalloc": ([ctypes.POINTER(Dims), _P, _P, _I, _P, _I, _P, _I, _I, _I, _P, _P,
                            _P], _I),
    "mla_pre_attention": ([ctypes.POINTER(Dims), _P, _I, _P, _P, _P, _P, _P, _I, _P, _I, _I,
                           _P], _I),
    "mla_decode_partial": ([ctypes.POINTER(Dims), _P, _P, _I, _P, _I, _P, _P, _I, _I, _I, _P,
                            _Z, _P, _P, _P], _I),
    "mla_combine_parts": ([ctypes.POINTER(Dims), _P, _P, _I, _I, _P, _P, _P], _I),
    "mla_decode_config": ([ctypes.POINTER(Dims), _I, _I, ctypes.POINTER(_I),
                           ctypes.POINTER(_I), ctypes.POINTER(_I)], _I),
    "mla_decode_noalloc_scratch_bytes": ([], _Z),
    "mla_cache_append_fp8": ([ctypes.POINTER(Dims), _P, _I, _P, _I, _P, _P, _P, _I, _P,
                              _I, _I, _P], _I),
    "mla_cache_quantize_fp8": ([ctypes.POINTER(Dims), _P, _P, _I, _P], _I),
    "mla_decode_fp8_workspace_size": ([ctypes.POINTER(Dims), _I, _I, _I], _Z),
    "mla_decode_fp8": ([ctypes.POINTER(Dims), _P, _P, _I, _P, _I, _P, _I, _I, _I, _P, _Z,
                        _P, _P, _P], _I),
    "mla_prefill_rebuild_kv": ([ctypes.POINTER(Dims), _P, _I, _P, _I, _P, _P, _P, _P, _P, _P],
                               _I),
    "mla_prefill_attention": ([ctypes.POINTER(Dims), _P, _I, _P, _P, _P, _I, _I, _P, _P, _P], _I),
}

FP8_ROW_BYTES = 656

DECODE_KERNEL_SIMT, DECODE_KERNEL_TC = 0, 1


def lib():
    """Load (once) and return the ctypes handle of libmla_b200.so."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mla_latent_kv_35_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(h, name)
            f.argtypes = args
            f.restype = res
        _lib = h
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(name, code):
    if code != 0:
        raise MLAError(name, code)


def _dev(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must live on the CUDA device")


# --------------------------------------------------------------------------
# one wrapper per entry point
# --------------------------------------------------------------------------

def mla_project(dims: MLADims, x, w, y, rows: int, in_f: int, out_f: int):
    _dev(x, w, y)
    _check("mla_project", lib().mla_project(ctypes.byref(dims.c()), _ptr(x), _ptr(w),
                                            _ptr(y), rows, in_f, out_f, _stream()))


def mla_absorb_q(dims: MLADims, q, q_stride_tok: int, w_uk, qbuf, T: int):
    _dev(q, w_uk, qbuf)
    _check("mla_absorb_q", lib().mla_absorb_q(ctypes.byref(dims.c()), _ptr(q), q_stride_tok,
                                              _ptr(w_uk), _ptr(qbuf), T, _stream()))


def mla_rope(dims: MLADims, x, xs_tok, xs_head, n_heads_x, y, ys_tok, ys_head, pos, T):
    _dev(x, y, pos)
    _check("mla_rope", lib().mla_rope(ctypes.byref(dims.c()), _ptr(x), xs_tok, xs_head,
                                      n_heads_x, _ptr(y), ys_tok, ys_head, _ptr(pos), T,
                                      _stream()))


def mla_cache_append(dims: MLADims, c, cs_tok, kr, ks_tok, batch_idx, pos, page_table,
                     max_pages, pool, n_pages, T):
    _dev(c, kr, batch_idx, pos, page_table, pool)
    _check("mla_cache_append", lib().mla_cache_append(
        ctypes.byref(dims.c()), _ptr(c), cs_tok, _ptr(kr), ks_tok, _ptr(batch_idx), _ptr(pos),
        _ptr(page_table), max_pages, _ptr(pool), n_pages, T, _stream()))


def mla_cache_append_fp8(dims: MLADims, c, cs_tok, kr, ks_tok, batch_idx, pos, page_table,
                         max_pages, pool8, n_pages, T):
    _dev(c, kr, batch_idx, pos, page_table, pool8)
    _check("mla_cache_append_fp8", lib().mla_cache_append_fp8(
        ctypes.byref(dims.c()), _ptr(c), cs_tok, _ptr(kr), ks_tok, _ptr(batch_idx), _ptr(pos),
        _ptr(page_table), max_pages, _ptr(pool8), n_pages, T, _stream()))


def mla_cache_quantize_fp8(dims: MLADims, pool, pool8, n_pages):
    _dev(pool, pool8)
    _check("mla_cache_quantize_fp8", lib().mla_cache_quantize_fp8(
        ctypes.byref(dims.c()), _ptr(pool), _ptr(pool8), n_pages, _stream()))


def mla_decode_fp8_workspace_size(dims: MLADims, B: int, S_q: int, num_workers: int = 0) -> int:
    return int(lib().mla_decode_fp8_workspace_size(ctypes.byref(dims.c()), B, S_q, num_workers))


def mla_decode_fp8(dims: MLADims, qbuf, pool8, n_pages, page_table, max_pages, seq_lens, B, S_q,
                   num_workers, workspace, o_lat, lse):
    _dev(qbuf, pool8, page_table, seq_lens, workspace, o_lat, lse)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("mla_decode_fp8", lib().mla_decode_fp8(
        ctypes.byref(dims.c()), _ptr(qbuf), _ptr(pool8), n_pages, _ptr(page_table), max_pages,
        _ptr(seq_lens), B, S_q, num_workers, _ptr(workspace), ws_bytes, _ptr(o_lat), _ptr(lse),
        _stream()))


def mla_pre_attention(dims: MLADims, y, y_stride_tok, w_uk, qbuf, batch_idx, pos, page_table,
                      max_pages, pool, n_pages, T):
    _dev(y, w_uk, qbuf, batch_idx, pos, page_table, pool)
    _check("mla_pre_attention", lib().mla_pre_attention(
        ctypes.byref(dims.c()), _ptr(y), y_stride_tok, _ptr(w_uk), _ptr(qbuf), _ptr(batch_idx),
        _ptr(pos), _ptr(page_table), max_pages, _ptr(pool), n_pages, T, _stream()))


def mla_decode_partial(dims: MLADims, qbuf, pool, n_pages, page_table, max_pages, seq_lens,
                       seq_tail, B, S_q, num_workers, workspace, o_lat, lse):
    _dev(qbuf, pool, page_table, seq_lens, seq_tail, workspace, o_lat, lse)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("mla_decode_partial", lib().mla_decode_partial(
        ctypes.byref(dims.c()), _ptr(qbuf), _ptr(pool), n_pages, _ptr(page_table), max_pages,
        _ptr(seq_lens), _ptr(seq_tail), B, S_q, num_workers, _ptr(workspace), ws_bytes,
        _ptr(o_lat), _ptr(lse), _stream()))


def mla_combine_parts(dims: MLADims, o_parts, lse_parts, n_parts, rows, o_lat, lse):
    _dev(o_parts, lse_parts, o_lat, lse)
    _check("mla_combine_parts", lib().mla_combine_parts(
        ctypes.byref(dims.c()), _ptr(o_parts), _ptr(lse_parts), n_parts, rows, _ptr(o_lat),
        _ptr(lse), _stream()))


def mla_decode_workspace_size(dims: MLADims, B: int, S_q: int, num_workers: int = 0) -> int:
    return int(lib().mla_decode_workspace_size(ctypes.byref(dims.c()), B, S_q, num_workers))


def mla_decode(dims: MLADims, qbuf, pool, n_pages, page_table, max_pages, seq_lens, B, S_q,
               num_workers, workspace, o_lat, lse):
    _dev(qbuf, pool, page_table, seq_lens, workspace, o_lat, lse)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("mla_decode", lib().mla_decode(
        ctypes.byref(dims.c()), _ptr(qbuf), _ptr(pool), n_pages, _ptr(page_table), max_pages,
        _ptr(seq_lens), B, S_q, num_workers, _ptr(workspace), ws_bytes, _ptr(o_lat), _ptr(lse),
        _stream()))


def mla_decode_config(dims: MLADims, S_q: int, num_workers: int = 0):
    """(kernel, block_tokens, workers) mla_decode uses for these dims."""
    k, bt, g = _I(), _I(), _I()
    _check("mla_decode_config", lib().mla_decode_config(
        ctypes.byref(dims.c()), S_q, num_workers, ctypes.byref(k), ctypes.byref(bt),
        ctypes.byref(g)))
    return k.value, bt.value, g.value


def mla_decode_noalloc_scratch_bytes() -> int:
    """Size of the library's built-in decode scratch array."""
    return int(lib().mla_decode_noalloc_scratch_bytes())


def mla_decode_noalloc(dims: MLADims, qbuf, pool, n_pages, page_table, max_pages, seq_lens,
                       B, S_q, num_workers, o_lat, lse):
    """mla_decode with the library's built-in scratch instead of a workspace
    (for callers that cannot allocate device memory; calls share the scratch
    and must not overlap on the GPU)."""
    _dev(qbuf, pool, page_table, seq_lens, o_lat, lse)
    _check("mla_decode_noalloc", lib().mla_decode_noalloc(
        ctypes.byref(dims.c()), _ptr(qbuf), _ptr(pool), n_pages, _ptr(page_table), max_pages,
        _ptr(seq_lens), B, S_q, num_workers, _ptr(o_lat), _ptr(lse), _stream()))


def mla_prefill_rebuild_kv(dims: MLADims, pool, n_pages, page_row, L, w_uk, w_uv, ctx,
                           k_nope, v):
    _dev(pool, page_row, w_uk, w_uv, ctx, k_nope, v)
    _check("mla_prefill_rebuild_kv", lib().mla_prefill_rebuild_kv(
        ctypes.byref(dims.c()), _ptr(pool), n_pages, _ptr(page_row), L, _ptr(w_uk), _ptr(w_uv),
        _ptr(ctx), _ptr(k_nope), _ptr(v), _stream()))


def mla_prefill_attention(dims: MLADims, q, q_stride_tok, ctx, k_nope, v, T, L, o, lse):
    _dev(q, ctx, k_nope, v, o, lse)
    _check("mla_prefill_attention", lib().mla_prefill_attention(
        ctypes.byref(dims.c()), _ptr(q), q_stride_tok, _ptr(ctx), _ptr(k_nope), _ptr(v), T, L,
        _ptr(o), _ptr(lse), _stream()))


def mla_out_proj_scratch_size(dims: MLADims, T: int) -> int:
    return int(lib().mla_out_proj_scratch_size(ctypes.byref(dims.c()), T))


def mla_out_proj(dims: MLADims, o_lat, w_uv, w_o, scratch, out, T: int):
    _dev(o_lat, w_uv, w_o, scratch, out)
    sb = scratch.numel() * scratch.element_size()
    _check("mla_out_proj", lib().mla_out_proj(ctypes.byref(dims.c()), _ptr(o_lat), _ptr(w_uv),
                                              _ptr(w_o), _ptr(scratch), sb, _ptr(out), T,
                                              _stream()))


def mla_get_device_status() -> int:
    """Synchronise the current stream; return and clear the device status."""
    return int(lib().mla_get_device_status(_stream()))


def mla_get_wait_diag():
    """(site, info, parity, cta) of the first bounded wait that gave up."""
    out = (ctypes.c_uint32 * 4)()
    _check("mla_get_wait_diag", lib().mla_get_wait_diag(out))
    return tuple(int(x) for x in out)


def mla_status_string(code: int) -> str:
    return lib().mla_status_string(code).decode()


def mla_launch_count() -> int:
    return int(lib().mla_launch_count())


def mla_selftest_wait_timeout(wait_ns: int):
    _check("mla_selftest_wait_timeout", lib().mla_selftest_wait_timeout(wait_ns, _stream()))
