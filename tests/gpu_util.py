"""Shared helpers of the GPU parity tests (tolerances, conversions)."""

import numpy as np
import torch

from mla_latent_kv_35_b200 import binding as B
from mla_latent_kv_35_b200 import build as _build
from mla_latent_kv_35_b200 import workloads as wl

DEV = "cuda"

# bf16 cache and weights with fp32 accumulation: max-abs 2e-2, mean-abs 2e-3;
# fp32 path: 1e-4 max-abs.  Relative L2 error is reported and bounded too
# (outputs shrink like L^-1/2 with N(0,1) data, so absolute bounds alone are
# loose at long context).
TOL = {"bf16": dict(max_abs=2e-2, mean_abs=2e-3, rel_l2=1e-2),
       "f32": dict(max_abs=1e-4, mean_abs=1e-5, rel_l2=1e-4)}


def ensure_lib():
    _build.build()
    return B.lib()


def dims(dtype="bf16", H=128, dn=128, dc=512, dr=64, dm=5120, page=64):
    return B.MLADims(H, dn, dc, dr, dn, dm, page, (dn + dr) ** -0.5, 10000.0, dtype)


def to_dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(DEV, torch.bfloat16 if dtype == "bf16" else torch.float32)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def q(x, dtype):
    """Round host values to what the device stores (bf16 RNE or fp32)."""
    x = np.asarray(x, dtype=np.float32)
    return wl.bf16_to_f32(wl.bf16_bits(x)) if dtype == "bf16" else x


def check(got, ref, dtype, what="", tol=None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    t = dict(TOL[dtype])
    if tol:
        t.update(tol)
    finite = np.isfinite(ref)
    assert (np.isfinite(got) == finite).all(), f"{what}: non-finite mismatch"
    d = np.abs(got[finite] - ref[finite])
    mx = float(d.max()) if d.size else 0.0
    mean = float(d.mean()) if d.size else 0.0
    nrm = float(np.linalg.norm(ref[finite]))
    rel = float(np.linalg.norm(d) / nrm) if nrm > 0 else 0.0
    msg = f"{what}: max_abs={mx:.3e} mean_abs={mean:.3e} rel_l2={rel:.3e}"
    print(msg)
    assert mx <= t["max_abs"], msg
    assert mean <= t["mean_abs"], msg
    assert rel <= t["rel_l2"], msg
    return mx, mean, rel


def check_stored_bf16(got, ref, what="", rotated=False, acc=None):
    """A value the GPU computes in fp32 and stores in bf16, against the
    oracle's fp64 value.

    A bf16 store rounds to nearest: |error| <= u |ref| with the unit roundoff
    u = 2^-8 of 8 significant bits.  `acc` (same shape) bounds the fp32
    accumulation that produced the value before the store, elementwise.  A
    RoPE-rotated key (rotated=True) is rounded twice: its pre-RoPE input is
    a bf16 projection output, and rotating a pair mixes the two rounded
    inputs, so element e of pair (x, y) may be off by u (|x_in| + |y_in|)
    <= u sqrt(2) |pair| (plus both inputs' accumulation bounds) before the
    final rounding of u |ref_e|."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    acc = np.zeros_like(ref) if acc is None else np.asarray(acc, np.float64)
    u = 2.0 ** -8
    bound = u * np.abs(ref)
    if rotated:
        pair = np.sqrt(ref[0::2] ** 2 + ref[1::2] ** 2)
        acc = np.repeat(np.maximum(acc[0::2], acc[1::2]) * 2, 2)
        bound = bound + u * np.sqrt(2.0) * np.repeat(pair, 2)
    bound = (bound + acc) * (1 + 1e-3) + 1e-7
    err = np.abs(got - ref)
    assert (err <= bound).all(), \
        f"{what}: worst error {err.max():.3e} (bound there {bound[np.argmax(err - bound)]:.3e})"


def fp32_accumulation_bound(x, w):
    """Bound on the fp32 accumulation error of y = x . w[o] on the tensor
    cores: each of the K/16 MMA steps adds one exactly formed partial product
    sum to an fp32 accumulator, so the error is at most (K/16) 2^-24
    sum_i |x_i w[o, i]|."""
    x = np.abs(np.asarray(x, np.float64))
    w = np.abs(np.asarray(w, np.float64))
    K = x.shape[-1]
    return (-(-K // 16)) * 2.0 ** -24 * (x @ w.T)


def status():
    return B.mla_get_device_status()
