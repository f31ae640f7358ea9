"""The pooled oracle reference used by the full-size GPU parity tests equals
the oracle's own decode_step (CPU only: it is test infrastructure too)."""

import numpy as np

import oracle
import oracle_pool
from mla_latent_kv_35_b200 import workloads as wl


def test_pooled_reference_equals_decode_step():
    w = wl.workload("long1", B=2, ctx=(70, 129), H=8, d_model=96)
    W = wl.draw_weights(w)
    h = wl.draw_h_new(w)
    ref = oracle_pool.workload_reference(w, W, h, [0, 1], head_chunk=3)
    for b in range(2):
        c, kr = wl.draw_prior(w, b)
        full = oracle.decode_step(h[b:b + 1], [c], [kr], W["W_Q"], W["W_DKV"], W["W_KR"],
                                  W["W_UK"], W["W_UV"], W["W_O"], w.scale, w.rope_base, w.H,
                                  prior_kr_rotated=True)
        for key in ("o_lat", "lse", "out", "c_new", "kr_new"):
            np.testing.assert_allclose(ref[b][key], full[key][0], rtol=0, atol=1e-10,
                                       err_msg=key)
