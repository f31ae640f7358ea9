"""Host-side checks of the seeded input generator (no GPU)."""

import numpy as np
import torch

from mla_latent_kv_35_b200 import workloads as wl


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0,
                                  65504.0, 1e-30], dtype=np.float32)])
    ours = wl.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy()
    np.testing.assert_array_equal(ours.view(np.int16), ref)
    np.testing.assert_array_equal(wl.bf16_bits(wl.bf16_to_f32(ours)), ours)


def test_named_workloads():
    w = wl.workload("tiny")
    assert (w.B, w.H, w.d_latent, w.d_rope, w.ctx, w.dtype) == \
        (2, 8, 64, 16, (37, 64), "f32")
    assert abs(w.scale - 48 ** -0.5) < 1e-15
    w = wl.workload("batch128")
    assert w.D == 576 and w.ctx[0] == 32768 and w.pages_per_seq[0] == 512
    assert abs(w.scale - 192 ** -0.5) < 1e-15
    w = wl.workload("ragged")
    prior = w.prior
    assert all(128 <= L <= 65536 for L in prior) and len(prior) == 64
    assert wl.workload("ragged").ctx == w.ctx            # seed 7 is fixed
    assert wl.workload("long4").S_q == 2


def test_page_layout_is_a_valid_partition():
    for name in ("tiny", "dsv2", "ragged", "batch128"):
        w = wl.workload(name)
        table, n_pages = wl.page_layout(w)
        used = []
        for b, nb in enumerate(w.pages_per_seq):
            assert (table[b, :nb] >= 0).all() and (table[b, nb:] == -1).all()
            used.extend(table[b, :nb].tolist())
        assert len(set(used)) == len(used) == n_pages - 1
        assert max(used) == n_pages - 2                  # last page is slack
    t1, _ = wl.page_layout(wl.workload("batch128"))
    t2, _ = wl.page_layout(wl.workload("batch128"))
    np.testing.assert_array_equal(t1, t2)
    assert not (t1[0, :8] == np.arange(8)).all()         # permuted


def test_prior_draws_are_per_sequence_streams():
    w = wl.workload("ragged")
    c3, k3 = wl.draw_prior(w, 3)
    assert c3.shape == (w.prior[3], 512) and k3.shape == (w.prior[3], 64)
    c3b, _ = wl.draw_prior_all(w, [2, 3])[1]
    np.testing.assert_array_equal(c3, c3b)
    np.testing.assert_array_equal(wl.bf16_to_f32(wl.bf16_bits(c3)), c3)


def test_positions():
    w = wl.workload("long4")
    bi, pos = wl.positions(w)
    assert bi.tolist() == [0, 0, 1, 1, 2, 2, 3, 3]
    assert pos.tolist() == [131070, 131071] * 4


def test_prefill_shards_are_distinct_sequences_of_the_same_chunk():
    """Weak scaling of the prefill line: rank r of N prefills global sequence r
    (its own prior cache and chunk), with the chunk's shapes unchanged and
    rank 0's shard equal to the unsharded workload."""
    w = wl.workload("prefill", H=4, S_q=8, ctx=(24,), d_model=32)
    s0, s1 = wl.shard(w, 0, 2), wl.shard(w, 1, 2)
    for s in (s0, s1):
        assert (s.B, s.S_q, s.ctx, s.H) == (1, 8, (24,), 4)
    assert np.array_equal(wl.draw_h_new(s0), wl.draw_h_new(w))
    assert not np.array_equal(wl.draw_h_new(s0), wl.draw_h_new(s1))
    c0, _ = wl.draw_prior(s0, 0)
    c1, _ = wl.draw_prior(s1, 0)
    assert c0.shape == c1.shape == (16, w.d_latent)
    assert not np.array_equal(c0, c1)
    bi, pos = wl.positions(s1)
    assert bi.tolist() == [0] * 8 and pos.tolist() == list(range(16, 24))
