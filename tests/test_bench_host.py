"""Host-side pieces of bench.py that need no GPU: the kernel-code digest that
decides whether the recorded ncu traffic still applies, the clock-sample
summary, the whole-job rate, and the prefill line's FLOP count and config."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_digest_ignores_comments_only(tmp_path):
    a = tmp_path / "a.cuh"
    b = tmp_path / "b.cuh"
    c = tmp_path / "c.cuh"
    a.write_text("// header\nint f(int x) {  // inline\n  return x + 1;\n}\n")
    b.write_text("/* another\n   header */\n\nint f(int x) {\n  return x + 1;  // changed note\n}\n")
    c.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.code_digest([str(a)]) == bench.code_digest([str(b)])
    assert bench.code_digest([str(a)]) != bench.code_digest([str(c)])


def test_recorded_traffic_applies_only_to_the_captured_source(tmp_path, monkeypatch):
    """The ncu DRAM bytes recorded under profiles/ are reported only while the
    kernel source (comments aside) is the one the capture ran."""
    import json
    src = tmp_path / "k.cuh"
    src.write_text("int f() { return 1; }  // kernel\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"dram_bytes_per_call": 123.0, "code_sha256": bench.code_digest([str(src)])}
    (prof / "decode_tc_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic_for([str(src)]) == 123.0
    src.write_text("int f() { return 1; }  // comment edited\n")
    assert bench._traffic_for([str(src)]) == 123.0
    src.write_text("int f() { return 2; }\n")
    assert bench._traffic_for([str(src)]) is None


def test_clock_summary_uses_samples_after_mark():
    s = bench.ClockSampler(0)
    s.lines = [(0.5, "0, 1000, 1965, 100.0, 0x0, Not Active, Not Active, Not Active, Not Active"),
               (2.0, "0, 1900, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active"),
               (2.1, "0, 1700, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active"),
               (2.2, "0, 1800, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active")]
    s.t_mark = 1.0
    out = s.summary()
    assert out == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3}
    s.t_mark = 5.0
    assert s.summary()["samples"] == 0


def test_whole_job_rate():
    assert bench.whole_job_rate(128, 1, 1.6) == pytest.approx(80000.0)
    assert bench.whole_job_rate(128, 8, 1.6) == pytest.approx(640000.0)


def test_prefill_flops_against_a_counted_chunk():
    """The prefill line's algorithmic FLOPs: each stage counted directly on a
    small chunk (every query's visible keys enumerated, every multiply-add
    counted as 2)."""
    from dataclasses import replace
    from mla_latent_kv_35_b200 import workloads as wl
    w = replace(wl.workload("prefill"), H=3, S_q=5, ctx=(12,), d_model=40)
    T, L, H = 5, 12, 3
    dqk, dv, dc, D = 128 + 64, 128, 512, 576
    pairs = 0
    for j in range(T):
        for t in range(L):
            if t <= L - T + j:
                pairs += 1
    assert pairs == sum(range(L - T + 1, L + 1))
    f = bench.prefill_flops(w)
    assert f["attention"] == 2 * pairs * H * (dqk + dv)
    assert f["rebuild"] == 2 * L * H * (128 + dv) * dc
    assert f["a0"] == 2 * T * w.d_model * (H * dqk + D)
    assert f["w_o"] == 2 * T * H * dv * w.d_model


def test_prefill_config_names_the_chunk():
    from mla_latent_kv_35_b200 import workloads as wl
    c = bench.prefill_config(wl.workload("prefill"), 1)
    assert c["workload"] == "prefill"
    assert (c["chunk_tokens"], c["cached_before"], c["context_after"]) == (4096, 4096, 8192)
    assert c["heads"] == 128 and c["parallelism"] == "single GPU"
