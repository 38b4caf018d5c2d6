"""Host-side logic of the benchmark (no GPU): the roofline arithmetic, the
algorithmic byte counts it divides by, the attended-pair count of the local
MQA and the guard that ties a recorded DRAM traffic figure to the kernel
sources it was measured on."""
import json

import numpy as np

import bench
from lm_causal_depthwise_b200 import workloads as W


def test_roofline_fraction_is_bytes_over_time_over_peak():
    r = bench.roofline(2_000_000_000, 0.5, {"hbm_gbs": 8000.0}, "measured", 123, ["k"])
    assert r["achieved"] == 4000.0          # 2e9 B / 0.5 ms = 4e12 B/s
    assert r["frac"] == 0.5
    assert r["traffic"] == 123 and r["bound"] == "hbm" and r["unit"] == "GB/s"


def test_prefill_bytes_follow_the_per_token_count():
    """6 D + 4 bytes per token in bf16 (x, g in; y out; int32 segment_pos),
    plus both states read and written and the parameters read once."""
    for name, total in (("prefill-2b", 506_560_512), ("prefill-long", 2_016_544_768),
                        ("prefill-9b", 3_227_385_856)):
        w = W.ALL[name]
        per_token = 6 * w.D + 4
        states = 2 * (w.B * w.D * 4 + 3 * w.B * w.D * 2)
        params = 2 * w.D * 256 * 2 + 8 * w.D * 4
        assert W.algorithmic_bytes(w) == w.B * w.T * per_token + states + params == total


def test_throughput_helpers():
    assert bench.job_throughput(1000, 4, 2.0) == 4000 / 2e-3
    assert bench.sharded_throughput(1000, 2.0) == 1000 / 2e-3


def test_mqa_valid_pairs_equals_brute_force():
    rng = np.random.default_rng(7)
    B, T, window = 3, 70, 16
    segpos = np.zeros((B, T), np.int32)
    for b in range(B):
        p = int(rng.integers(0, 40))                  # a document begun before the call
        for t in range(T):
            if rng.random() < 0.08:
                p = 0
            segpos[b, t] = p
            p += 1
    want = 0
    for b in range(B):
        for t in range(T):
            want += sum(1 for s in range(T) if t - window < s <= t and s >= t - segpos[b, t])
    assert bench.mqa_valid_pairs(segpos, window) == want


def test_traffic_record_is_used_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic_demo.json").write_text(json.dumps({"source_digest": "abc", "dram_bytes_per_launch": 42}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_digest", lambda: "abc")
    assert bench.recorded_traffic("demo") == 42
    monkeypatch.setattr(bench, "source_digest", lambda: "changed")
    assert bench.recorded_traffic("demo") is None
    assert bench.recorded_traffic("missing") is None
