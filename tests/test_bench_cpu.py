"""Host-side arithmetic of bench.py (CPU only): the algorithmic bytes per unit that the
roofline divides by, the gate that reports ncu traffic only for unchanged kernel sources,
the decode-vs-recompute ratio, and the varlen leg's batch."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.argv = sys.argv[:1]
import bench  # noqa: E402

MB = 1e6


def test_prefill_and_decode_bytes_per_unit():
    # the 2.7B-shaped layer: x, y (B L H P bf16), B, C (B L G N bf16), dt (B L H bf16), h_final
    B, L, H, P, G, N = 1, 4096, 80, 64, 1, 128
    assert bench.prefill_bytes(B, L, H, P, G, N) == (
        B * L * (2 * H * P * 2 + 2 * G * N * 2 + H * 2) + B * H * P * N * 4)
    assert bench.prefill_bytes(B, L, H, P, G, N) / MB == pytest.approx(89.3, abs=0.05)
    # decode: state read + write dominates: 5.38 MB at batch 1, 85.3 MB at batch 16
    assert bench.decode_bytes(1, H, P, G, N, 4) / MB == pytest.approx(5.38, abs=0.01)
    assert bench.decode_bytes(16, H, P, G, N, 4) / MB == pytest.approx(85.3, abs=0.05)
    assert bench.decode_bytes(16, H, P, G, N, 4) > 8 * 16 * H * P * N


def test_tensor_core_kernel_bytes():
    B, L, H, P, G, N = 1, 4096, 80, 64, 1, 128
    got = {k: f(B, L, H, P, G, N) / MB for k, f in bench.KERNEL_BYTES.items()}
    assert got["chunk_state"] == pytest.approx(130.2, abs=0.1)
    assert got["state_pass"] == pytest.approx(128.5, abs=0.1)
    assert got["chunk_scan"] == pytest.approx(130.5, abs=0.1)


def test_traffic_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    # a record taken with the current sources is reported; one whose hash does not match the
    # sources (the kernel changed since the capture) is not
    names = list(bench.KERNEL_SOURCES)
    fresh = {n: {"dram_bytes": 1e6 * (i + 1), "source_sha256": bench.kernel_source_sha(n)}
             for i, n in enumerate(names)}
    fake_root = tmp_path / "repo"
    (fake_root / "profiles").mkdir(parents=True)
    (fake_root / bench.TRAFFIC_FILE).write_text(json.dumps(fresh))
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    # the sources are hashed under the real root, before ROOT pointed at the fake one
    monkeypatch.setattr(bench, "kernel_source_sha", lambda name: fresh[name]["source_sha256"])
    for i, name in enumerate(names):
        assert bench.measured_traffic(name) == 1e6 * (i + 1)
    assert bench.measured_traffic("no_such_kernel") is None
    monkeypatch.setattr(bench, "kernel_source_sha", lambda name: "1" * 64)
    for name in names:
        assert bench.measured_traffic(name) is None


def test_decode_vs_recompute_ratio():
    r = bench.decode_vs_recompute(5.0, {"b1": {"steps_per_s": 4000.0}}, [{"L": 1024}])
    assert r["cached_decode_step_ms"] == pytest.approx(0.25)
    assert r["speedup"] == pytest.approx(20.0)
    assert r["context"] == bench.PF["L"] and r["by_context"] == [{"L": 1024}]
    assert bench.decode_vs_recompute(5.0, {}) is None


def test_varlen_bench_batch():
    # the packed batch the varlen leg times (and the GPU test checks on sampled heads): 64
    # sequences of 64 .. 4096 tokens, log-uniform, seeded, the same on every call
    import ssd_synth as S
    lengths = S.varlen_lengths()
    assert lengths == S.varlen_lengths()
    assert len(lengths) == 64 and min(lengths) >= 64 and max(lengths) <= 4096
    assert sum(lengths) == 51908
    assert sum(-(-n // 128) for n in lengths) == 439  # 128-token blocks of the one-pass kernels
    # a wide spread: a few long sequences beside many short ones
    assert sum(n >= 2048 for n in lengths) < sum(n < 512 for n in lengths)
