"""bench.py's measurement arithmetic on the host (no GPU)."""
import json

import numpy as np
import pytest

import bench


def test_draft_bytes_at_qwen3():
    # base read + z write (2 B K V 4) + Bf once (r V 2) + gathered A rows + per-position outputs
    B, K, V, r = 64, 8, 151936, 256
    got = bench.draft_bytes(B, K, V, r, 2)
    assert got == 2 * B * K * V * 4 + r * V * 2 + B * K * r * 2 + B * K * (4 + 4 + 8 + 4)
    assert got / 1e6 == pytest.approx(700.4, abs=0.05)


def test_verify_bytes_counts_rows_and_rejected_z_rows():
    V, K = 1000, 4
    L = np.array([4, 0, 2])
    acc = np.array([4, 0, 1])  # request 2 rejected its second draft; 0 and 1 accepted all
    assert bench.verify_bytes(V, K, L, acc) == (5 + 1 + 3) * V * 4 + 1 * V * 4
    # every length K and nothing rejected: the upper bound of the table, 389 MB less the z rows
    assert bench.verify_bytes(151936, 8, np.full(64, 8), np.full(64, 8)) / 1e6 == pytest.approx(350.1, abs=0.05)


def test_variant_b_bytes():
    # variant B: no z write (the operand rows instead); base + Bf is 389.0 MB at qwen3
    B, K, V, r = 64, 8, 151936, 256
    got = bench.draft_bytes(B, K, V, r, 2, "b")
    assert got == B * K * V * 4 + B * K * r * 2 + r * V * 2 + B * K * r * 2 + B * K * (4 + 4 + 8 + 4)
    assert (got - B * K * r * 4 - B * K * 20) / 1e6 == pytest.approx(389.0, abs=0.05)
    # verify B reads each rejected request's base row instead of its z row, plus Bf once and the operand rows
    V, K = 1000, 4
    L = np.array([4, 0, 2])
    acc = np.array([4, 0, 1])
    assert bench.verify_bytes(V, K, L, acc, 64, 2, "b") == (5 + 1 + 3) * V * 4 + V * 4 + 64 * V * 2 + 64 * 2
    # nothing rejected: no recompute
    assert bench.verify_bytes(V, K, L, L, 64, 2, "b") == (5 + 1 + 3) * V * 4


def test_round_variant_choice():
    assert bench.round_variant("auto", 64) == "a"
    assert bench.round_variant("auto", 256) == "b"
    assert bench.round_variant("a", 512) == "a" and bench.round_variant("b", 1) == "b"


def test_traffic_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    rec = {"workload": "qwen3", "source_sha256": "0" * 64, "dram_bytes_per_launch": {"draft_tc_kernel": 1}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "source_digest", lambda: "0" * 64)
    assert bench.measured_traffic("qwen3") == {"draft_tc_kernel": 1}
    assert bench.measured_traffic("latency") == {}
    monkeypatch.setattr(bench, "source_digest", lambda: "1" * 64)
    assert bench.measured_traffic("qwen3") == {}


def test_source_digest_covers_the_kernels():
    d1 = bench.source_digest()
    assert len(d1) == 64 and d1 == bench.source_digest()
