"""Host-side accounting of bench.py (no GPU): the window pair count behind every SW-SKA FLOP
figure, and the source-hash gate on the recorded DRAM traffic."""
import json
import os

import pytest

import bench


def _pairs_brute(T, W):
    # a query t sees the keys j with t - W < j <= t (the window holds W keys, self included)
    return sum(1 for t in range(T) for j in range(T) if 0 <= t - j < W)


@pytest.mark.parametrize("T", [1, 2, 3, 7, 16, 33])
@pytest.mark.parametrize("W", [1, 2, 5, 16, 40])
def test_window_pairs_match_brute_force(T, W):
    assert bench.swska_pairs(T, W) == _pairs_brute(T, W)


def test_window_pairs_closed_forms():
    # W = 1 keeps only the diagonal; W >= T is full causal attention
    assert bench.swska_pairs(4096, 1) == 4096
    assert bench.swska_pairs(4096, 4096) == 4096 * 4097 // 2
    assert bench.swska_pairs(100, 10 ** 6) == 100 * 101 // 2
    # the stack layer: every query past the first W - 1 sees exactly W keys
    T, W = 131072, 4096
    assert bench.swska_pairs(T, W) == (T - W + 1) * W + (W - 1) * W // 2


def test_recorded_traffic_entries_are_consistent():
    with open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)
    for key, e in rec.items():
        if key.startswith("_"):
            continue
        assert len(e["source_hash"]) == 16 and int(e["source_hash"], 16) >= 0, key
        assert e["command"].startswith("ncu ") and "--clock-control none" in e["command"], key
        if "per_kernel" in e:
            total = sum(r + w for r, w in e["per_kernel"].values())
        else:
            total = e["read"] + e["write"]
        assert e["dram_bytes_per_launch"] == total, key


def test_recorded_traffic_is_dropped_once_the_kernel_source_changes(tmp_path, monkeypatch):
    csrc = tmp_path / "sliding_window_attention_chunked_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("// kernel v1\n")
    (csrc / "h.cuh").write_text("// header v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash("k.cu", "h.cuh")
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(
        json.dumps({"case": {"source_hash": h, "dram_bytes_per_launch": 1234}}))
    assert bench.recorded_traffic("case", ["k.cu", "h.cuh"]) == 1234
    assert bench.recorded_traffic("other", ["k.cu", "h.cuh"]) is None
    (csrc / "h.cuh").write_text("// header v2\n")  # an included header counts too
    assert bench.recorded_traffic("case", ["k.cu", "h.cuh"]) is None
