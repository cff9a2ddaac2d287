"""bench.py's bookkeeping without a GPU: the algorithmic byte counts per kernel
(each input read once, each output written once) and the rule that committed
DRAM counters are reported only while the kernel's own sources are unchanged."""
import json
import os

import bench


def test_algorithmic_bytes_full_path():
    T, H, L, J, D, G = 65536, 7168, 2, 8, 64, 148
    ab = bench.algorithmic_bytes(T, H, L, J, D, G)
    # hash+gather: token read, 16 indices written, 16 rows of 128 B read and written
    assert ab["hash_gather"] == T * (8 + 16 * 8 + 2 * 16 * 128) == 277348352
    # gate forward: x, k, v read, out written (2H bytes each), gate written, wh, we read
    assert ab["gate_fwd"] == T * (8 * H + 4) + 4 * H
    # fused gate backward: g, x, k, v read, dx, dk, dv written, partial rows
    # written, wh, we read; then the reduction: partial rows read, dwh, dwe
    # written, wh, we read
    assert ab["gate_bwd"] == (T * 14 * H + G * 4 * H + 4 * H) + (G * 4 * H + 8 * H + 4 * H)
    assert set(ab) == {"hash_gather", "gate_fwd", "gate_bwd"}


def test_kernel_entry_fractions():
    e = bench.kernel_entry(100.0, 560_000_000, 7000.0)        # 5.6 TB/s
    assert e["GB/s"] == 5600.0
    assert e["frac"] == 0.8 and e["frac_nominal"] == 0.7
    assert e["us_at_bar"] == 100.0                            # exactly at 70% of 8 TB/s


def test_gather_bwd_bytes():
    # full path: 1,048,576 entries (8 B index + 128 B gradient row each) and
    # 821,830 distinct table rows (256 B fp32, read and written)
    assert bench.gather_bwd_bytes(65536, 2, 8, 64, 821830) == 1048576 * 136 + 821830 * 512 \
        == 563383296
    # no entries, nothing to move; one row read by every entry is read and written once
    assert bench.gather_bwd_bytes(0, 2, 8, 64, 0) == 0
    assert bench.gather_bwd_bytes(10, 1, 1, 8, 1) == 10 * 24 + 64


def test_every_kernel_has_sources_and_a_digest():
    for k in ("hash_gather", "gate_fwd", "gate_bwd", "gather_bwd"):
        d = bench.source_digest(k)
        assert len(d) == 16 and int(d, 16) >= 0
    # the gate kernels share their sources, the gather backward has its own
    assert bench.source_digest("gate_fwd") == bench.source_digest("gate_bwd")
    assert bench.source_digest("gather_bwd") != bench.source_digest("gate_bwd")


def test_committed_traffic_needs_matching_digest(tmp_path, monkeypatch):
    entry = {"source_digest": bench.source_digest("gate_bwd"), "units": 1000,
             "dram_bytes": 14_000_000}
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps({"gate_bwd": entry}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(p))
    assert bench.committed_traffic("gate_bwd", 2000) == 28_000_000   # scaled by units
    entry["source_digest"] = "0" * 16
    p.write_text(json.dumps({"gate_bwd": entry}))
    assert bench.committed_traffic("gate_bwd", 2000) is None
    assert bench.committed_traffic("hash_gather", 2000) is None       # no entry


def test_committed_traffic_file_is_current():
    # the profiles/traffic.json in the repository was taken on the current
    # sources of every kernel it lists
    with open(bench.TRAFFIC_FILE) as f:
        d = json.load(f)
    for k, e in d.items():
        if k.startswith("_"):
            continue
        assert e["source_digest"] == bench.source_digest(k), f"{k}: counters are stale"
        assert e["dram_bytes"] == e["dram_read"] + e["dram_write"]


def test_measured_peak_falls_back_without_the_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peak, kind = bench.measured_peak()
    assert kind == "fallback" and peak == bench.FALLBACK_HBM_GBS
    assert os.path.basename(bench.TRAFFIC_FILE) == "traffic.json"
