"""bench.py's host-side logic on CPU: roofline arithmetic against the burst peak, the gating of recorded
DRAM traffic by the kernel sources' hash, and the parsing of sampled clocks."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6550.0, "bf16_tflops": 1673.1, "bf16_tflops_sustained": 1383.4, "source": "measured"}


def test_tensor_roofline_uses_the_burst_peak():
    r = bench.tensor_roofline(5.0e12, 5.0, PEAKS)  # 5 TFLOP in 5 ms = 1000 TFLOP/s
    assert abs(r["achieved"] - 1000.0) < 1e-9
    assert r["peak"] == 1673.1 and abs(r["frac"] - 1000.0 / 1673.1) < 1e-12
    assert abs(r["frac_of_sustained_peak"] - 1000.0 / 1383.4) < 1e-12
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["traffic"] is None


def test_hbm_roofline():
    r = bench.hbm_roofline(6.55e9, 1.0, PEAKS)  # 6.55 GB in 1 ms
    assert abs(r["achieved"] - 6550.0) < 1e-6 and abs(r["frac"] - 1.0) < 1e-12 and r["unit"] == "GB/s"


def test_recorded_traffic_is_gated_by_the_source_hash(tmp_path, monkeypatch):
    rec = tmp_path / "t.json"
    sha = bench.sources_sha256(["merge.cu"])
    rec.write_text(json.dumps({"entries": {
        "ok": {"bytes_per_launch": 123, "sources": ["merge.cu"], "sources_sha256": sha, "how": "test"},
        "stale": {"bytes_per_launch": 456, "sources": ["merge.cu"], "sources_sha256": "0" * 64}}}))
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(rec))
    assert bench.recorded_traffic("ok") == (123, "test")
    val, why = bench.recorded_traffic("stale")
    assert val is None and "changed" in why
    val, why = bench.recorded_traffic("missing")
    assert val is None
    r = bench.hbm_roofline(1e9, 1.0, PEAKS, "ok")
    assert r["traffic"] == 123


def test_committed_traffic_record_is_well_formed():
    with open(bench.TRAFFIC_RECORD) as f:
        d = json.load(f)
    for key, e in d["entries"].items():
        assert int(e["bytes_per_launch"]) > 0, key
        assert len(e["sources_sha256"]) == 64 and e["sources"], key
        assert "ncu" in e["command"] and "--clock-control none" in e["command"], key


def test_clock_rows_parse():
    out = "\n".join(["1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
                     "1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
                     "1700, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
                     "garbage"])
    c = bench.parse_clock_rows(out)
    assert c["sm_mhz"] == 1800 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
    assert c["samples"] == 3
    assert bench.parse_clock_rows("") is None
