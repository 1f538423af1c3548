"""bench.py's roofline bookkeeping on the CPU: the score kernel's bound, peak
and flop count, the update kernel's bytes, and the traffic lookup gated by the
kernel sources' hash."""
import json
import os

import pytest

import bench

PEAKS = {"hbm_gbs": 6529.4, "bf16_tflops": 1674.6, "bf16_tflops_sustained": 1388.6, "sm_max_mhz": 1965.0}


def test_score_roofline_hbm_below_ridge():
    # 64 flop per byte is under the burst ridge (1674.6 TFLOP/s / 6529.4 GB/s = 256.5)
    r = bench.score_roofline(64e12, 1e12, 1000.0, PEAKS, True)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(1000.0) and r["peak"] == PEAKS["hbm_gbs"]
    assert r["flop_per_byte"] == pytest.approx(64.0)
    assert r["tensor_frac"] == pytest.approx(64.0 / 1674.6)


def test_score_roofline_tensor_above_ridge_uses_the_burst_peak():
    r = bench.score_roofline(500e12, 1e12, 1000.0, PEAKS, True)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["peak"] == 1674.6 and r["peak_kind"] == "burst"
    assert r["achieved"] == pytest.approx(500.0)
    assert r["hbm_frac"] == pytest.approx(1000.0 / 6529.4)


def test_score_roofline_ridge():
    assert bench.score_roofline(257e12, 1e12, 1.0, PEAKS, True)["bound"] == "tensor"
    assert bench.score_roofline(256e12, 1e12, 1.0, PEAKS, True)["bound"] == "hbm"


def test_score_roofline_counts_the_recompute_apart():
    # the method's work is one product per (beacon, key) pair; pass 2's recompute is reported, not counted
    r = bench.score_roofline(300e12, 1e12, 1000.0, PEAKS, True, recompute_flops=290e12)
    assert r["achieved"] == pytest.approx(300.0)
    assert r["executed_tflops"] == pytest.approx(590.0)
    assert r["algorithmic_flops_per_launch"] == 300e12 and r["recompute_flops_per_launch"] == 290e12


def test_score_roofline_simt():
    r = bench.score_roofline(74.4e12, 1e12, 1000.0, PEAKS, False)
    assert r["bound"] == "alu" and r["kernel"] == "beacon_score_simt"
    assert r["peak"] == pytest.approx(148 * 128 * 2 * 1965e6 / 1e12)


def test_update_roofline_bytes():
    import types
    w = types.SimpleNamespace(dtype="bf16", num_beacons=64, head_dim=128, query_window=64, G=4, segments=36864)
    r = bench.update_roofline(w, 2.0, PEAKS, True)
    per_seg = 64 * 4 * 128 * 2 + 64 * 128 * 10 + 64 * 12
    assert r["algorithmic_bytes_per_launch"] == 36864 * per_seg
    assert r["achieved"] == pytest.approx(36864 * per_seg / 2e-3 / 1e9)
    assert r["bound"] == "hbm" and r["kernel"] == "beacon_update_tc"


def test_traffic_lookup_gated_by_source_hash(tmp_path, monkeypatch):
    src = ["select_compact.cu", "philox.cuh"]
    good = {"sources": src, "source_hash": bench.kernel_source_hash(src), "unit": "moved row",
            "dram_bytes_per_unit": 1000.0}
    stale = dict(good, source_hash="0" * 16)
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps({"select_compact": {"a": good, "b": stale}}))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(path))
    assert bench.profiled_traffic("select_compact", "a", 3.0) == pytest.approx(3000.0)
    assert bench.profiled_traffic("select_compact", "b", 3.0) is None
    assert bench.profiled_traffic("select_compact", "missing", 3.0) is None
    assert bench.profiled_traffic("decode_attention", "a", 3.0) is None


def test_committed_traffic_entries_are_well_formed():
    with open(bench.PROFILE_TRAFFIC) as f:
        t = json.load(f)
    csrc = os.path.join(bench.ROOT, "decode_kv_cache_paged_b200", "csrc")
    n = 0
    for kernel, entries in t.items():
        if kernel == "about":
            continue
        for workload, e in entries.items():
            assert e["dram_bytes_per_unit"] > 0 and e["unit"] and e["captured"], (kernel, workload)
            assert all(os.path.exists(os.path.join(csrc, s)) for s in e["sources"]), (kernel, workload)
            assert len(e["source_hash"]) == 16
            n += 1
    assert n >= 4


def test_workload_overrides():
    """--requests/--layers/--beacons reach the workload; a random selector drops the beacon state."""
    import types
    args = types.SimpleNamespace(workload="long_trace", requests=2, layers=4, beacons=128, selector=None)
    w, sel = bench.make_workload(args)
    assert (w.num_requests, w.num_layers, w.num_beacons, sel) == (2, 4, 128, "beacon")
    assert len(w.length) == 2 and int(w.length[0]) == 32768
    args = types.SimpleNamespace(workload="beacon_serving", requests=None, layers=None, beacons=None,
                                 selector="random")
    w, sel = bench.make_workload(args)
    assert sel == "random" and w.num_beacons == 0 and w.query_window == 0


def test_pool_jobs_carry_the_beacon_override(monkeypatch):
    """The all-cores oracle rebuilds the workload in each worker from the job tuple: the beacon override
    must travel with it."""
    import types
    seen = []

    def fake_rate(w, sel, budget_s, rank_seed=0, seg_offset=0):
        seen.append(w.num_beacons)
        return 1.0, "", 1
    monkeypatch.setattr(bench, "oracle_sample_rate", fake_rate)
    bench._pool_worker(("long_trace", 1, 1, 64, "beacon", 0.01, 0))
    assert seen == [64]
