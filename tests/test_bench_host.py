"""CPU: host-side choices of bench.py (the bf16 denominator follows the
sampled clocks)."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

PEAKS = (6546.9, 1676.5, 1374.1, "measured")


def test_burst_peak_at_full_clock():
    r = bench.roofline_tensor(1000.0, {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, PEAKS)
    assert r["peak"] == 1676.5 and r["frac"] == round(1000 / 1676.5, 4)
    assert r["frac_of_sustained_peak"] == round(1000 / 1374.1, 4)


def test_sustained_peak_only_when_power_capped_and_slow():
    slow = {"sm_mhz": 1330, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.roofline_tensor(1000.0, slow, PEAKS)["peak"] == 1374.1
    # Power cap flagged but the clock stayed near its maximum: burst.
    fast = {"sm_mhz": 1900, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.roofline_tensor(1000.0, fast, PEAKS)["peak"] == 1676.5
    # Slow clock without the power cap (e.g. a clock lock): still burst.
    locked = {"sm_mhz": 1100, "sm_max_mhz": 1965, "reasons": []}
    assert bench.roofline_tensor(1000.0, locked, PEAKS)["peak"] == 1676.5
    # No clock record at all: burst.
    assert bench.roofline_tensor(1000.0, {"sm_mhz": None, "sm_max_mhz": None, "reasons": []},
                                 PEAKS)["peak"] == 1676.5


def test_nominal_fractions_reported_beside_measured():
    r = bench.roofline_tensor(1125.0, {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, PEAKS)
    assert r["frac_of_nominal"] == 0.5
    h = bench.roofline_hbm(6000.0, 6546.9, "measured", kernel="k", traffic=None)
    assert h["bound"] == "hbm" and h["frac"] == round(6000 / 6546.9, 4)
    assert h["frac_of_nominal"] == 0.75 and h["kernel"] == "k" and h["traffic"] is None


def test_both_arms_print_the_same_config():
    """The reference arm's `config` is the GPU arm's dict for the same
    workload (the driver compares them)."""
    from block_sparse_attention_layerrouter_b200.inputs import WORKLOADS
    wl = WORKLOADS[bench.DEFAULT_WORKLOAD]
    cfg = bench.prefill_config(wl, 1)
    assert cfg["workload"] == "qwen3-8b-layer-s262144" and cfg["S"] == 262144
    assert set(cfg) >= {"workload", "router", "step", "parallelism", "l2"}
    assert bench.prefill_config(wl, 1) == cfg            # deterministic from the workload alone
    assert "replicas" in bench.prefill_config(wl, 2)["parallelism"]


def test_traffic_record_needs_the_same_device_code_and_workload(tmp_path, monkeypatch):
    rec = tmp_path / "traffic.txt"
    sha = bench.prefill_device_sha()
    rec.write_text("# comment: ignored\nworkload: qwen3-8b-layer-s262144 (B=1)\n"
                   "device_code_sha256_16: %s\ndram_bytes_per_full_launch: 12345\n" % sha)
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.kernel_traffic("qwen3-8b-layer-s262144")[0] == 12345.0
    assert bench.kernel_traffic("qwen3-4b-layer-s8192")[0] is None          # other workload
    rec.write_text("workload: qwen3-8b-layer-s262144\ndevice_code_sha256_16: 0000\n"
                   "dram_bytes_per_full_launch: 12345\n")
    assert bench.kernel_traffic("qwen3-8b-layer-s262144")[0] is None        # other code


def test_committed_traffic_record_matches_the_current_device_code():
    """profiles/ holds the DRAM record of the bench's FULL launch taken on
    the device code that is in the tree (else roofline.traffic is null)."""
    b, wl, why = bench.kernel_traffic(bench.DEFAULT_WORKLOAD)
    assert b is not None and b > 0, why
