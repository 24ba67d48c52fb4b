"""Host helpers of bench.py: the code hash that keeps a recorded ncu traffic
figure tied to the kernel sources it was taken on, the clock summary that
decides whether a run was throttled, the peaks the roofline divides by, and
the whole-job aggregate."""
import json

import pytest

import bench


def test_code_tokens_ignore_comments_and_layout():
    a = "int a = 1; // one\n/* two\n   three */ float b;\n"
    b = "int a = 1;   // reworded\n\n\n float b;  /* another */"
    assert bench.code_tokens(a) == bench.code_tokens(b) == "int a = 1; float b;"


def test_code_tokens_keep_code_and_literals():
    assert bench.code_tokens("x = 1;") != bench.code_tokens("x = 2;")
    src = 'asm volatile("bar.sync 1; // kept" ::: "memory"); char c = \'"\'; // gone'
    assert bench.code_tokens(src) == 'asm volatile("bar.sync 1; // kept" ::: "memory"); char c = \'"\';'


def test_traffic_record_follows_the_code(tmp_path, monkeypatch):
    csrc = tmp_path / "pagedattention_paged_kv_decode_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    kernel = csrc / "k.cuh"
    kernel.write_text("int f() { return 1; }  // first wording\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    key = bench.kernel_source_hash(("k.cuh",))
    (tmp_path / "profiles" / "t.json").write_text(
        json.dumps({"w": {"kernel_source_hash": key, "dram_bytes_per_launch": 123}}))
    assert bench.recorded_traffic("w", "t.json", ("k.cuh",)) == 123
    kernel.write_text("/* reworded */\nint f() {\n    return 1;\n}\n")
    assert bench.recorded_traffic("w", "t.json", ("k.cuh",)) == 123
    kernel.write_text("int f() { return 2; }\n")
    assert bench.recorded_traffic("w", "t.json", ("k.cuh",)) is None
    assert bench.recorded_traffic("other", "t.json", ("k.cuh",)) is None


def test_committed_records_are_well_formed():
    # one entry per workload: a 16-hex-digit code hash, bytes per launch and
    # the summary the figure comes from (a stale hash only makes bench report
    # traffic as unknown)
    for name in ("decode_dram_traffic.json", "prefill_dram_traffic.json"):
        with open(f"{bench.ROOT}/profiles/{name}") as f:
            rec = json.load(f)
        assert rec
        for ent in rec.values():
            assert len(ent["kernel_source_hash"]) == 16 and int(ent["kernel_source_hash"], 16) >= 0
            assert isinstance(ent["dram_bytes_per_launch"], int) and ent["dram_bytes_per_launch"] > 0
            assert ent["source"].startswith("profiles/")


def _smi_row(sm, max_sm, reasons):
    # the ClockSampler field order: timestamp, index, clocks.sm, clocks.max.sm, power.draw,
    # clocks_event_reasons.active, then hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    return ["2026/01/01 00:00:00.000", "0", str(sm), str(max_sm), "700.0", "0x0"] + reasons


def test_clock_summary_reads_the_timed_window():
    off = ["Not Active"] * 4
    cs = bench.ClockSampler("0")
    cs.rows = [(0.0, _smi_row(1200, 1965, off)),
               (10.0, _smi_row(1965, 1965, off[:3] + ["Active"])),           # sw_power_cap
               (10.4, _smi_row(1900, 1965, ["Active"] + off[1:])),           # hw_slowdown
               (60.0, _smi_row(800, 1965, off[:1] + ["Active"] + off[2:]))]  # outside the window
    s = cs.summary(10.0, 10.4)
    assert s == {"sm_mhz": 1932.5, "sm_max_mhz": 1965.0, "reasons": ["hw_slowdown", "sw_power_cap"], "samples": 2,
                 "source": "nvidia-smi"}
    # no sample inside the window (a short run): every sample counts
    s = cs.summary(30.0, 30.1)
    assert s["samples"] == 4 and s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]
    assert bench.ClockSampler("0").summary(0.0, 1.0)["reasons"] == ["nvidia-smi unavailable"]


def test_clock_summary_of_nvml_samples_keeps_to_the_timed_window():
    # NVML rows come about every millisecond: only those inside the timed
    # region count (idle samples before and after it would lower the median)
    off = ["Not Active"] * 4
    cs = bench.ClockSampler("0")
    cs.source = "nvml"
    cs.rows = [(9.9, _smi_row(600, 1965, off)),                       # idle, before the region
               (10.001, _smi_row(1965, 1965, off)),
               (10.002, _smi_row(1950, 1965, off[:3] + ["Active"])),   # sw_power_cap
               (10.003, _smi_row(1965, 1965, off)),
               (10.2, _smi_row(600, 1965, ["Active"] + off[1:]))]      # after the region
    s = cs.summary(10.0, 10.0035)
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3, "source": "nvml"}
    # a region shorter than the period: the nearest sample alone
    s = cs.summary(10.0015, 10.0016)
    assert s["samples"] == 1 and s["sm_mhz"] == 1950.0     # the sample at 10.002


def test_peaks_come_from_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    assert bench.tensor_peak() == (1590.0, 1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        json.dumps({"hbm_gbs": 6000.5, "bf16_tflops": 1600, "bf16_tflops_sustained": 1300}))
    assert bench.hbm_peak() == (6000.5, "measured")
    assert bench.tensor_peak() == (1600.0, 1300.0, "measured")


def test_aggregate_is_all_ranks_bytes_over_the_slowest_time():
    assert bench.aggregate_gbs(1, 10**9, 1000.0) == pytest.approx(1.0)
    assert bench.aggregate_gbs(4, 10**9, 500.0) == pytest.approx(8.0)


@pytest.mark.parametrize("cfg", [1, 2])
def test_cpu_baseline_reports_both_legs(cfg):
    import oracle
    import workloads as W
    w = W.named(cfg)
    cb = bench.cpu_baseline_both(w, 0.2)
    assert cb["kind"] == "oracle" and cb["unit"] == "GB/s" and cb["value"] > 0
    assert cb["cores"] == oracle.max_threads() and str(cb["cores"]) in cb["sample"]
    assert cb["single_thread"]["cores"] == 1 and cb["single_thread"]["value"] > 0
    assert "single-thread" in cb["single_thread"]["sample"]


def test_cpu_baseline_step_matches_the_oracle_decode():
    """The timed oracle step computes the workload's attention: its slot and
    cache write, then the threaded attention, equal the plain oracle calls."""
    import numpy as np
    import oracle
    import workloads as W
    w = W.named(1)
    st = bench.OracleState(w)
    seqs = [2, 0, 3]
    bench._oracle_steps(w, st, seqs, threads=3)
    kc, vc = w.pool_host()
    slots = oracle.slot_mapping(w.block_tables, w.context_lens, w.block_size)
    oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots)
    # the sampled sequences' rows are written; the rest of the pools are untouched
    for s in seqs:
        b, o = divmod(int(slots[s]), w.block_size)
        assert np.array_equal(st.kc[b, o].view(np.uint16), kc[b, o].view(np.uint16))


def test_unique_bytes_count_shared_blocks_once():
    import workloads as W
    w = W.named(2)
    assert w.unique_kv_bytes() == w.kv_bytes()
    w = W.named(4)
    row = w.num_heads * w.head_size * w.elem_bytes * 2
    shared = w.shared_blocks * w.block_size
    assert w.unique_kv_bytes() == (int((w.context_lens - shared).sum()) + shared) * row
    assert w.unique_kv_bytes() < w.kv_bytes()


def test_line_puts_the_first_workload_on_top_and_the_rest_beside_it():
    import argparse
    args = argparse.Namespace(steps=20, warmup=5)

    def result(name, value, launches):
        return {"metric": bench.METRIC, "value": value, "unit": "GB/s", "ms_per_step": 0.1, "dtype": "f32",
                "config": {"workload": name}, "roofline": {"frac": 0.9}, "e2e": {"value": 1.0},
                "gpu_launches": launches, "clocks": {}, "cpu_baseline": {"cores": 16}}

    line = bench.assemble_line([result("w3", 6000.0, 40), result("w2", 1500.0, 20), result("w5", 5500.0, 40)],
                               args, 1)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
                "clocks", "cpu_baseline"):
        assert key in line, key
    assert line["config"]["workload"] == "w3" and line["value"] == 6000.0 and line["n_gpus"] == 1
    assert list(line["workloads"]) == ["w2", "w5"]
    assert line["workloads"]["w5"]["value"] == 5500.0 and "metric" not in line["workloads"]["w5"]
    assert line["gpu_launches"] == 40 and line["gpu_launches_all_workloads"] == 100
    one = bench.assemble_line([result("w3", 6000.0, 40)], args, 2)
    assert "workloads" not in one and one["n_gpus"] == 2
