"""Host helpers of bench.py: the code hash that keeps a recorded ncu traffic
figure tied to the kernel sources it was taken on."""
import json

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
