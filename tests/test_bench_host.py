"""Host-side logic of bench.py (no GPU): the compulsory-byte accounting and
the guard that reports ncu traffic only for the kernel sources it was taken
on."""
import bench
import synth


def test_compulsory_bytes_match_the_stated_formula():
    # read every key, read the kept values, write kept keys and values,
    # 12 bytes of index / position per kept row
    c2 = synth.SPECS["c2"]
    per_unit = 32768 * 128 * 2 + 2048 * 128 * 2 + 2 * 2048 * 128 * 2 + 12 * 2048
    assert bench.compulsory_bytes(c2) == 4 * per_unit == 39944192
    c1 = synth.SPECS["c1"]
    assert bench.compulsory_bytes(c1) == 4096 * 512 + 512 * 512 * 3 + 12 * 512
    c4 = synth.SPECS["c4"]
    assert bench.score_bytes(c4) == 1024 * 131072 * 256


def test_source_hash_ignores_comments_only():
    a = "int f(int x) {  // doubles\n  return 2 * x; /* twice */ }\n"
    b = "int f(int x) {\n    return 2 * x; }  // other words\n"
    c = "int f(int x) { return 3 * x; }"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_traffic_reported_only_for_the_captured_sources(monkeypatch):
    key = ("c2", "prune_coop_kernel")
    rec = bench.TRAFFIC[key]
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda *k: rec["src"])
    assert bench.measured_traffic(*key, False) == rec["bytes_per_launch"]
    assert bench.measured_traffic(*key, True) is None          # a cut workload
    assert bench.measured_traffic("c2", "other_kernel", False) is None
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda *k: "0" * 16)
    assert bench.measured_traffic(*key, False) is None          # sources changed


def test_kernel_hash_covers_its_own_sources_only(tmp_path, monkeypatch):
    csrc = tmp_path / "rope_aware_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "coop.cu").write_text('#include "common.cuh"\nint coop;\n')
    (csrc / "fused.cu").write_text('#include "common.cuh"\nint fused;\n')
    (csrc / "common.cuh").write_text("int shared;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    coop0, fused0 = (bench.kernel_sources_hash("prune_coop_kernel"),
                     bench.kernel_sources_hash("prune_fused_kernel"))
    (csrc / "fused.cu").write_text('#include "common.cuh"\nint fused2;\n')
    assert bench.kernel_sources_hash("prune_coop_kernel") == coop0
    assert bench.kernel_sources_hash("prune_fused_kernel") != fused0
    (csrc / "common.cuh").write_text("int shared2;\n")
    assert bench.kernel_sources_hash("prune_coop_kernel") != coop0
