"""bench.py's committed DRAM traffic figures (CPU, no GPU).

The roofline object quotes the DRAM bytes per forward that an ncu capture
measured, but only while the sources of the path that capture ran on are
unchanged: a kernel edit makes the figure null until it is captured again.
"""
import json
import os

import bench


def _entries():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        return json.load(f)


def test_every_entry_names_its_sources():
    csrc = os.path.join(bench.ROOT, "binary_factorized_weight_b200", "csrc")
    for key, entry in _entries().items():
        files = entry.get("source_files")
        assert files, key
        for name in files:
            assert os.path.isfile(os.path.join(csrc, name)), (key, name)
        per_kernel = sum(k["dram_read"] + k["dram_write"] for k in entry["kernels"].values())
        assert per_kernel == entry["dram_bytes_per_forward"], key


def test_bench_quotes_a_figure_only_for_current_sources():
    # every committed figure is quoted while its sources are unchanged, and never after
    for key, entry in _entries().items():
        current = entry["source_hash"] == bench.kernel_source_hash(entry["source_files"])
        assert bench.traffic_for(key) == (entry["dram_bytes_per_forward"] if current else None), key


def test_changed_sources_void_the_figure(tmp_path, monkeypatch):
    t = _entries()
    t["attn_1b_b1"]["source_hash"] = "0" * 16
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(t))
    real_csrc = os.path.join(bench.ROOT, "binary_factorized_weight_b200")
    (tmp_path / "binary_factorized_weight_b200").symlink_to(real_csrc)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("attn_1b_b1") is None
    assert bench.traffic_for("no_such_workload") is None


def test_path_hash_ignores_other_paths_sources():
    # a prefill edit must not void a decode figure and vice versa
    assert "prefill.cu" not in bench.DECODE_SOURCES
    assert "decode.cu" not in bench.PREFILL_SOURCES
    assert bench.kernel_source_hash(bench.DECODE_SOURCES) != bench.kernel_source_hash(bench.PREFILL_SOURCES)
