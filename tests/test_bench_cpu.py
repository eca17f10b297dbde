"""CPU checks of bench.py's bookkeeping (no GPU): the recorded ncu counters are keyed by the code of a
kernel family, so a comment edit keeps them and a code edit drops them."""
import importlib.util
import os
import shutil

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_counters_survive_comment_edits_but_not_code_edits(tmp_path, monkeypatch):
    bench = load_bench()
    csrc = tmp_path / "nvfp4_grouped_gemm_indices_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "nvfp4_grouped_gemm_indices_b200", "csrc"), csrc)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = {f: bench.kernel_source_hash(f) for f in bench.KERNEL_SOURCES}
    assert before == {f: load_bench().kernel_source_hash(f) for f in bench.KERNEL_SOURCES}
    q = csrc / "bsg_quant.cuh"
    q.write_text(q.read_text() + "\n// a note\n\n")                      # comment and blank lines only
    assert bench.kernel_source_hash("quant") == before["quant"]
    q.write_text(q.read_text() + "constexpr int kUnused = 1;\n")          # code
    assert bench.kernel_source_hash("quant") != before["quant"]
    # the families are independent: the other hashes did not move
    for f in ("fp8", "nvfp4", "moe"):
        assert bench.kernel_source_hash(f) == before[f]


def test_every_recorded_workload_belongs_to_a_known_family():
    bench = load_bench()
    import json
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        d = json.load(fh)
    for name, entry in d.items():
        if name.startswith("_"):
            continue
        assert bench.kernel_family(name) in bench.KERNEL_SOURCES, name
        assert entry["bytes_per_launch"] > 0 and entry["kernel"].startswith("bsg_")
