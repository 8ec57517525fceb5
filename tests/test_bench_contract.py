"""bench.py's output contract, on the CPU: the reference arm's JSON line (the
oracle timed on the host cores, on the tiny workload), and the rule that ties
the roofline's DRAM traffic to the kernel sources it was measured on."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config"}


def test_reference_arm_json_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert KEYS <= set(d), KEYS - set(d)
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"].startswith("tiny") and "model" not in d["config"]
    # tokens/s = sequences per step / step time
    assert d["value"] > 0
    assert abs(d["value"] - d["config"]["batch"] / (d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_source_sha_ignores_comments_only(tmp_path, monkeypatch):
    """The traffic ratios stay valid across comment edits and lapse on any code edit."""
    csrc = tmp_path / "tree_indexed_sparse_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("// one\nint f() { return 1; }  /* two */\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    a = bench.source_sha()
    (csrc / "k.cu").write_text("// changed comment\nint f() {   return 1; }\n")
    assert bench.source_sha() == a
    (csrc / "k.cu").write_text("int f() { return 2; }\n")
    assert bench.source_sha() != a


def test_traffic_needs_matching_sources(tmp_path, monkeypatch):
    """A kernel's traffic ratio holds while its own translation unit and the
    headers are unchanged: another unit's edit leaves it, its own or a
    header's voids it."""
    csrc = tmp_path / "tree_indexed_sparse_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "zha_route.cu").write_text("int f() { return 1; }\n")
    (csrc / "zha_attn.cu").write_text("int g() { return 1; }\n")
    (csrc / "zha_common.cuh").write_text("int h();\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    entry = {"dram_bytes_per_alg_byte": 1.25, "dram_bytes": 1.25e9, "alg_bytes": 1e9,
             "source_sha": bench.source_sha("zha_route.cu")}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"kernels": {"score[l1]": entry}}))
    assert bench.traffic_for("score[l1]", 2e9) == pytest.approx(2.5e9)
    assert bench.traffic_for("attn_sparse", 2e9) is None
    (csrc / "zha_attn.cu").write_text("int g() { return 2; }\n")
    assert bench.traffic_for("score[l1]", 2e9) == pytest.approx(2.5e9)
    (csrc / "zha_common.cuh").write_text("int h(int);\n")
    assert bench.traffic_for("score[l1]", 2e9) is None
    (csrc / "zha_common.cuh").write_text("int h();\n")
    (csrc / "zha_route.cu").write_text("int f() { return 3; }\n")
    assert bench.traffic_for("score[l1]", 2e9) is None