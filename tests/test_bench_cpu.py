"""bench.py on the host (CPU only): the reference arm's JSON line, and the
bookkeeping that decides whether a committed ncu traffic figure still applies."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_complete_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["steps"] == 1 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "llama1b_c8"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"] and cb["unit"] == d["unit"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_code_hash_ignores_comments_and_blank_lines(tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("int f(int x) {\n  return x + 1;\n}\n")
    b.write_text("// a comment\nint f(int x) {   // trailing comment\n\n  return x + 1;  \n}\n")
    c.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.code_hash(str(a)) == bench.code_hash(str(b))
    assert bench.code_hash(str(a)) != bench.code_hash(str(c))


def test_traffic_figure_only_while_the_decode_sources_match(tmp_path, monkeypatch):
    src = tmp_path / "compressed_decode_attention_fdms_b200" / "csrc"
    src.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (src / "fdms_decode.cu").write_text("int split() { return 1; }\n")
    (src / "fdms_internal.cuh").write_text("struct S { int a; };\n")
    h = [bench.code_hash(str(src / f)) for f in ("fdms_decode.cu", "fdms_internal.cuh")]
    (tmp_path / "profiles" / "decode_traffic.txt").write_text(
        "# comment line\nllama1b_c8 1234 %s %s\n" % (h[0], h[1]))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("llama1b_c8")[0] == 1234.0
    assert bench.load_traffic("qwen8b_c8_fp8") == (None, "no capture for this workload")
    (src / "fdms_decode.cu").write_text("// only a comment more\nint split() { return 1; }\n")
    assert bench.load_traffic("llama1b_c8")[0] == 1234.0
    (src / "fdms_decode.cu").write_text("int split() { return 2; }\n")
    assert bench.load_traffic("llama1b_c8") == (None,
                                                "decode kernels changed since the ncu capture")
