"""Host logic of bench.py that decides whether a committed DRAM-traffic record still
describes the kernels being timed: the record carries a hash of the projection kernels'
code (comments removed), so a comment edit keeps it and any code edit drops it."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_removes_comments_and_blank_lines():
    src = "int a = 1;  // one\n\n/* block\n   comment */ int b = 2;   \n// whole line\nreturn a + b;\n"
    assert bench.code_only(src) == "int a = 1;\n int b = 2;\nreturn a + b;"
    assert bench.code_only("x = y / z;  // ratio") == "x = y / z;"  # a lone slash is code


def _tree(tmp_path, texts):
    csrc = tmp_path / "hashed_gram_embedding_horner_b200" / "csrc"
    csrc.mkdir(parents=True, exist_ok=True)
    for name, text in texts.items():
        (csrc / name).write_text(text)
    return tmp_path


def test_traffic_record_follows_the_code_not_the_comments(tmp_path, monkeypatch):
    texts = {name: f"// {name}\nint f{i}() {{ return {i}; }}\n" for i, name in enumerate(bench.PROJECTION_SOURCES)}
    root = _tree(tmp_path, texts)
    monkeypatch.setattr(bench, "ROOT", str(root))
    (root / "profiles").mkdir()
    rec = {"kernel": "k", "workload": "w", "bytes_per_launch": 1234, "source_sha256": bench.kernel_source_hash()}
    scaled = dict(rec, workload="w2", measured_on="w2_small", scale_to_workload=2.0)
    (root / bench.TRAFFIC_RECORDS).write_text(json.dumps({"records": [rec, scaled]}))
    assert bench.profiled_traffic("k", "w") == 1234.0
    assert bench.profiled_traffic("k", "w2") == 2468.0  # a smaller case's capture, scaled by units
    assert bench.profiled_traffic("k", "other") is None
    # a comment edit keeps the record
    name = bench.PROJECTION_SOURCES[-1]
    _tree(tmp_path, {name: "/* reworded */\n" + texts[name].replace("// ", "// note: ")})
    assert bench.profiled_traffic("k", "w") == 1234.0
    # a code edit drops it
    _tree(tmp_path, {name: texts[name].replace("return", "return 1 +")})
    assert bench.profiled_traffic("k", "w") is None


def test_reference_arm_line_on_the_host():
    """`bench.py --impl reference` times the fp64 oracle on the host cores and prints the
    contract's line: the same metric, unit and workload as the GPU arm, `impl` reference,
    a cpu_baseline describing this run and an e2e object with no device copies."""
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--ref-step-seconds", "0.2"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["metric"].startswith("N-gram embed tokens/s")
    assert line["config"]["workload"] == "full_scale_bf16_D4096_N5_K2" and line["steps"] == 1
    assert line["config"]["tokens_per_step"] == 32768 and line["config"]["tables_gb"] > 59
    assert line["value"] > 0 and line["n_gpus"] == 1 and line["vs_baseline"] is None
    # each step is the timed sample: its own tokens and milliseconds, not an extrapolation
    n = line["sample_tokens_per_step"]
    assert 1 <= n <= 2048 and abs(line["value"] * line["ms_per_step"] / 1e3 - n) < 1e-6 * n
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and "sampled" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
