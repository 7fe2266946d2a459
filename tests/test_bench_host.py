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
    (root / "profiles" / "k_w.md").write_text("# k\n\ntraffic_record: " + json.dumps(rec) + "\n")
    assert bench.profiled_traffic("k", "w") == 1234.0
    assert bench.profiled_traffic("k", "other") is None
    # a comment edit keeps the record
    name = bench.PROJECTION_SOURCES[-1]
    _tree(tmp_path, {name: "/* reworded */\n" + texts[name].replace("// ", "// note: ")})
    assert bench.profiled_traffic("k", "w") == 1234.0
    # a code edit drops it
    _tree(tmp_path, {name: texts[name].replace("return", "return 1 +")})
    assert bench.profiled_traffic("k", "w") is None
