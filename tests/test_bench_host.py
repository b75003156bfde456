"""Host logic of bench.py that needs no GPU: the code-only hash that keys recorded DRAM
traffic (comments and blank lines do not change it, code does), the lookup of recorded
traffic (null for other code), and the command-line defaults."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_ignores_comments_and_blank_lines():
    a = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    b = "/* header\n   text */\nint f(int x) {\n\n  return x + 1;\n}   \n// trailing note\n"
    c = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_source_sha_is_stable_and_keys_recorded_traffic(tmp_path, monkeypatch):
    sha = bench.source_sha(bench.DECODE_SOURCES)
    assert len(sha) == 16 and sha == bench.source_sha(bench.DECODE_SOURCES)
    # a traffic file keyed by this hash is read; another hash gives no traffic
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "dram_traffic.txt").write_text(
        "# comment line\n"
        f"k_decode decode-stream {sha} 123456   # read + write\n"
        "k_decode decode-l 0000000000000000 999\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k_decode", "decode-stream", sha) == 123456.0
    assert bench.recorded_traffic("k_decode", "decode-l", sha) is None
    assert bench.recorded_traffic("k_decode", "decode-s", sha) is None


def test_default_arguments():
    a = bench.parse([])
    assert a.gpus == 1 and a.impl == "tq" and a.warmup >= 3
    assert a.decode_workload == bench.HEADLINE == "decode-stream"
