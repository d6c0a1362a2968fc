"""bench.py's host-side pieces that need no GPU: the kernel code hash that
keys a recorded ncu traffic figure, and --record-traffic's CSV reading."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_code_hash_ignores_comments_and_layout():
    a = "int f(int x) {  // add one\n  return x + 1; /* done */\n}\n"
    b = "/* header */\nint f(int x) {\n\treturn x + 1;\n}"
    c = "int f(int x) { return x + 2; }"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_record_traffic_reads_ncu_raw_csv(tmp_path, monkeypatch):
    csv = tmp_path / "raw.csv"
    csv.write_text('"ID","Kernel Name","dram__bytes_read.sum","dram__bytes_write.sum"\n'
                   '"","","Mbyte","Kbyte"\n'
                   '"0","k","250.5","1,024"\n'
                   '"1","k","249.5","976"\n')
    store = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(store))
    entry = bench.record_traffic("probe", str(csv), ["gemv.cu"], 2, "ncu ...")
    assert entry["dram_bytes_per_launch"] == 250_000_000 + 1_000_000
    assert json.loads(store.read_text())["probe"]["code_hash"] == bench.kernel_code_hash(["gemv.cu"])
    assert bench.profile_traffic("probe") == 251_000_000
    assert bench.profile_traffic("absent") is None
