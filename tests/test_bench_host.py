"""Host-side pieces of bench.py that need no GPU: the conversion of an ncu launch
list into stored per-call DRAM traffic, and the source hash that guards it."""
import json
import os

import pytest

import bench

HEADER = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
          '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')


def _row(i, kernel, metric, unit, value):
    return (f'"{i}","1","python3","h","{kernel}","1","7","(256, 1, 1)","(1, 1, 1)","0","10.0",'
            f'"Command line profiler metrics","{metric}","{unit}","{value}"\n')


def test_traffic_from_launch_list(tmp_path, monkeypatch):
    lines = ["==PROF== Connected\n", HEADER]
    launches = [("at::FillFunctor", 5e8), ("cr::seg_table_kernel(Segs)", 1000), ("cr::gram_tc_kernel<256>(x)", 2e6),
                ("tk::offsets_kernel(x)", 10), ("tk::select_kernel(x)", 300),
                ("cr::seg_table_kernel(Segs)", 1000), ("cr::gram_tc_kernel<256>(x)", 2e6)]
    for i, (k, b) in enumerate(launches):
        lines.append(_row(i, k, "dram__bytes_read.sum", "byte", f"{b:.0f}"))
        lines.append(_row(i, k, "dram__bytes_write.sum", "Kbyte", "1"))
        lines.append(_row(i, k, "gpu__time_duration.sum", "ns", "5"))
    csv = tmp_path / "launches.csv"
    csv.write_text("".join(lines))
    out_dir = tmp_path / "profiles"
    out_dir.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_sha256", lambda: "abc")
    bench.write_traffic(str(csv))
    t = json.loads((out_dir / "dram_traffic_byteflow.json").read_text())
    assert t["csrc_sha256"] == "abc"
    per = t["bytes_per_call"]
    # two calls of the coding rate (seg_table starts each call): (1000 + 2e6) read + 2 KB written per call
    assert per["chunk_coding_rate"] == pytest.approx(1000 + 2e6 + 2000)
    assert per["chunk_topk_select"] == pytest.approx(310 + 2000)
    assert "chunk_gather" not in per
    assert bench.stored_traffic("chunk_coding_rate") == pytest.approx(per["chunk_coding_rate"])
    # a capture taken on other kernel sources is not used
    monkeypatch.setattr(bench, "csrc_sha256", lambda: "other")
    assert bench.stored_traffic("chunk_coding_rate") is None


def test_source_hash_covers_every_kernel_file():
    h1 = bench.csrc_sha256()
    assert len(h1) == 64 and h1 == bench.csrc_sha256()
    csrc = os.path.join(bench.ROOT, "dynamic_byte_chunking_b200", "csrc")
    assert any(f.endswith(".cu") for f in os.listdir(csrc))


def test_comment_edits_keep_the_source_hash():
    code = "int f(int x) {\n    return x + 1;   // add one\n}\n"
    same = "// a new comment\nint f(int x) {\n    /* note */ return x + 1;\n}\n"
    other = "int f(int x) {\n    return x + 2;\n}\n"
    assert bench.strip_comments(code) == bench.strip_comments(same)
    assert bench.strip_comments(code) != bench.strip_comments(other)
    # string literals keep their slashes
    assert '"a // b"' in bench.strip_comments('asm("a // b");\n')
