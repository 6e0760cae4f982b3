"""Host-side logic of bench.py that needs no GPU: the traffic summary written
from an ncu CSV and the staleness rule that reads it back."""

from __future__ import annotations

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

HEADER = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
          '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')


def _row(i, kernel, metric, unit, value):
    return (f'"{i}","1","python3","127.0.0.1","{kernel}","1","7","(512, 1, 1)","(148, 1, 1)","0",'
            f'"10.0","Command line profiler metrics","{metric}","{unit}","{value}"\n')


def test_traffic_summary_from_ncu_csv(tmp_path):
    launches = 2
    lines = ["==PROF== Connected to process 1\n", HEADER]
    i = 0
    expect = []
    for name, K, N, _ in bench.DECODE_SHAPES:
        for j in range(launches):
            rd = bench.alg_bytes("int4", 1, N, K) + 1000 * (j + 1)
            wr = 64 * (j + 1)
            k = "void w4::gemv_kernel<0, 1, 4, 0>(w4::Params)"
            lines.append(_row(i, k, "dram__bytes_read.sum", "byte", f"{rd:,}"))
            lines.append(_row(i, k, "dram__bytes_write.sum", "Kbyte", f"{wr / 1000:.3f}"))
            lines.append(_row(i, k, "gpu__time_duration.sum", "usecond", "12.5"))
            i += 1
        expect.append(rd + wr)           # the last launch of each shape counts
    csv_path = tmp_path / "t.csv"
    csv_path.write_text("".join(lines))
    out = tmp_path / "traffic.json"
    bench.write_traffic(str(csv_path), launches, out_path=str(out))
    d = json.loads(out.read_text())
    assert d["dram_bytes_per_launch"] == round(sum(expect) / 4)
    assert d["source_hash"] == bench.kernel_source_hash()
    assert all(v["ncu_duration_ns"] == 12500 for v in d["per_shape"].values())
    alg = [bench.alg_bytes("int4", 1, N, K) for _, K, N, _ in bench.DECODE_SHAPES]
    assert d["algorithmic_bytes_per_launch"] == sum(alg) // 4


def test_traffic_summary_rejects_a_short_capture(tmp_path):
    csv_path = tmp_path / "t.csv"
    csv_path.write_text(HEADER + _row(0, "gemv_kernel", "dram__bytes_read.sum", "byte", "1"))
    try:
        bench.write_traffic(str(csv_path), 1, out_path=str(tmp_path / "o.json"))
    except SystemExit as e:
        assert "expected 4" in str(e)
    else:
        raise AssertionError("a capture with one launch was accepted")
