"""Host-side logic of bench.py that needs no GPU: the DRAM traffic it reports next to the
roofline comes from a committed ncu record and is withheld once any of the kernel sources
the record names has changed (the counters would describe another kernel); for another
workload it is scaled by B*H*N (the quantized inputs plus the output)."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


@pytest.fixture()
def bench_mod():
    import bench
    return bench


def _write_record(root, srcs, bytes_per_launch, workload):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    h = hashlib.sha256()
    for s in srcs:
        with open(os.path.join(root, s), "rb") as f:
            h.update(f.read())
    rec = {"sources": srcs, "source_sha256_prefix": h.hexdigest()[:16], "captured_workload": workload,
           "dram_bytes_per_launch": bytes_per_launch}
    with open(os.path.join(root, "profiles", "attn_fp4_fwd_kernel_traffic.json"), "w") as f:
        json.dump(rec, f)


def test_traffic_reported_while_sources_match(bench_mod, tmp_path, monkeypatch):
    from microscaling_fp4_quantized_b200 import workloads as W
    for name in ("a.cuh", "b.h"):
        (tmp_path / name).write_text(f"// {name}\n")
    _write_record(str(tmp_path), ["a.cuh", "b.h"], 1000.0, W.PROFILE.name)
    monkeypatch.setattr(bench_mod, "ROOT", str(tmp_path))
    t, src = bench_mod._attn_traffic(W.PROFILE)
    assert t == 1000.0 and W.PROFILE.name in src
    # another workload: scaled by B*H*N
    t2, src2 = bench_mod._attn_traffic(W.LONG)
    scale = (W.LONG.B * W.LONG.H * W.LONG.N) / (W.PROFILE.B * W.PROFILE.H * W.PROFILE.N)
    assert t2 == pytest.approx(1000.0 * scale) and "scaled" in src2
    # any named source edited: withheld
    (tmp_path / "b.h").write_text("// edited\n")
    t3, src3 = bench_mod._attn_traffic(W.PROFILE)
    assert t3 is None and "changed" in src3


def test_traffic_absent_record(bench_mod, tmp_path, monkeypatch):
    from microscaling_fp4_quantized_b200 import workloads as W
    monkeypatch.setattr(bench_mod, "ROOT", str(tmp_path))
    assert bench_mod._attn_traffic(W.LONG) == (None, "no capture")


def test_write_traffic_record_from_ncu_csv(bench_mod, tmp_path, monkeypatch):
    """The record is written from an ncu CSV (one row per launch and metric, bytes in any
    of ncu's units) and hashed over the sources as they are when it is written, so that
    _attn_traffic reports it until a source changes."""
    from microscaling_fp4_quantized_b200 import workloads as W
    kernel, name, srcs = bench_mod.TRAFFIC_SOURCES[False]
    for s in srcs:
        os.makedirs(os.path.dirname(str(tmp_path / s)), exist_ok=True)
        (tmp_path / s).write_text(f"// {s}\n")
    os.makedirs(str(tmp_path / "profiles"))
    head = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Section Name",'
            '"Metric Name","Metric Unit","Metric Value"')
    rows = [
        '"0","1","python","h","stats_kernel<128>","1","7","","dram__bytes_read.sum","Mbyte","9.00"',
        f'"4","1","python","h","void sage::{kernel}<128, false, 0>(...)","1","7","","dram__bytes_read.sum","Mbyte","60.50"',
        f'"4","1","python","h","void sage::{kernel}<128, false, 0>(...)","1","7","","dram__bytes_write.sum","byte","16,777,216"',
    ]
    csv_path = tmp_path / "traffic.csv"
    csv_path.write_text("==PROF== noise line\n" + head + "\n" + "\n".join(rows) + "\n")
    monkeypatch.setattr(bench_mod, "ROOT", str(tmp_path))
    rec = bench_mod.write_traffic_record(str(csv_path), W.PROFILE, False)
    assert rec["dram_bytes_per_launch"] == pytest.approx(60.5e6 + 16777216)
    assert rec["launches_captured"] == 1
    t, src = bench_mod._attn_traffic(W.PROFILE)
    assert t == pytest.approx(60.5e6 + 16777216) and W.PROFILE.name in src
    (tmp_path / srcs[0]).write_text("// edited\n")
    assert bench_mod._attn_traffic(W.PROFILE)[0] is None


def test_committed_record_names_existing_sources(bench_mod):
    """The committed record (if any) names files of the tree; bench reports its figure while
    they match and null (not an error) once the kernel changed."""
    from microscaling_fp4_quantized_b200 import workloads as W
    path = os.path.join(ROOT, "profiles", "attn_fp4_fwd_kernel_traffic.json")
    if not os.path.exists(path):
        assert bench_mod._attn_traffic(W.LONG) == (None, "no capture")
        return
    with open(path) as f:
        rec = json.load(f)
    for s in rec["sources"]:
        assert os.path.isfile(os.path.join(ROOT, s)), s
    t, src = bench_mod._attn_traffic(W.LONG)
    assert (t is not None and t > 0) or src == "kernel changed since the capture", src


def test_quant_algorithmic_bytes_long_workload():
    """The quantizer's algorithmic bytes for the long workload: Q, K, V read (604 MB), K
    read again (201 MB), FP4 codes and scales written (170 MB) -- 975 MB."""
    import bench
    from microscaling_fp4_quantized_b200 import workloads as W
    E = 24 * 32768 * 128
    assert bench.quant_algorithmic_bytes(W.LONG) == 4 * E * 2 + 3 * E * 0.5625
    assert abs(bench.quant_algorithmic_bytes(W.LONG) / 1e6 - 975.2) < 0.5
    assert bench.quant_algorithmic_bytes(W.LONG, b8=True) == 13 * E
