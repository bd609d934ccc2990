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


def test_committed_record_names_existing_sources(bench_mod):
    """The committed record names files of the tree; bench reports its figure while they
    match and null (not an error) once the kernel changed."""
    from microscaling_fp4_quantized_b200 import workloads as W
    with open(os.path.join(ROOT, "profiles", "attn_fp4_fwd_kernel_traffic.json")) as f:
        rec = json.load(f)
    for s in rec["sources"]:
        assert os.path.isfile(os.path.join(ROOT, s)), s
    t, src = bench_mod._attn_traffic(W.LONG)
    assert (t is not None and t > 0) or src == "kernel changed since the capture", src
