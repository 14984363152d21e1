"""bench.py's roofline.traffic comes from a committed ncu record of the
dominant kernel, and only while that record still describes the kernel: same
kernel and workload, and the kernel's source files hashing to the recorded
value.  Host logic only (no GPU); the records here are temporary copies of the
committed one, so the tests hold whether or not it is current."""
import hashlib
import os

import bench


def _fields(path):
    rec = {}
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#") and "=" in line:
            k, v = line.split("=", 1)
            rec[k.strip()] = v.strip()
    return rec


def _record(tmp_path, **over):
    """A copy of the committed record whose hash is that of the sources as they
    are now, with the given fields replaced."""
    src = os.path.join(bench.ROOT, bench.TRAFFIC_RECORDS[0])
    h = hashlib.sha256()
    for f in _fields(src)["kernel_sources"].split():
        with open(os.path.join(bench.ROOT, f), "rb") as fh:
            h.update(fh.read())
    over = {"kernel_sources_sha256": h.hexdigest(), **over}
    lines = []
    for line in open(src):
        key = line.split("=", 1)[0].strip()
        if key in over and not line.startswith("#"):
            line = f"{key}={over[key]}\n"
        lines.append(line)
    p = tmp_path / "record.traffic.txt"
    p.write_text("".join(lines))
    return str(p)


def test_matching_record_gives_its_traffic(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_RECORDS", [_record(tmp_path, dram_bytes_per_launch="123456")])
    traffic, source = bench.recorded_traffic("experts_fused_gate_up_down", 128, 0.15)
    assert traffic == 123456.0 and source.endswith("record.traffic.txt")


def test_changed_sources_give_no_traffic(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_RECORDS", [_record(tmp_path, kernel_sources_sha256="0" * 64)])
    traffic, why = bench.recorded_traffic("experts_fused_gate_up_down", 128, 0.15)
    assert traffic is None and "changed" in why


def test_other_workload_or_kernel_gives_no_traffic(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_RECORDS", [_record(tmp_path)])
    assert bench.recorded_traffic("experts_fused_gate_up_down", 256, 0.15)[0] is None
    assert bench.recorded_traffic("experts_fused_gate_up_down", 128, 0.35)[0] is None
    assert bench.recorded_traffic("router_gemm", 128, 0.15)[0] is None
    assert bench.recorded_traffic("experts_fused_gate_up_down", 128, 0.15)[0] is not None
