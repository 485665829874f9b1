"""The DRAM-traffic records bench.py reports are tied to the kernel sources
they were measured on: a kernel's sources are its translation unit and every
csrc/ header it includes (transitively), and a record whose hash no longer
matches those sources is reported as null."""
import importlib.util
import json
import os
import shutil

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_sources_follow_includes():
    b = _bench()
    src = b.kernel_sources("fused_fwd_t2")
    assert "conv1d_t2.cu" in src
    for header in ("umma.cuh", "tc_common.cuh", "plan.h"):
        assert header in src
    assert not any(f.endswith("fftconv.h") for f in src)
    assert "conv1d_simt.cu" in b.kernel_sources("mp_pass2") and "tables.h" in b.kernel_sources("mp_pass2")
    assert b.kernel_sources("no_such_kernel") == []


def test_any_included_header_changes_the_hash(tmp_path, monkeypatch):
    b = _bench()
    csrc = tmp_path / "csrc"
    shutil.copytree(b.CSRC, csrc)
    monkeypatch.setattr(b, "CSRC", str(csrc))
    before = b.kernel_source_hash("fused_fwd_t2")
    with open(csrc / "tc_common.cuh", "a") as f:   # a header reached only through an include
        f.write("\n// edited\n")
    assert b.kernel_source_hash("fused_fwd_t2") != before
    other = b.kernel_source_hash("c2_pass2")         # conv2d_simt.cu does not include it
    with open(csrc / "tc_common.cuh", "a") as f:
        f.write("// again\n")
    assert b.kernel_source_hash("c2_pass2") == other


def test_stale_or_foreign_records_report_nothing(tmp_path, monkeypatch):
    b = _bench()
    path = tmp_path / "traffic.json"
    good = b.kernel_source_hash("fused_fwd_t2")
    json.dump({"w": {"kernel": "fused_fwd_t2", "dram_bytes_per_launch": 123.0, "source_hash": good},
               "stale": {"kernel": "fused_fwd_t2", "dram_bytes_per_launch": 5.0, "source_hash": "0" * 16}},
              open(path, "w"))
    monkeypatch.setattr(b, "TRAFFIC_JSON", str(path))
    assert b.recorded_traffic("w", "fused_fwd_t2") == 123.0
    assert b.recorded_traffic("w", "fused_fwd_tc") is None       # another kernel
    assert b.recorded_traffic("stale", "fused_fwd_t2") is None    # sources changed since
    assert b.recorded_traffic("absent", "fused_fwd_t2") is None


def test_committed_records_name_known_kernels():
    b = _bench()
    recs = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for cfg, e in recs.items():
        assert e["kernel"] in b.KERNEL_UNITS, cfg
        assert e["dram_bytes_per_launch"] > 0 and e["command"], cfg
