"""Host logic of bench.py's roofline fields: a committed traffic record is
used only while the kernel sources it names still hash to the recorded
value, and every record names sources that exist."""
import glob
import os

import pytest

import bench


def _records():
    return sorted(glob.glob(os.path.join(bench.ROOT, "profiles", "gemm1_*_traffic.txt")))


def _fields(path):
    vals = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    return vals


@pytest.mark.parametrize("path", _records(), ids=lambda p: os.path.basename(p))
def test_record_is_well_formed(path):
    vals = _fields(path)
    for key in ("kernel_sources", "kernel_source_sha256_16", "small_case_units", "full_size_units",
                "dram_bytes_per_launch_small", "dram_bytes_per_launch_full_size"):
        assert key in vals, key
    for name in vals["kernel_sources"].split():
        assert os.path.exists(os.path.join(bench.ROOT, bench.CSRC, name)), name
    small, full = int(vals["dram_bytes_per_launch_small"]), int(vals["dram_bytes_per_launch_full_size"])
    su, fu = int(vals["small_case_units"]), int(vals["full_size_units"])
    assert abs(full - small / su * fu) <= 1  # the full-size figure is the small case scaled by units
    # the command that produced it is in the header, with the clock flag
    text = open(path).read()
    assert "ncu --metrics" in text and "--clock-control none" in text


def test_decode_records_match_the_current_sources():
    # the decode kernel's records are keyed on moe_gemm.cu + moe_ptx.cuh
    for path in _records():
        vals = _fields(path)
        if vals["kernel_sources"].split() == ["moe_gemm.cu", "moe_ptx.cuh"]:
            name = os.path.basename(path)[len("gemm1_"):-len("_traffic.txt")]
            assert bench.recorded_traffic(name) == float(vals["dram_bytes_per_launch_full_size"]), name


def test_a_stale_hash_gives_no_traffic(tmp_path, monkeypatch):
    src = _records()[0]
    text = open(src).read()
    vals = _fields(src)
    stale = text.replace(vals["kernel_source_sha256_16"], "0" * 16)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / os.path.basename(src)).write_text(stale)
    # sources still resolve from the real tree; only the record lives in tmp
    real_root = bench.ROOT
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    for sub in ("fp4_block_scaled_route_b200",):
        os.symlink(os.path.join(real_root, sub), tmp_path / sub)
    name = os.path.basename(src)[len("gemm1_"):-len("_traffic.txt")]
    assert bench.recorded_traffic(name) is None
    assert bench.recorded_traffic("no_such_workload") is None
