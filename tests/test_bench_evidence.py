"""bench.py's traffic evidence: how ncu DRAM figures are tied to the kernel
sources they were taken on, and that the committed figures are sane."""
import json
import os
import shutil

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _copy_csrc(tmp_path):
    dst = tmp_path / "paged_kv_cache_424_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "paged_kv_cache_424_b200", "csrc"), dst)
    return str(tmp_path), dst


def test_tensor_core_files_key_only_the_tensor_core_kernel(tmp_path):
    root, csrc = _copy_csrc(tmp_path)
    tc0, simt0 = bench.kernel_source_hash(True, root), bench.kernel_source_hash(False, root)
    assert (tc0, simt0) == (bench.kernel_source_hash(True), bench.kernel_source_hash(False))
    for name in bench.TC_ONLY_SOURCES:
        assert (csrc / name).exists()
    (csrc / "pa_decode_tc.cu").write_text((csrc / "pa_decode_tc.cu").read_text() + "\n// edit\n")
    assert bench.kernel_source_hash(True, root) != tc0
    assert bench.kernel_source_hash(False, root) == simt0
    # a file both kernels are built from changes both keys
    (csrc / "pa_common.cuh").write_text((csrc / "pa_common.cuh").read_text() + "\n// edit\n")
    assert bench.kernel_source_hash(False, root) != simt0


def test_committed_traffic_entries_are_sane():
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    wl = rec["workloads"]
    assert {"mha7b", "gqa8b", "long70b", "mha7b-fp8", "gqa8b-fp8", "long70b-fp8"} <= set(wl)
    for name, e in wl.items():
        assert len(e["kernel_src_sha"]) == 16, name
        assert ("decode_tc_kernel" in e["kernel"]) != ("decode_part_kernel" in e["kernel"]), name
        # DRAM bytes of one launch: the algorithmic bytes plus table, length and partial overhead
        assert 1.0 <= e["traffic_over_algorithmic"] <= 1.1, name
        total = e["dram_read_bytes"] + e["dram_write_bytes"]
        assert total == pytest.approx(e["dram_bytes_per_unit"] * e["units"], rel=1e-9), name
        assert "--clock-control none" in e["command"], name


def test_traffic_lookup_follows_the_hash(tmp_path, monkeypatch):
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    name, ent = "mha7b", rec["workloads"]["mha7b"]
    fake = tmp_path / "traffic.json"
    ent = dict(ent, kernel_src_sha=bench.kernel_source_hash("decode_tc_kernel" in ent["kernel"]))
    fake.write_text(json.dumps({"workloads": {name: ent}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(fake))
    assert bench.ncu_traffic(name, 1000.0) == pytest.approx(ent["dram_bytes_per_unit"] * 1000.0)
    assert bench.ncu_traffic("no-such-workload", 1000.0) is None
    fake.write_text(json.dumps({"workloads": {name: dict(ent, kernel_src_sha="0" * 16)}}))
    assert bench.ncu_traffic(name, 1000.0) is None  # taken on other sources: no figure
