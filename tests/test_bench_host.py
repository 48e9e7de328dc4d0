"""Host logic of bench.py on CPU: which sources key a committed ncu traffic figure, and how a
figure captured on one workload is carried to another workload of the same kernel."""
import json

import pytest

import bench


def _tree(tmp_path, header_body):
    (tmp_path / "k.cu").write_text('#include "a.cuh"\n#include <cuda.h>\n__global__ void k() {}\n')
    (tmp_path / "a.cuh").write_text('#include "b.cuh"\n' + header_body)
    (tmp_path / "b.cuh").write_text("// leaf\n")
    return str(tmp_path)


def test_sources_follow_local_includes(tmp_path):
    csrc = _tree(tmp_path, "int x;\n")
    assert bench.kernel_sources("k.cu", csrc) == ["k.cu", "a.cuh", "b.cuh"]


def test_hash_changes_with_an_included_header(tmp_path):
    csrc = _tree(tmp_path, "int x;\n")
    h0 = bench.kernel_source_hash("k.cu", csrc)
    (tmp_path / "b.cuh").write_text("// leaf, edited\n")
    assert bench.kernel_source_hash("k.cu", csrc) != h0


def test_every_kernel_entry_names_its_sources():
    with open(bench.PROFILE_TRAFFIC) as f:
        d = json.load(f)
    for kernel, e in d.items():
        if kernel.startswith("_"):
            continue
        assert e["sources"] == bench.kernel_sources(e["source"])


def test_traffic_is_scaled_to_the_benchmarked_launch(tmp_path):
    src = "gdr_prefill_tc.cu"
    entry = {"source": src, "source_hash": bench.kernel_source_hash(src), "workload": "w",
             "dram_bytes_per_launch_scaled": 1000, "algorithmic_bytes_per_launch": 2000}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps({"k": entry}))
    assert bench.traffic_for("k", src, 2000, str(path)) == (1000, None)
    t, note = bench.traffic_for("k", src, 8000, str(path))
    assert t == pytest.approx(4000) and "scaled" in note
    entry["source_hash"] = "stale"
    path.write_text(json.dumps({"k": entry}))
    assert bench.traffic_for("k", src, 2000, str(path)) == (None, None)
