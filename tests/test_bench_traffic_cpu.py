"""bench.py's DRAM-traffic bookkeeping on CPU: which source changes retire an ncu entry.

An entry of profiles/traffic.txt holds the DRAM bytes ncu measured for one kernel and
workload, keyed by a hash of the kernel's source file and the device headers that file
includes (recursively).  Any change to those files must retire the entry; a change to a
header the kernel does not include must not.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _tree(tmp_path):
    (tmp_path / "k.cu").write_text('#include <cuda.h>\n#include "a.cuh"\n__global__ void k() {}\n')
    (tmp_path / "a.cuh").write_text('#pragma once\n#include "b.cuh"\n')
    (tmp_path / "b.cuh").write_text("#pragma once\nconstexpr int kB = 1;\n")
    (tmp_path / "other.cuh").write_text("#pragma once\nconstexpr int kOther = 1;\n")
    return str(tmp_path / "k.cu")


def test_hash_follows_included_headers_only(tmp_path):
    src = _tree(tmp_path)
    h0 = bench.source_sha(src)
    (tmp_path / "other.cuh").write_text("#pragma once\nconstexpr int kOther = 2;\n")
    assert bench.source_sha(src) == h0                       # not included
    (tmp_path / "b.cuh").write_text("#pragma once\nconstexpr int kB = 2;\n")
    h1 = bench.source_sha(src)
    assert h1 != h0                                           # included through a.cuh
    (tmp_path / "k.cu").write_text('#include <cuda.h>\n#include "a.cuh"\n__global__ void k() { }\n')
    assert bench.source_sha(src) != h1                        # the kernel file itself


def test_include_cycles_terminate(tmp_path):
    src = _tree(tmp_path)
    (tmp_path / "b.cuh").write_text('#pragma once\n#include "a.cuh"\n')
    assert len(bench.source_sha(src)) == 12


def test_every_recorded_entry_names_a_kernel_source_and_is_well_formed():
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    sources = {"tq_tc_kernel": "transform_quant_tc.cu", "qgemm_pair_kernel": "qgemm.cu",
               "hgemm_pair_kernel": "qgemm_int4.cu"}
    for line in open(path):
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        assert f["kernel"] in sources and f["workload"] in ("up_proj", "down_proj", "int4")
        assert len(f["src_sha"]) == 12 and int(f["dram_bytes_per_launch"]) > 0
        assert os.path.exists(os.path.join(ROOT, f["source"]))
