"""The boundary is a C ABI: a C99 program compiles against include/wush.h with
-Wall -Werror (no C++, no CUDA headers), links libwush.so and runs host-only
calls -- sizes, status strings, calibration, the non-finite check, a transforms
checkpoint round trip and an argument check of a device entry point."""
import os
import shutil
import subprocess

import pytest

aq = pytest.importorskip("activation_quantization_b200")
HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_consumer(tmp_path):
    exe = tmp_path / "consumer"
    lib_dir = os.path.dirname(aq.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(HERE, "c_consumer", "consumer.c"),
                    "-o", str(exe), "-L", lib_dir, "-l:libwush.so", f"-Wl,-rpath,{lib_dir}", "-lm"],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe), str(tmp_path / "t.wush")], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "c consumer ok" in r.stdout
