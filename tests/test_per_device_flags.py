"""The per-device flag behind the attention kernels' shared-memory attribute
(CUDA sets it for the current device only), compiled and run on the host."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "paged_kv_cache_frame_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_attribute_is_set_once_per_device(tmp_path):
    exe = tmp_path / "per_device_flags"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, os.path.join(HERE, "cpp", "per_device_flags.cpp"),
                    "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("ok ") == 9, r.stdout
