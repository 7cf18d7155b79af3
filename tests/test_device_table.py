"""The per-device once-guards of the library's host code (kernel attribute
opt-ins, SM counts) are kept per device ordinal: a process that drives two
GPUs sets each kernel's shared-memory opt-in on both. Compiled from the
library's own header with the host C++ compiler; no GPU needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_device_table_is_indexed_by_device(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path / "device_table_check")
    subprocess.run([cxx, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "vlm_visual_token_b200", "csrc"),
                    os.path.join(ROOT, "tests", "cpp", "device_table_check.cpp"), "-o", exe],
                   check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "device table ok" in out.stdout


def test_graph_list_schedule_is_complete_and_deadlock_free(tmp_path):
    """The host list schedule of the single-launch connector GEMM: every
    tile once, increasing per-pair lists, and an execution that respects the
    row-block dependencies always finishes."""
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path / "graph_schedule_check")
    subprocess.run([cxx, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "vlm_visual_token_b200", "csrc"),
                    os.path.join(ROOT, "tests", "cpp", "graph_schedule_check.cpp"), "-o", exe],
                   check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "graph schedule ok" in out.stdout
