"""The C ABI from plain C: tests/c_abi_check.c includes include/fa.h under
gcc -std=c99 -Wall -Werror, links the built library and calls every entry
point with arguments the library must reject (or accept as empty) before any
CUDA call, so it runs on a machine without a GPU."""
import os
import shutil
import subprocess

import pytest

from tiled_attention_16_b200.build import LIB, build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_header_compiles_as_c99_and_entry_points_reject_bad_arguments(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    build()
    exe = tmp_path / "c_abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(HERE, "c_abi_check.c"), LIB, f"-Wl,-rpath,{os.path.dirname(LIB)}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, f"check {r.returncode} failed: {r.stderr}"
    assert r.stdout.strip() == "c abi ok"
