"""The C ABI from C: tests/c/abi_check.c includes include/omni.h as C99
(-Wall -Werror), links libomni.so and checks the host-side argument checks
of every entry point.  CPU only: nothing it calls reaches the GPU."""
import os
import shutil
import subprocess

import pytest

from atomic_expert_layer_b200 import _lib, build as lib_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_host_checks_hold(tmp_path):
    lib_build.build()
    exe = tmp_path / "abi_check"
    pkg = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_check.c"),
                    "-L", pkg, "-l:libomni.so", "-Wl,-rpath," + pkg, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "all expectations held" in r.stdout
