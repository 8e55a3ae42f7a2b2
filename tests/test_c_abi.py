"""The public header compiles as plain C (C11, warnings as errors) and a C program links the shared library and
gets answers from its host-only entry points (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from sparse_expert_moe_b200 import moe

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CUDA_INCLUDE = "/usr/local/cuda/include"


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.isdir(CUDA_INCLUDE),
                    reason="needs gcc and the CUDA headers")
def test_c_client_builds_links_and_runs(tmp_path):
    if not os.path.exists(moe.LIB_PATH):
        from sparse_expert_moe_b200 import build
        build.build()
    exe = tmp_path / "abi_check"
    lib_dir = os.path.dirname(moe.LIB_PATH)
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), "-isystem", CUDA_INCLUDE,
           os.path.join(HERE, "c_abi", "abi_check.c"), "-o", str(exe),
           "-L", lib_dir, "-l:libmoe_b200.so", f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAIL" not in r.stdout
