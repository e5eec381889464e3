"""The C ABI from a C program (no Python in between): the header compiles as C99 with gcc, the
program links against the built library and its rule checks answer before any CUDA call, so it
runs without a GPU."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is needed to build the C client")
def test_c_client_builds_links_and_gets_rule_errors(tmp_path):
    from nvfp4_block_scaled_mm_b200.build import build
    lib = build(quiet=True)
    exe = tmp_path / "abi_from_c"
    src = os.path.join(ROOT, "tests", "c_abi", "abi_from_c.c")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
           "-o", str(exe), "-L", os.path.dirname(lib), "-lnvfp4lora", "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.count("ok ") == 7 and "FAIL" not in run.stdout
