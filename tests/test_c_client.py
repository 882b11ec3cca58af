"""The C ABI from plain C (CPU only): tests/c_abi_host.c includes include/nvfp4_moe.h as C99,
links the library and calls the entry points that need no GPU."""

import os
import shutil
import subprocess

import pytest

from nvfp4_block_scaled_gsa_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c99_client_builds_links_and_passes(tmp_path):
    lib = B.build()
    exe = tmp_path / "c_abi_host"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-o", str(exe),
           os.path.join(ROOT, "tests", "c_abi_host.c"), "-I", os.path.join(ROOT, "include"),
           "-L", libdir, "-lnvfp4moe", f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = r.stdout.splitlines()
    assert len(lines) == 16 and all(line.startswith("ok ") for line in lines), r.stdout
