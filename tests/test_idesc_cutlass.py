"""The tcgen05 block-scaled instruction descriptors the kernels issue (NVFP4: E2M1 x E2M1 with
E4M3 scales per 16; MXFP4: UE8M0 scales per 32, with the per-MMA scale byte index) are checked
field for field against CUTLASS's sm100 construction of the same descriptors, before any of them
reaches a GPU (CPU only: nvcc compiles a host program; skipped when nvcc or the CUTLASS headers
are missing)."""

import glob
import os
import shutil
import subprocess
import sysconfig

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _cutlass_include():
    site = sysconfig.get_paths()["purelib"]
    for pat in ("flashinfer/data/cutlass/include", "tilelang/3rdparty/cutlass/include"):
        for d in glob.glob(os.path.join(site, pat)):
            if os.path.exists(os.path.join(d, "cute", "arch", "mma_sm100_desc.hpp")):
                return d
    return None


def _nvcc():
    for c in ("/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    return None


FIELDS = {  # name: (first bit, width), from the sm100 block-scaled descriptor layout
    "b_sf_id": (4, 2), "a_format": (7, 3), "b_format": (10, 3), "a_major": (15, 1),
    "b_major": (16, 1), "n_dim": (17, 6), "scale_format": (23, 1), "m_dim": (24, 5),
    "a_sf_id": (29, 2), "k_size": (31, 1),
}


def test_descriptors_match_cutlass(tmp_path):
    inc, nvcc = _cutlass_include(), _nvcc()
    if inc is None or nvcc is None:
        pytest.skip("CUTLASS headers or nvcc not available")
    exe = str(tmp_path / "idesc_check")
    subprocess.run([nvcc, "-std=c++17", "-arch=sm_100a", "-I", inc, "-o", exe,
                    os.path.join(HERE, "idesc_check.cu")], check=True, capture_output=True)
    lines = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
    seen = 0
    for line in filter(None, lines):
        name, ours, theirs = line.split()
        ours, theirs = int(ours, 16), int(theirs, 16)
        for field, (lo, width) in FIELDS.items():
            a = (ours >> lo) & ((1 << width) - 1)
            b = (theirs >> lo) & ((1 << width) - 1)
            assert a == b, f"{name}: {field} {a} != {b}"
        assert ours == theirs, name
        if name.startswith("mxf4") and "byte2" in name:
            assert (ours >> 29) & 3 == 2 and (ours >> 4) & 3 == 2
        if name.startswith("mxf4"):
            assert (ours >> 23) & 1 == 1   # UE8M0 scales
        seen += 1
    assert seen == 9
