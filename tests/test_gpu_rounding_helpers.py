"""Exhaustive GPU checks of the row-wise append kernel's rounding helpers.

The fast encoding of that kernel divides each group's abs-max by 7 with
Markstein's method (one product with RN(1/7) and one fused correction) and takes
the reciprocal of the binary16 scale with rcp.approx.f32. Its exactness argument
needs the first to equal the IEEE division for every finite abs-max, and the
second to stay within one unit in the last place. This test compiles
tests/cuda/check_rounding_helpers.cu against the library's own device header and
checks both over every input they can receive.
"""
import json
import os
import shutil
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_div7_and_rcp_over_every_input(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "check_rounding_helpers")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-Xcompiler", "-ffp-contract=off", "-o", exe,
                    os.path.join(HERE, "cuda", "check_rounding_helpers.cu")], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=120).stdout
    res = json.loads(out.strip().splitlines()[-1])
    assert res["cuda"] == "no error"
    assert res["div7_checked"] == 0x7F800000  # +0 and every positive finite binary32
    assert res["div7_mismatches"] == 0, f"first mismatch at bits {res['first_mismatch']:#x}"
    assert res["rcp_max_rel_err_ulp23"] <= 1.0
