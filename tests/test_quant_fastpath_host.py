"""The NF4 quantiser's fast division-free code path, checked exhaustively on
the host.

For block scales in [2^-90, 2^100) the kernel replaces x = RN32(w / c) by a
correctly rounded reciprocal and one fused correction step, and the
nearest-level search by a fitted polynomial plus one threshold compare.
``fastpath_check.cpp`` replays that arithmetic for every bf16 pair (w, c)
with |w| <= c in that range (about 8.2e8 pairs) and requires the code of the
IEEE quotient (number of thresholds below w / c) every time.  Scales outside
the range take the IEEE division on the GPU (covered by the GPU quantiser
tests)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_nf4_quantized_15_b200", "csrc")


@pytest.mark.slow
def test_fast_quotient_gives_the_ieee_code_for_every_bf16_pair(tmp_path):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    cuda_inc = "/usr/local/cuda/include"
    exe = str(tmp_path / "fastpath_check")
    cmd = [cxx, "-O2", "-ffp-contract=off", "-fopenmp", "-std=c++17", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
           "-I", cuda_inc, os.path.join(ROOT, "tests", "fastpath_check.cpp"), os.path.join(CSRC, "nf4_tables.cpp"),
           "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=900)
    line = out.stdout.strip().splitlines()[-1]
    fields = dict(kv.split("=") for kv in line.split())
    assert out.returncode == 0, out.stdout
    assert int(fields["mismatches"]) == 0 and int(fields["k_out_of_range"]) == 0
    assert int(fields["pairs"]) > 8.0e8
