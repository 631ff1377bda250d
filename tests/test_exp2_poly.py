"""The emulated exp2 (Cody-Waite reduction + degree-3 minimax polynomial)
that the prefill softmax runs on the FMA pipes for part of its exponentials,
checked on the CPU against std::exp2: the header is host-compilable and IEEE
fp32 FMA arithmetic is the same on the host and the GPU."""

import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_exp2_poly_error_bound():
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "exp2_poly_check")
        subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-o", exe,
                        os.path.join(HERE, "native", "exp2_poly_check.cpp")], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split()
    max_rel, worst_x, int_rel, below, neg_inf = map(float, out)
    assert max_rel < 8e-5, (max_rel, worst_x)      # minimax bound 7.5e-5 in fp32
    assert int_rel < 8e-5                          # p(0) = c0 = 1 - 7.2e-5
    assert 0.0 < below < 4e-38 and 0.0 < neg_inf < 4e-38  # clamped, never negative
