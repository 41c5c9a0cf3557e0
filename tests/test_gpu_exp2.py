"""The attention softmax runs part of its exponentials on the FMA pipe (exp2_poly / exp2_poly2,
csrc/sm100.cuh: round-to-nearest split t = n + f, a cubic for 2^f fitted on [-1/2, 1/2], 2^n added
to the exponent bits). This test compiles tests/gpu/exp2_poly_check.cu with nvcc, runs it on the
GPU over a dense sweep of [-120, 8] and checks the stated bound against 2^t computed in double
precision on the host: max relative error <= 2.21e-4, the paired form bit-identical to the single
form, and the result non-decreasing across the sweep (including every split point n + 1/2)."""
import json
import os
import subprocess
import tempfile

import pytest

from block_sparse_long_moba_b200 import build

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gpu", "exp2_poly_check.cu")


def test_exp2_poly_error_bound_and_monotonicity():
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "exp2_poly_check")
        cmd = [build.nvcc(), *build.ARCH, "-O3", "-std=c++17", "-I", build.CSRC, SRC, "-o", exe]
        r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout + r.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
        assert r.returncode == 0, r.stdout + r.stderr
    res = json.loads(r.stdout.strip().splitlines()[-1])
    print(res)
    assert res["points"] == 128 * 8192 + 1
    assert res["max_rel"] <= 2.21e-4
    assert res["max_rel_pair"] <= 2.21e-4
    assert res["pair_mismatch"] == 0
    assert res["nonmonotone"] == 0
