"""The quantizer divides each block's 16 elements by one decode scale with a
reciprocal plus one Markstein correction step (csrc/fp_div.cuh), two
quotients at a time with the packed f32x2 instructions.  This test compiles a
small CUDA program against that header and compares both forms, bit for bit,
with CUDA's IEEE division __fdiv_rn: every bf16 significand against every
fp32 significand (both signs, quotients across ten binades), and every finite
bf16 value against random divisors over the whole accepted range (quotients
below 2^-20, which all encode to +-0, need only stay below 0.25 with the right
sign)."""
import os
import re
import subprocess
import tempfile

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "nvfp4_w4a4_quantized_act_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def test_shared_divisor_division_is_ieee_exact():
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "div_exhaustive")
        subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                               "-I", CSRC, "-o", exe, os.path.join(HERE, "cuda", "div_exhaustive.cu")])
        out = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    m = re.search(r"checked=(\d+) mismatches=(\d+) accepted=(\d+)", out.stdout)
    assert m, out.stdout
    checked, bad, accepted = map(int, m.groups())
    assert checked > 30_000_000_000 and accepted > 1_000_000
    assert bad == 0, out.stdout
