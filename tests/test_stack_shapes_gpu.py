"""The fused GEMM shapes of the 496-linear stack at one 8192-token prefill
chunk, each checked against the oracle at full size through
nvfp4_linear_fused.

Every input-sharing group of modules is one GEMM with a global scale per
module ("Why Gated DeltaNet Survives 4-Bit Quantization", kipquest.com, "The
abstract" and "The deep dive": W4A4 on all linears, per-module calibrated
scales, fused modules).  The stack has six distinct GEMM shapes besides the
MLP's gate/up and down (covered in test_linear_gpu.py / test_mlp_gpu.py):

  GDN input projection   N = 8192 | 6144 | 48 | 48 = 14432, K = 5120
  attention q+gate/k/v   N = 12288 | 1024 | 1024  = 14336, K = 5120
  GDN out / attention o  N = 5120, K = 6144 (activation width 6144)

Each test compares >= 4096 sampled outputs plus every N-tail and
segment-boundary column of 64 rows with the oracle at
|gpu - oracle| <= 1e-5 * sum|a*b| + 1e-6, and checks the quantized operands
of the sampled rows bit for bit.  The K = 6144 activation is also quantized
whole and compared with the oracle's codec bit for bit (codes, swizzled
scales with their padding, global scale).
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import DEV, full_size_check, host

pytestmark = pytest.mark.gpu

TOKENS = 8192


def _stack_linear(name):
    for _, lins in wl.stack_layers():
        for lin in lins:
            if lin.name == name:
                return lin
    raise KeyError(name)


def _stack_activation(K, seed, n_outliers=4):
    # the stack's activations: N(0, 1) with 4 outlier channels x50 (none for
    # the attention/GDN output Y)
    return wl.activation_normal(TOKENS, K, seed, n_outliers=n_outliers)


@pytest.mark.parametrize("name,seed", [("gdn_in_proj", 51), ("attn_qkv", 52), ("gdn_out", 53)])
def test_stack_gemm_shape_full_size(name, seed):
    lin = _stack_linear(name)
    X = _stack_activation(lin.K, seed, n_outliers=0 if lin.K == 6144 else 4)
    W = wl.fused_weight(lin, seed)
    assert W.shape == (lin.N, lin.K)
    r = full_size_check(X, W, lin.segments, seed + 100)
    assert r <= 1.0


def test_stack_k6144_activation_codec_bit_exact():
    """The out/o projection's input Y [8192, 6144]: codes, swizzled scales
    (padding included) and the global scale, whole tensor, bit for bit."""
    Y = _stack_activation(6144, 54, n_outliers=0)
    yb = wl.bf16_bits(Y)
    codes, sf, g = ops.quantize_act(Y.to(DEV))
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    c_ref, s_ref, g_ref = oracle.quantize_tensor(yb)
    assert float(host(g)[0]) == float(g_ref)
    assert np.array_equal(host(codes).reshape(TOKENS, 3072), c_ref)
    assert np.array_equal(host(sf), oracle.swizzle(s_ref, 6144))
