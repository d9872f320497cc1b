"""Gated-MLP intermediate on the GPU: h = bf16(silu(gate) * up) from the
fused gate/up output, its dynamic NVFP4 quantization, and the down
projection -- each stage checked against the oracle applied to the GPU's
own input to that stage, so errors do not cascade."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import DEV, check_gemm, host

pytestmark = pytest.mark.gpu


def _ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    def key(b):
        b = b.astype(np.int64)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(key(a_bits) - key(b_bits))


@pytest.mark.parametrize("M,F", [(1, 16), (130, 64), (300, 336)])
def test_swiglu_quantize_small(M, F):
    rng = np.random.default_rng(M + F)
    gu = wl.to_bf16(rng.standard_normal((M, 2 * F)) * 4)
    h, hc, hsf, gh = ops.swiglu_quantize(gu.to(DEV))
    torch.cuda.synchronize()
    h_bits = host(h.view(torch.int16)).view(np.uint16)
    h_ref = oracle.swiglu(wl.bf16_bits(gu))
    assert np.max(_ulp_distance(h_bits, h_ref)) <= 1
    # quantization of the GPU's h is the oracle's, bit for bit
    c_ref, s_ref, g_ref = oracle.quantize_tensor(h_bits)
    assert float(host(gh)[0]) == float(g_ref)
    assert np.array_equal(host(hc), c_ref)
    assert np.array_equal(host(hsf), oracle.swizzle(s_ref, F))


def test_prefill_mlp_full_size():
    """gate_up (fused, 2 segments) -> SwiGLU + quantize -> down, M=8192,
    hidden 5120, width 17408."""
    gu_lin, down_lin = wl.mlp_modules()
    M, K, F = 8192, 5120, 17408
    X = wl.activation_normal(M, K, 2)
    Wgu = wl.fused_weight(gu_lin, 2)
    Wd = wl.weight_normal(K, F, 0.02, 77)
    qgu = ops.quantize_weights(Wgu.to(DEV), gu_lin.segments)
    qd = ops.quantize_weights(Wd.to(DEV))
    gate_up = ops.linear_fused(X.to(DEV), qgu)
    h, hc, hsf, gh = ops.swiglu_quantize(gate_up)
    y = ops.gemm_prequant(hc, hsf, gh, M, F, qd, out_fp32=True)
    assert ops.get_status() == 0
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.integers(0, M, 48), [0, M - 1]]))
    gu_bits = host(gate_up.view(torch.int16)).view(np.uint16)
    h_bits = host(h.view(torch.int16)).view(np.uint16)
    # SwiGLU on the GPU's gate_up rows
    assert np.max(_ulp_distance(h_bits[rows], oracle.swiglu(np.ascontiguousarray(gu_bits[rows])))) <= 1
    # the dynamic scale of the GPU's h, and its codes for the sampled rows
    g_ref = oracle.global_scale(oracle.amax(h_bits))
    assert float(host(gh)[0]) == g_ref
    c_ref, s_ref = oracle.quantize(np.ascontiguousarray(h_bits[rows]), np.float32(g_ref))
    assert np.array_equal(host(hc)[rows], c_ref)
    assert np.array_equal(oracle.unswizzle(host(hsf), M, F)[rows], s_ref)
    # down projection on sampled outputs
    wd_bits = wl.bf16_bits(Wd)
    g_d = oracle.global_scale(oracle.amax(wd_bits))
    cols = np.unique(np.concatenate([rng.integers(0, K, 96), np.arange(K - 40, K)]))
    wc, wsc = oracle.quantize(np.ascontiguousarray(wd_bits[cols]), np.float32(g_d))
    assert np.array_equal(host(qd.codes)[cols], wc)
    im, inn = np.meshgrid(np.arange(len(rows)), np.arange(len(cols)), indexing="ij")
    C, B = oracle.linear_sampled(c_ref, s_ref, g_ref, wc, wsc, np.float32(g_d), im.ravel(), inn.ravel())
    got = host(y)[rows][:, cols].ravel()
    check_gemm(got, C, B, "down projection")
