"""Block-scaled FP4 GEMM on the tensor cores against the oracle's fp64 GEMM
over the same (oracle-quantized) operands: every output within
1e-5 * sum|a*b| + 1e-6; bf16 outputs equal the RNE rounding of the fp32
path; exact-integer problems bit-exact; no byte around an output buffer
is written (ragged tiles clipped at the edges).  Shapes with M > 128 run on the
CTA-pair kernel by default; each check also runs the one-CTA kernel
(NVFP4_SINGLE_CTA) on the same operands."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import (DEV, Guarded, bf16_of_f32, check_gemm, dev_u8, host, oracle_act_on_device,
                            oracle_weight_on_device)

pytestmark = pytest.mark.gpu


KERNELS = {"auto": 0, "single_cta": ops.NVFP4_SINGLE_CTA}


def _run(xb, wb, segments, flags=0):
    M, K = xb.shape
    (ac, asf, ga), (oc, os_, og) = oracle_act_on_device(xb)
    qw, (wc, ws, wg) = oracle_weight_on_device(wb, segments)
    g32 = Guarded((M, wb.shape[0]), torch.float32, fill=float("nan"))
    g16 = Guarded((M, wb.shape[0]), torch.bfloat16, fill=float("nan"))
    ops.gemm_prequant(ac, asf, ga, M, K, qw, out=g32.t, out_fp32=True, debug_flags=flags)
    ops.gemm_prequant(ac, asf, ga, M, K, qw, out=g16.t, debug_flags=flags)
    out32 = g32.check("fp32 output")
    out16 = g16.check("bf16 output")
    grow = oracle.rows_scale(segments, wg, wb.shape[0])
    C, B = oracle.linear_full(oc, os_, og, wc, ws, grow)
    return host(out32), host(out16.view(torch.int16)).view(np.uint16), C, B


def test_tiny_linear_full_parity():
    X, W = wl.tiny_linear(0)
    o32, o16, C, B = _run(wl.bf16_bits(X), wl.bf16_bits(W), [(0, 128)])
    check_gemm(o32, C, B, "tiny fp32")
    assert np.array_equal(o16, bf16_of_f32(o32))


SHAPES = [
    (1, 8, 64), (64, 48, 64), (129, 191, 192), (128, 192, 256), (300, 200, 320), (77, 385, 1024),
    (256, 400, 576), (5, 1000, 128), (513, 64, 2048), (200, 17, 256),
]


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_ragged_shapes(M, N, K, kernel):
    X = wl.activation_normal(M, K, seed=M + N + K, n_outliers=min(4, K // 16), scale=50.0)
    W = wl.weight_normal(N, K, 0.02, seed=3 * N + K)
    o32, o16, C, B = _run(wl.bf16_bits(X), wl.bf16_bits(W), [(0, N)], KERNELS[kernel])
    check_gemm(o32, C, B, f"{M}x{N}x{K}")
    assert np.array_equal(o16, bf16_of_f32(o32))


def _pack(cu):
    return (cu[:, 0::2] | (cu[:, 1::2] << 4)).astype(np.uint8)


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("M,N,K", [(128, 192, 256), (200, 400, 1024), (64, 130, 4096), (520, 700, 1280)])
def test_exact_integer_problem_bit_exact(M, N, K, kernel):
    """Codes in {0, +-1, +-2, +-4}, every scale 1.0, g = 1: all partial sums
    are integers below 2^24, so the tensor-core result must be exact."""
    rng = np.random.default_rng(M * N)
    choices = [0, 2, 4, 6, 10, 12, 14]
    ca = rng.choice(choices, size=(M, K))
    cw = rng.choice(choices, size=(N, K))
    one = 0x38
    sa = np.full((M, K // 16), one, np.uint8)
    sw = np.full((N, K // 16), one, np.uint8)
    a_codes, w_codes = _pack(ca), _pack(cw)
    qw = ops.QuantizedWeight(dev_u8(w_codes).view(N, K // 2), dev_u8(oracle.swizzle(sw, K)),
                             torch.ones(1, dtype=torch.float32, device=DEV), [(0, N)], N, K)
    g1 = torch.ones(1, dtype=torch.float32, device=DEV)
    out = ops.gemm_prequant(dev_u8(a_codes).view(M, K // 2), dev_u8(oracle.swizzle(sa, K)), g1, M, K, qw,
                            out_fp32=True, debug_flags=KERNELS[kernel])
    want = oracle.e2m1_table()[ca].astype(np.int64) @ oracle.e2m1_table()[cw].astype(np.int64).T
    assert np.array_equal(host(out).astype(np.float64), want.astype(np.float64))


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_scale_layout_drives_the_mma(kernel):
    """Distinct power-of-two scales per block and row: any mistake in the
    scale-factor layout or its TMEM placement changes the result."""
    rng = np.random.default_rng(21)
    M, N, K = 256, 384, 512
    ca = rng.choice([2, 10], size=(M, K))  # +-1
    cw = rng.choice([2, 10], size=(N, K))
    sa = rng.choice([0x28, 0x30, 0x38, 0x40, 0x48], size=(M, K // 16)).astype(np.uint8)  # 1/4 .. 4
    sw = rng.choice([0x28, 0x30, 0x38, 0x40, 0x48], size=(N, K // 16)).astype(np.uint8)
    qw = ops.QuantizedWeight(dev_u8(_pack(cw)).view(N, K // 2), dev_u8(oracle.swizzle(sw, K)),
                             torch.ones(1, dtype=torch.float32, device=DEV), [(0, N)], N, K)
    g1 = torch.ones(1, dtype=torch.float32, device=DEV)
    out = ops.gemm_prequant(dev_u8(_pack(ca)).view(M, K // 2), dev_u8(oracle.swizzle(sa, K)), g1, M, K, qw,
                            out_fp32=True, debug_flags=KERNELS[kernel])
    C, B = oracle.linear_full(_pack(ca), sa, 1.0, _pack(cw), sw, np.float32(1.0))
    assert np.array_equal(host(out).astype(np.float64), C)


def test_zero_sized():
    qw = ops.QuantizedWeight(torch.zeros((8, 32), dtype=torch.uint8, device=DEV),
                             torch.zeros(ops.sf_bytes(8, 64), dtype=torch.uint8, device=DEV),
                             torch.ones(1, device=DEV), [(0, 8)], 8, 64)
    g1 = torch.ones(1, dtype=torch.float32, device=DEV)
    a = torch.zeros((1, 32), dtype=torch.uint8, device=DEV)
    out = ops.gemm_prequant(a, torch.zeros(512, dtype=torch.uint8, device=DEV), g1, 0, 64, qw)
    assert out.shape == (0, 8)
