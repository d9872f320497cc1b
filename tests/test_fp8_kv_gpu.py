"""FP8 (E4M3) KV-cache quantization on the GPU against the oracle: the
calibrated scale and every code bit-exact, for ragged and strided shapes,
static scales that saturate or take the exact-division fallback, signed
zeros, invalid scales, and the full-size KV cache of one attention layer."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import DEV, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols", [(1, 8), (37, 64), (300, 136), (129, 1024), (2, 4096)])
def test_calibrate_and_quantize_bit_exact(rows, cols):
    X = wl.activation_normal(rows, cols, seed=rows + cols, n_outliers=min(2, cols // 8), scale=30.0)
    xd = X.to(DEV)
    s = ops.fp8_kv_calibrate(xd)
    q = ops.fp8_kv_quantize(xd, s)
    assert ops.get_status() == 0
    xb = wl.bf16_bits(X)
    s_ref = oracle.fp8_kv_scale(oracle.amax(xb))
    assert float(host(s)[0]) == s_ref
    assert np.array_equal(host(q), oracle.fp8_kv_quantize(xb, s_ref))


def test_strided_input_and_output():
    rows = 53
    base = wl.activation_student_t(rows, 200, seed=9).to(DEV)
    X = base[:, 24:24 + 128]  # leading dimension 200, base 48 bytes in
    out_base = torch.full((rows, 160), 0xAB, dtype=torch.uint8, device=DEV)
    out = out_base[:, :128]
    s = ops.fp8_kv_calibrate(X)
    ops.fp8_kv_quantize(X, s, out=out)
    assert ops.get_status() == 0
    xb = wl.bf16_bits(X)
    s_ref = oracle.fp8_kv_scale(oracle.amax(np.ascontiguousarray(xb)))
    assert float(host(s)[0]) == s_ref
    assert np.array_equal(host(out), oracle.fp8_kv_quantize(np.ascontiguousarray(xb), s_ref))
    assert np.all(host(out_base)[:, 128:] == 0xAB)  # padding columns untouched


@pytest.mark.parametrize("scale", [2.0 ** -90, 1e-3, 0.05, 7.3, 2.0 ** 90])
def test_static_scales(scale):
    """A too-small scale saturates most codes at +-448; 2^-90 takes the IEEE
    division path (the shared-divisor quotient would leave its exact range);
    2^90 sends everything to signed zero."""
    X = wl.activation_normal(64, 256, seed=17, n_outliers=4, scale=50.0)
    xd = X.to(DEV)
    s = torch.tensor([scale], dtype=torch.float32, device=DEV)
    q = ops.fp8_kv_quantize(xd, s)
    assert ops.get_status() == 0
    ref = oracle.fp8_kv_quantize(wl.bf16_bits(X), float(np.float32(scale)))
    assert np.array_equal(host(q), ref)


def test_zero_tensor_and_signed_zero():
    x = np.zeros((16, 32), dtype=np.float32)
    x[::2, ::3] = -0.0
    X = wl.to_bf16(x)
    xd = X.to(DEV)
    s = ops.fp8_kv_calibrate(xd)
    q = ops.fp8_kv_quantize(xd, s)
    assert ops.get_status() == 0
    assert float(host(s)[0]) == 1.0
    assert np.array_equal(host(q), oracle.fp8_kv_quantize(wl.bf16_bits(X), 1.0))
    assert set(np.unique(host(q))) <= {0x00, 0x80}


@pytest.mark.parametrize("bad", [0.0, -1.0, float("nan"), float("inf")])
def test_invalid_scale_latches_nonfinite(bad):
    xd = wl.activation_normal(8, 16, seed=1).to(DEV)
    out = torch.full((8, 16), 0xAB, dtype=torch.uint8, device=DEV)
    ops.fp8_kv_quantize(xd, torch.tensor([bad], dtype=torch.float32, device=DEV), out=out)
    assert ops.get_status() == 6  # NVFP4_ERR_NONFINITE, read and cleared
    assert ops.get_status() == 0
    assert np.all(host(out) == 0xAB)


def test_empty():
    xd = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    q = ops.fp8_kv_quantize(xd, torch.ones(1, device=DEV))
    assert q.shape == (0, 64)
    s = ops.fp8_kv_calibrate(xd)
    assert ops.get_status() == 0 and float(host(s)[0]) == 1.0


def test_full_size_attention_kv_cache():
    """K and V caches of one attention layer at 8192 tokens, 8 KV heads x 128
    (the stack's attention k/v projection width 1024): calibrated scale
    bit-exact on the whole tensor, codes bit-exact on sampled rows plus the
    first and last."""
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([rng.integers(0, 8192, 64), [0, 8191]]))
    for seed in (101, 102):
        X = wl.activation_normal(8192, 1024, seed=seed, n_outliers=8, scale=20.0)
        xd = X.to(DEV)
        s = ops.fp8_kv_calibrate(xd)
        q = ops.fp8_kv_quantize(xd, s)
        assert ops.get_status() == 0
        xb = wl.bf16_bits(X)
        s_ref = oracle.fp8_kv_scale(oracle.amax(xb))
        assert float(host(s)[0]) == s_ref
        assert np.array_equal(host(q)[rows], oracle.fp8_kv_quantize(np.ascontiguousarray(xb[rows]), s_ref))
