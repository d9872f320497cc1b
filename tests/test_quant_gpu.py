"""Activation / weight quantization on the GPU against the oracle: packed
codes, swizzled scale bytes (padding included) and global scales must match
bit for bit, and no byte around the codes and scale buffers may change."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import DEV, Guarded, dev_u8, host

pytestmark = pytest.mark.gpu


def _gpu_quant(X: torch.Tensor):
    M, K = X.shape
    gc = Guarded(M * K // 2, torch.uint8, fill=0x5A)
    gs = Guarded(ops.sf_bytes(M, K), torch.uint8, fill=0x5A)
    codes, sf, g = ops.quantize_act(X.to(DEV), codes=gc.t, sf=gs.t)
    gc.check("codes")
    gs.check("scale factors")
    return host(codes), host(sf), float(host(g)[0])


def _assert_same(X: torch.Tensor):
    xb = wl.bf16_bits(X)
    M, K = xb.shape
    c_gpu, sf_gpu, g_gpu = _gpu_quant(X)
    c_ref, s_ref, g_ref = oracle.quantize_tensor(xb)
    assert g_gpu == float(g_ref)
    assert np.array_equal(c_gpu.reshape(M, K // 2), c_ref)
    sw_ref = oracle.swizzle(s_ref, K)
    assert sf_gpu.shape[0] == sw_ref.shape[0]
    if not np.array_equal(sf_gpu, sw_ref):
        got = oracle.unswizzle(sf_gpu, M, K)
        bad = np.argwhere(got != s_ref)
        raise AssertionError(f"scale mismatch at {bad[:5].tolist()} (padding ok: "
                             f"{np.array_equal(got, s_ref)})")


def test_tiny_linear_operands_bit_exact():
    X, W = wl.tiny_linear(0)
    _assert_same(X)
    _assert_same(W)


@pytest.mark.parametrize("M,K", [(1, 16), (7, 48), (3, 80), (130, 64), (257, 272), (64, 320), (300, 1024), (33, 5120)])
def test_ragged_shapes_bit_exact(M, K):
    _assert_same(wl.activation_normal(M, K, seed=M * 31 + K, n_outliers=min(4, K // 16), scale=50.0))


def test_student_t_full_size_bit_exact():
    """The activation-quantize workload at full size: [8192, 5120]
    Student-t(3) with 1% of channels x100."""
    _assert_same(wl.act_quant_input())


def test_special_values():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((256, 128)).astype(np.float32)
    x[0, :16] = 0.0                           # all-zero block
    x[1, :16] = -0.0                          # negative zeros
    x[2, :16] = 1e-30                         # scale underflows to zero
    x[3, 16:32] = [6.0] + [-0.01] * 15        # negatives rounding to -0
    x[4, :] = np.float32(2.0) ** -100         # tiny block scales
    x[5, :16] = np.linspace(-3, 3, 16)        # exact ties after scaling
    x[6, :] = 1e4                             # one dominant row sets g
    x[7, :16] = [448.0 * 6] * 16
    _assert_same(wl.to_bf16(x))


def test_all_zero_tensor():
    _assert_same(torch.zeros((64, 256), dtype=torch.bfloat16))


def test_exhaustive_bf16_values():
    """Every finite bf16 value appears once, in blocks paired with a pivot
    that fixes each block's scale, across several tensor scales."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_bits_to_f32(allbits)
    fin = allbits[np.isfinite(vals)]
    n = len(fin)
    for pivot in (6.0, 1.0, 3.0e5, 1e-20):
        rows = (n + 14) // 15
        blk = np.zeros((rows, 16), dtype=np.uint16)
        blk[:, 0] = wl.bf16_bits(wl.to_bf16(np.array([pivot])))[0]
        flat = np.zeros(rows * 15, dtype=np.uint16)
        flat[:n] = fin
        blk[:, 1:] = flat.reshape(rows, 15)
        X = torch.from_numpy(blk.view(np.int16).reshape(-1, 64)).view(torch.bfloat16)
        _assert_same(X)


def test_static_scale():
    X = wl.activation_normal(200, 512, 5)
    xb = wl.bf16_bits(X)
    for g in (1e-3, 0.02, 7.5):  # the last saturates scales at 448 for the outliers
        g_t = torch.tensor([g], dtype=torch.float32, device=DEV)
        codes, sf, _ = ops.quantize_act(X.to(DEV), g_a=g_t, static_scale=True)
        c_ref, s_ref = oracle.quantize(xb, np.float32(g))
        assert np.array_equal(host(codes), c_ref)
        assert np.array_equal(host(sf), oracle.swizzle(s_ref, 512))


def test_weights_per_segment_bit_exact():
    lin = wl.gdn_inproj_linear()
    small = [(m.width // 16 if m.width > 48 else m.width) for m in lin.modules]
    segs = wl.segments_from_widths(small)
    parts = [wl.weight_normal(w, 256, m.sigma, 90 + i) for i, (w, m) in enumerate(zip(small, lin.modules))]
    W = torch.cat(parts, 0)
    qw = ops.quantize_weights(W.to(DEV), segs)
    torch.cuda.synchronize()
    c_ref, s_ref, g_ref = oracle.quantize_segments(wl.bf16_bits(W), segs)
    assert np.array_equal(host(qw.g_w), g_ref)
    assert np.array_equal(host(qw.codes), c_ref)
    assert np.array_equal(host(qw.sf), oracle.swizzle(s_ref, 256))


@pytest.mark.parametrize("M,K", [(128, 64), (1024, 512)])  # every CTA takes max|x| / a separate amax pass
def test_nonfinite_input_is_reported(M, K):
    x = np.ones((M, K), dtype=np.float32)
    x[5, 7] = np.inf
    ops.quantize_act(wl.to_bf16(x).to(DEV))
    assert ops.get_status() == 6
    assert ops.get_status() == 0  # cleared
    ops.quantize_act(torch.ones((M, K), dtype=torch.bfloat16, device=DEV))
    assert ops.get_status() == 0


def test_empty_rows():
    codes, sf, g = ops.quantize_act(torch.empty((0, 64), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert float(host(g)[0]) == 1.0
    assert codes.numel() == 0
