"""The seeded input recipes (no GPU): the shapes, counts and distributions
the benchmark and the parity tests rely on."""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_act_b200 import workloads as wl


def _bits(t):
    return wl.bf16_bits(t)


def test_inputs_are_seeded():
    a, b, c = (wl.activation_normal(16, 256, s) for s in (5, 5, 6))
    assert np.array_equal(_bits(a), _bits(b))
    assert not np.array_equal(_bits(a), _bits(c))
    t1, t2 = wl.activation_student_t(8, 512, 2), wl.activation_student_t(8, 512, 2)
    assert np.array_equal(_bits(t1), _bits(t2))
    w1, w2 = wl.weight_normal(32, 64, 0.02, 9), wl.weight_normal(32, 64, 0.02, 9)
    assert np.array_equal(_bits(w1), _bits(w2))


def test_outlier_columns_are_distinct_and_scaled():
    cols = wl.outlier_columns(5120, 51, 1)
    assert len(np.unique(cols)) == 51 and np.all(np.diff(cols) > 0) and cols.max() < 5120
    # N(0,1) activations: 4 columns x50
    x = wl.activation_normal(2048, 512, 3).float().numpy()
    std = x.std(axis=0)
    hot = np.sort(np.argsort(std)[-4:])
    assert np.array_equal(hot, wl.outlier_columns(512, 4, 3))
    assert np.all(np.abs(std[hot] / 50.0 - 1.0) < 0.1)
    assert np.all(np.abs(np.delete(std, hot) - 1.0) < 0.15)


def test_student_t_workload_has_one_percent_hot_channels():
    x = wl.activation_student_t(1024, 5120, 1).float().numpy()
    med = np.median(np.abs(x), axis=0)
    hot = wl.outlier_columns(5120, 51, 1)                        # floor(1% of 5120) = 51
    cold = np.delete(np.arange(5120), hot)
    ratio = np.median(med[hot]) / np.median(med[cold])
    assert 90.0 < ratio < 110.0                                  # channels x100
    assert x.dtype == np.float32


def test_gdn_module_scales_span_ten_times():
    sig = wl.gdn_inproj_sigmas()
    assert len(sig) == 6
    assert min(sig) == pytest.approx(0.005) and max(sig) == pytest.approx(0.05)
    assert all(0.005 - 1e-12 <= s <= 0.05 + 1e-12 for s in sig)
    lin = wl.gdn_inproj_linear()
    assert [m.width for m in lin.modules] == [2048, 2048, 6144, 6144, 48, 48]
    assert sum(m.width for m in lin.modules) == 16480 and lin.K == 5120


def test_stack_shapes_flops_and_weight_bytes():
    layers = wl.stack_layers()
    kinds = [k for k, _ in layers]
    assert len(layers) == 64 and kinds.count("gdn") == 48 and kinds.count("attention") == 16
    assert sum(len(lins) for _, lins in layers) == 256                 # fused GEMMs per step
    assert wl.count_stack_linears() == 496
    widths = {lin.name: (sum(m.width for m in lin.modules), lin.K) for _, lins in layers for lin in lins}
    assert widths == {"gdn_in_proj": (14432, 5120), "gdn_out": (5120, 6144), "gate_up": (34816, 5120),
                      "down": (5120, 17408), "attn_qkv": (14336, 5120), "attn_o": (5120, 6144)}
    tokens = 8192
    flops = sum(2.0 * tokens * sum(m.width for m in lin.modules) * lin.K for _, lins in layers for lin in lins)
    assert flops / 1e12 == pytest.approx(390.7, abs=0.05)

    def nvfp4_bytes(N, K):                                         # codes + scales in the 128 x 4 tile layout
        return N * K // 2 + (N + 127) // 128 * 128 * ((K // 16 + 3) // 4 * 4)

    wbytes = sum(nvfp4_bytes(sum(m.width for m in lin.modules), lin.K) for _, lins in layers for lin in lins)
    assert wbytes == 13_414_563_840


def test_bf16_conversion_rounds_to_nearest_even():
    # 1 + 2^-8 lies halfway between bf16 1.0 and 1 + 2^-7: ties to the even 1.0
    v = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], dtype=np.float32)
    assert _bits(wl.to_bf16(v)).tolist() == [0x3F80, 0x3F82]
    assert wl.to_bf16(v).dtype == torch.bfloat16
