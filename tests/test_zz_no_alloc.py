"""The allocation-free fused linear, nvfp4_linear_fused_noalloc.

It exists for callers that cannot allocate device memory where the layer
runs (a host runtime that owns all device memory and gives its operators no
allocator, or a serving loop that must not pay cudaMalloc's device-wide
synchronization).  Its scratch lives in a fixed device array inside the
library, so these tests check that:
  * two calls in a row through the C ABI agree with the oracle within the
    GEMM tolerance the other tests use, and with the workspace-taking
    nvfp4_linear_fused on the same inputs -- the second call uses a tensor
    with a much smaller amax, so a stale amax left in the shared scratch
    would show;
  * decode-sized inputs (M <= 128, the single-CTA kernel without split-K)
    agree with the oracle the same way, on a ragged N with several modules;
  * inputs larger than the array are refused before anything runs.
This file is collected last on purpose: a failure here stops an -x run only
after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _call_noalloc(X, qw, out, flags=0):
    arr, n = ops._segs(qw.segments)
    M, K = X.shape
    return ops.lib().nvfp4_linear_fused_noalloc(
        ctypes.c_void_p(X.data_ptr()), M, K, ctypes.c_void_p(qw.codes.data_ptr()),
        ctypes.c_void_p(qw.sf.data_ptr()), qw.N, arr, ctypes.c_void_p(qw.g_w.data_ptr()), n,
        ctypes.c_void_p(out.data_ptr()), flags, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _oracle_check(X, cw, sw, grow, got):
    ca, sa, ga = oracle.quantize_tensor(wl.bf16_bits(X))
    C, B = oracle.linear_full(ca, sa, ga, cw, sw, grow)
    err = np.abs(got.cpu().numpy().astype(np.float64) - C)
    assert np.all(err <= oracle.gemm_tolerance(B)), float(np.max(err / oracle.gemm_tolerance(B)))


def test_noalloc_matches_oracle_and_workspace_entry_point_twice():
    widths = [96, 160, 48]
    segs = wl.segments_from_widths(widths)
    K = 1024
    W = torch.cat([wl.weight_normal(w, K, s, 70 + i) for i, (w, s) in enumerate(zip(widths, [0.005, 0.05, 0.02]))])
    qw = ops.quantize_weights(W.to(DEV), segs)
    inputs = [wl.activation_normal(256, K, 71, n_outliers=4, scale=50.0),
              wl.activation_normal(130, K, 72, n_outliers=0)]  # much smaller amax on the second call
    cw, sw, gseg = oracle.quantize_segments(wl.bf16_bits(W), segs)
    grow = oracle.rows_scale(segs, gseg, W.shape[0])
    for X in inputs:
        Xd = X.to(DEV)
        M = X.shape[0]
        ref = ops.linear_fused(Xd, qw, out_fp32=True)
        got = torch.full((M, qw.N), float("nan"), dtype=torch.float32, device=DEV)
        rc = _call_noalloc(Xd, qw, got, ops.NVFP4_OUT_FP32)
        assert rc == 0, ops.status_string(rc)
        got16 = torch.empty((M, qw.N), dtype=torch.bfloat16, device=DEV)
        assert _call_noalloc(Xd, qw, got16) == 0
        ref16 = ops.linear_fused(Xd, qw)
        assert ops.get_status() == 0
        _oracle_check(X, cw, sw, grow, got)
        # both entry points run the same kernels on the same operands
        assert torch.equal(got, ref)
        assert torch.equal(got16, ref16)


def test_noalloc_decode_sizes_match_oracle():
    """M <= 128: the allocation-free call runs the single-CTA GEMM over the
    whole K (it has no room for split-K partials), so it is compared with the
    oracle, not bit for bit with nvfp4_linear_fused (which may split K)."""
    widths = [200, 72, 48, 17]  # N = 337: a ragged last tile
    segs = wl.segments_from_widths(widths)
    K = 2048
    W = torch.cat([wl.weight_normal(w, K, s, 80 + i)
                   for i, (w, s) in enumerate(zip(widths, [0.02, 0.005, 0.05, 0.01]))])
    qw = ops.quantize_weights(W.to(DEV), segs)
    cw, sw, gseg = oracle.quantize_segments(wl.bf16_bits(W), segs)
    grow = oracle.rows_scale(segs, gseg, W.shape[0])
    for M, seed in ((1, 81), (16, 82), (100, 83), (16, 84)):
        X = wl.activation_normal(M, K, seed, n_outliers=2 if seed % 2 else 0)
        got = torch.full((M, qw.N), float("nan"), dtype=torch.float32, device=DEV)
        rc = _call_noalloc(X.to(DEV), qw, got, ops.NVFP4_OUT_FP32)
        assert rc == 0, ops.status_string(rc)
        assert ops.get_status() == 0
        _oracle_check(X, cw, sw, grow, got)


def test_noalloc_rejects_oversize_and_static_scale():
    qw = ops.quantize_weights(wl.weight_normal(64, 4096, 0.02, 5).to(DEV))
    big = torch.zeros((2048, 4096), dtype=torch.bfloat16, device=DEV)  # M*K = 2^23 > 2^22
    out = torch.empty((2048, 64), dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(big, qw, out) == 7
    ok = torch.ones((16, 4096), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((16, 64), dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(ok, qw, out, ops.NVFP4_STATIC_SCALE) == 1
    assert _call_noalloc(ok, qw, out) == 0
    assert ops.get_status() == 0
