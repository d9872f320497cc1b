"""End-to-end NVFP4 W4A4 linear layers (on-the-fly activation quantization +
block-scaled GEMM + per-module global-scale epilogue) against the oracle, at
small sizes in full and at the full prefill sizes on sampled outputs."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import DEV, Guarded, bf16_of_f32, check_gemm, full_size_check, host

pytestmark = pytest.mark.gpu


def test_linear_tiny_end_to_end():
    X, W = wl.tiny_linear(0)
    xb, wb = wl.bf16_bits(X), wl.bf16_bits(W)
    qw = ops.quantize_weights(W.to(DEV))
    M, K = X.shape
    ws = torch.empty(ops.workspace_bytes(M, 128, K), dtype=torch.uint8, device=DEV)
    out32 = ops.linear(X.to(DEV), qw, out_fp32=True, ws=ws)
    torch.cuda.synchronize()
    ca, sa, ga = oracle.quantize_tensor(xb)
    cw, sw, gw = oracle.quantize_tensor(wb)
    g_ws, c_ws, sf_ws = ops.linear_workspace_views(ws, M, K)
    assert float(host(g_ws)[0]) == float(ga)
    assert np.array_equal(host(c_ws), ca)
    assert np.array_equal(host(sf_ws), oracle.swizzle(sa, K))
    C, B = oracle.linear_full(ca, sa, ga, cw, sw, gw)
    check_gemm(host(out32), C, B, "tiny linear")
    out16 = ops.linear(X.to(DEV), qw)
    assert np.array_equal(host(out16.view(torch.int16)).view(np.uint16), bf16_of_f32(host(out32)))


def _small_fused():
    widths = [64, 64, 192, 192, 48, 48]
    sig = wl.gdn_inproj_sigmas()
    segs = wl.segments_from_widths(widths)
    parts = [wl.weight_normal(w, 512, s, 40 + i) for i, (w, s) in enumerate(zip(widths, sig))]
    return torch.cat(parts, 0), segs, parts


def test_fused_matches_oracle_and_concat_of_modules():
    W, segs, parts = _small_fused()
    M, K = 300, 512
    X = wl.activation_normal(M, K, 8)
    qw = ops.quantize_weights(W.to(DEV), segs)
    gout = Guarded((M, W.shape[0]), torch.float32, fill=float("nan"))
    fused = ops.linear_fused(X.to(DEV), qw, out=gout.t, out_fp32=True)
    gout.check("fused output")
    ca, sa, ga = oracle.quantize_tensor(wl.bf16_bits(X))
    cw, sw, gseg = oracle.quantize_segments(wl.bf16_bits(W), segs)
    C, B = oracle.linear_full(ca, sa, ga, cw, sw, oracle.rows_scale(segs, gseg, W.shape[0]))
    check_gemm(host(fused), C, B, "fused")
    # the fused GEMM equals running every module as its own linear, bit for bit
    for (a, b), p in zip(segs, parts):
        qm = ops.quantize_weights(p.to(DEV))
        single = ops.linear(X.to(DEV), qm, out_fp32=True)
        assert np.array_equal(host(single), host(fused)[:, a:b])


def test_single_global_scale_mismatch_is_reproduced():
    """Serving a per-module-calibrated fused weight with one global scale
    (the first module's) scales module m by g_0 / g_m: the fault the
    per-segment epilogue repairs ("Why Gated DeltaNet Survives 4-Bit
    Quantization", kipquest.com, "The abstract" and "The deep dive").  The
    mismatched output is the oracle's GEMM of the same per-module codes and
    block scales with g_0 on every row, within the GEMM tolerance."""
    W, segs, _ = _small_fused()
    for M in (128, 300):  # split-K single-CTA kernel, CTA-pair kernel
        K = 512
        X = wl.activation_normal(M, K, 9)
        qw = ops.quantize_weights(W.to(DEV), segs)
        good = host(ops.linear_fused(X.to(DEV), qw, out_fp32=True))
        bad_w = ops.QuantizedWeight(qw.codes, qw.sf, qw.g_w[:1].clone(), [(0, qw.N)], qw.N, qw.K)
        bad = host(ops.linear_fused(X.to(DEV), bad_w, out_fp32=True))
        assert ops.get_status() == 0
        g = host(qw.g_w)
        assert len(set(g.tolist())) == len(segs)
        ca, sa, ga = oracle.quantize_tensor(wl.bf16_bits(X))
        cw, sw, gseg = oracle.quantize_segments(wl.bf16_bits(W), segs)
        assert np.array_equal(gseg, g)
        # against the oracle: the per-module codes and block scales, g_0 on every row
        C_bad, B = oracle.linear_full(ca, sa, ga, cw, sw, np.full(W.shape[0], gseg[0], dtype=np.float32))
        check_gemm(bad, C_bad, B, f"single-scale mismatch M={M}")
        C_good, B = oracle.linear_full(ca, sa, ga, cw, sw, oracle.rows_scale(segs, gseg, W.shape[0]))
        check_gemm(good, C_good, B, f"repaired M={M}")
        # and the factor itself: where K is split (small M) each partial is
        # scaled before the partials are added, so the identity holds to an
        # ulp of the partials' magnitude
        for (a, b), gm in zip(segs, g):
            ratio = np.float64(g[0]) / np.float64(gm)
            ref = good[:, a:b] * ratio
            np.testing.assert_allclose(bad[:, a:b], ref, rtol=2e-6, atol=2.0 ** -21 * np.max(np.abs(ref)))
        assert np.max(np.abs(g / g[0])) > 2 or np.min(np.abs(g / g[0])) < 0.5


def test_gdn_in_projection_full_size():
    """Fused GDN input projection: M=16384, K=5120, q/k/v/z/b/a = 2048, 2048,
    6144, 6144, 48, 48 rows, per-module sigma spread 10x."""
    lin = wl.gdn_inproj_linear()
    X = wl.activation_normal(16384, 5120, 3)
    W = wl.fused_weight(lin, 3)
    full_size_check(X, W, lin.segments, 31)


def test_mlp_gate_up_full_size():
    """Prefill MLP gate/up: M=8192, K=5120, N=2x17408 with a global scale per half."""
    gu, _ = wl.mlp_modules()
    X = wl.activation_normal(8192, 5120, 2)
    W = wl.fused_weight(gu, 2)
    full_size_check(X, W, gu.segments, 32)
