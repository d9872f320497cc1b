"""Gated MLP up projection with the SwiGLU in the GEMM epilogue
(nvfp4_quantize_weights_gated + nvfp4_linear_swiglu) against the oracle:
the interleaved weight layout and the quantized operands bit for bit, h
within the GEMM tolerance carried through silu(g)*u plus bf16 rounding, and
the requantization of the GPU's own h bit for bit; no byte around h, its
codes, scales or the workspace may change."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import DEV, Guarded, host

pytestmark = pytest.mark.gpu


def _gate_up(F, K, seed, sig=(0.02, 0.03)):
    gate = wl.weight_normal(F, K, sig[0], seed)
    up = wl.weight_normal(F, K, sig[1], seed + 1)
    return torch.cat([gate, up], 0)


def test_gated_weight_layout_bit_exact():
    F, K = 384, 320
    W = _gate_up(F, K, 50)
    qw = ops.quantize_weights_gated(W.to(DEV))
    torch.cuda.synchronize()
    segs = [(0, F), (F, 2 * F)]
    c_ref, s_ref, g_ref = oracle.quantize_segments(wl.bf16_bits(W), segs)
    assert np.array_equal(host(qw.g_w), g_ref)
    assert np.array_equal(host(qw.codes), oracle.interleave_gate_up(c_ref, F))
    assert np.array_equal(host(qw.sf), oracle.swizzle(oracle.interleave_gate_up(s_ref, F), K))


def _h_tolerance(Cg, Bg, Cu, Bu, h_ref):
    """GEMM tolerance on gate and up carried through h = silu(g) u (|silu'| <=
    1.1), plus fp32 evaluation error and half a bf16 ulp of the result."""
    tg = oracle.gemm_tolerance(Bg)
    tu = oracle.gemm_tolerance(Bu)
    s = np.abs(oracle.silu_mul(Cg, np.ones_like(Cg)))
    a = np.maximum(np.abs(h_ref), 1e-38)
    ulp = np.exp2(np.floor(np.log2(a)) - 7)
    return 1.1 * tg * (np.abs(Cu) + tu) + s * tu + 1e-6 * np.abs(h_ref) + 0.5 * ulp * (1 + 1e-6) + 1e-30


def _check(M, K, F, X, W, rows, cols, single_cta=False):
    qw = ops.quantize_weights_gated(W.to(DEV))
    gh_ = Guarded((M, F), torch.bfloat16, fill=float("nan"))
    gc_ = Guarded(M * F // 2, torch.uint8, fill=0x5A)
    gs_ = Guarded(ops.sf_bytes(M, F), torch.uint8, fill=0x5A)
    gw_ = Guarded(ops.workspace_bytes(M, 2 * F, K, 2), torch.uint8)
    h, hc, hsf, gh = ops.linear_swiglu(X.to(DEV), qw, h=gh_.t, h_codes=gc_.t, h_sf=gs_.t, ws=gw_.t,
                                       single_cta=single_cta)
    for g, what in ((gh_, "h"), (gc_, "h codes"), (gs_, "h scale factors"), (gw_, "workspace")):
        g.check(what)
    assert ops.get_status() == 0
    xb, wb = wl.bf16_bits(X), wl.bf16_bits(W)
    g_a = oracle.global_scale(oracle.amax(xb))
    gseg = oracle.segment_scales(wb, [(0, F), (F, 2 * F)])
    ac, asc = oracle.quantize(np.ascontiguousarray(xb[rows]), g_a)
    gc, gsc = oracle.quantize(np.ascontiguousarray(wb[cols]), gseg[0])
    uc, usc = oracle.quantize(np.ascontiguousarray(wb[F + cols]), gseg[1])
    im, inn = np.meshgrid(np.arange(len(rows)), np.arange(len(cols)), indexing="ij")
    Cg, Bg = oracle.linear_sampled(ac, asc, g_a, gc, gsc, gseg[0], im.ravel(), inn.ravel())
    Cu, Bu = oracle.linear_sampled(ac, asc, g_a, uc, usc, gseg[1], im.ravel(), inn.ravel())
    h_ref = oracle.silu_mul(Cg, Cu)
    h_bits = host(h.view(torch.int16)).view(np.uint16)
    got = oracle.bf16_bits_to_f32(h_bits[rows][:, cols].ravel()).astype(np.float64)
    tol = _h_tolerance(Cg, Bg, Cu, Bu, h_ref)
    bad = np.abs(got - h_ref) > tol
    assert not np.any(bad), f"{int(bad.sum())} h values outside tolerance, e.g. {got[bad][:3]} vs {h_ref[bad][:3]}"
    # h requantized with its own dynamic scale: the oracle on the GPU's h
    g_ref = oracle.global_scale(oracle.amax(h_bits))
    assert float(host(gh)[0]) == g_ref
    c_ref, s_ref = oracle.quantize(np.ascontiguousarray(h_bits[rows]), np.float32(g_ref))
    assert np.array_equal(host(hc)[rows], c_ref)
    assert np.array_equal(oracle.unswizzle(host(hsf), M, F)[rows], s_ref)


@pytest.mark.parametrize("single_cta", [False, True])
@pytest.mark.parametrize("M,K,F", [(200, 512, 384), (300, 768, 640), (1, 512, 384), (77, 256, 256)])
def test_linear_swiglu_small_full_check(M, K, F, single_cta):
    """Every h value: M > 128 runs the CTA-pair kernel unless single_cta;
    decode-sized M (one partial 128-row block) the single-CTA gated kernel."""
    X = wl.activation_normal(M, K, 51 + M)
    W = _gate_up(F, K, 52 + F)
    _check(M, K, F, X, W, np.arange(M), np.arange(F), single_cta)


def test_linear_swiglu_prefill_mlp_full_size():
    """gate/up of the prefill MLP, M=8192, K=5120, F=17408, on sampled rows
    and columns (every column of the last h tile included)."""
    M, K, F = 8192, 5120, 17408
    X = wl.activation_normal(M, K, 2)
    W = _gate_up(F, K, 53, (0.02, 0.02))
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([rng.integers(0, M, 24), [0, M - 1]]))
    cols = np.unique(np.concatenate([rng.integers(0, F, 96), np.arange(F - 130, F)]))
    _check(M, K, F, X, W, rows, cols)


def test_split_calls_equal_linear_swiglu():
    """nvfp4_quantize_act + nvfp4_gemm_prequant_swiglu + nvfp4_quantize_act
    (NVFP4_AMAX_GIVEN) is nvfp4_linear_swiglu, bit for bit."""
    M, K, F = 130, 256, 256
    X = wl.activation_normal(M, K, 60).to(DEV)
    qw = ops.quantize_weights_gated(_gate_up(F, K, 61).to(DEV))
    h1, c1, s1, g1 = ops.linear_swiglu(X, qw)
    ac, asf, ga = ops.quantize_act(X)
    h2, ws = ops.gemm_prequant_swiglu(ac, asf, ga, M, K, qw)
    c2, s2, g2 = ops.quantize_act(h2, ws=ws, amax_given=True)
    assert ops.get_status() == 0
    assert torch.equal(h1, h2) and torch.equal(g1, g2)
    assert torch.equal(c1, c2) and torch.equal(s1[: ops.sf_bytes(M, F)], s2[: ops.sf_bytes(M, F)])
