"""The binding's argument checks (no GPU).

The C library receives only addresses, so the binding checks every buffer a
kernel will access: dtype, contiguity, and size against what the call
writes.  Here the library's compute entry points are replaced by a recorder
(its size queries still come from the real library), and the device checks
are lifted so that CPU tensors stand in for device ones.  Valid calls, in the
forms the benchmark and the GPU tests use, must reach the library; malformed
ones must raise ValueError before any library call.
"""
import pytest
import torch

from nvfp4_w4a4_quantized_act_b200 import ops

PURE = {"nvfp4_sf_bytes", "nvfp4_workspace_bytes", "nvfp4_quant_workspace_bytes", "nvfp4_gemm_workspace_bytes",
        "nvfp4_linear_act_scale_offset"}


class _Recorder:
    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in PURE:
            return getattr(self.real, name)
        if not name.startswith("nvfp4_"):
            raise AttributeError(name)

        def call(*args):
            self.calls.append(name)
            return 0
        return call


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder(ops.lib())
    monkeypatch.setattr(ops, "lib", lambda: r)
    monkeypatch.setattr(ops, "_require_cuda", lambda *ts: None)
    monkeypatch.setattr(ops, "_stream", lambda stream=None: None)
    return r


bf16, f32, u8 = torch.bfloat16, torch.float32, torch.uint8


def _u8(n):
    return torch.zeros(max(int(n), 1), dtype=u8)


def _weight(N, K, segments=None, gated=False):
    segments = segments or [(0, N)]
    return ops.QuantizedWeight(_u8(N * K // 2).view(N, K // 2), _u8(ops.sf_bytes(N, K)),
                               torch.ones(len(segments), dtype=f32), segments, N, K, gated)


def test_valid_calls_reach_the_library(rec):
    M, K, N, F = 16, 512, 384, 256
    X = torch.zeros((M, K), dtype=bf16)
    qw = _weight(N, K, [(0, 128), (128, N)])
    qg = _weight(2 * F, K, [(0, F), (F, 2 * F)], gated=True)
    # shared buffers sized for the largest K, as the benchmark's stack does
    maxK = 2 * K
    codes, sf = _u8(M * maxK // 2), _u8(ops.sf_bytes(M, maxK))
    g = torch.zeros(1, dtype=f32)
    qws = _u8(ops.quant_workspace_bytes(1))
    ws = _u8(ops.workspace_bytes(M, 2 * F, maxK, 2))

    ac, asf, ga = ops.quantize_act(X)
    assert ac.shape == (M, K // 2)
    ac2, asf2, _ = ops.quantize_act(X, g_a=g, codes=codes, sf=sf, ws=qws)
    assert ac2.shape == (M, K // 2) and ac2.data_ptr() == codes.data_ptr()
    ops.quantize_act(X, g_a=g, static_scale=True)
    ops.gemm_prequant(ac, asf, ga, M, K, qw)
    ops.gemm_prequant(ac, asf, ga, M, K, qw, out=torch.zeros((M, N), dtype=bf16))
    ops.gemm_prequant(ac, asf, ga, M, K, qw, out=torch.zeros((M, N), dtype=f32), out_fp32=True)
    ops.gemm_prequant(ac, asf, ga, M, K, qw, out_fp32=True, ws=_u8(ops.gemm_workspace_bytes(M, N, K)))
    ops.gemm_prequant(torch.zeros((1, 32), dtype=u8), _u8(512), g, 0, 64, _weight(64, 64))      # M = 0
    ops.linear_fused(X, qw, out=torch.zeros((M, N), dtype=bf16), ws=ws)
    ops.linear(X, _weight(N, K), out=torch.zeros((M, N), dtype=bf16), ws=ws)
    ops.linear_fused_noalloc(X, qw)
    h = torch.zeros((M, F), dtype=bf16)
    _, hc, _, _ = ops.linear_swiglu(X, qg, h=h, h_codes=codes, h_sf=sf, g_h=g, ws=ws)
    assert hc.shape == (M, F // 2)
    ops.gemm_prequant_swiglu(ac, asf, ga, M, K, qg, h=h, ws=qws)
    ops.swiglu_quantize(torch.zeros((M, 2 * F), dtype=bf16))
    g_ws, c_ws, sf_ws = ops.linear_workspace_views(ws, M, K)
    ops.gemm_prequant(c_ws, sf_ws, g_ws, M, K, qw, out_fp32=True)
    kv = torch.zeros((53, 200), dtype=bf16)[:, 24:152]
    s = ops.fp8_kv_calibrate(kv)
    ops.fp8_kv_quantize(kv, s, out=torch.zeros((53, 160), dtype=u8)[:, :128])
    assert rec.calls == ["nvfp4_quantize_act"] * 3 + ["nvfp4_gemm_prequant"] * 3 + ["nvfp4_gemm_prequant_ws"] + \
        ["nvfp4_gemm_prequant", "nvfp4_linear_fused", "nvfp4_linear", "nvfp4_linear_fused_noalloc",
         "nvfp4_linear_swiglu", "nvfp4_gemm_prequant_swiglu", "nvfp4_swiglu_quantize", "nvfp4_gemm_prequant",
         "nvfp4_fp8_kv_calibrate", "nvfp4_fp8_kv_quantize"]


def _bad_calls():
    M, K, N, F = 16, 512, 384, 256
    X = torch.zeros((M, K), dtype=bf16)
    qw = _weight(N, K)
    qg = _weight(2 * F, K, [(0, F), (F, 2 * F)], gated=True)
    ac, asf, ga = _u8(M * K // 2).view(M, K // 2), _u8(ops.sf_bytes(M, K)), torch.ones(1, dtype=f32)
    h = torch.zeros((M, F), dtype=bf16)
    return {
        "fp32 input": lambda: ops.quantize_act(X.float()),
        "1-D input": lambda: ops.quantize_act(X.view(-1)),
        "column stride": lambda: ops.quantize_act(X.t()),
        "static scale without g_a": lambda: ops.quantize_act(X, static_scale=True),
        "codes too small": lambda: ops.quantize_act(X, codes=_u8(M * K // 2 - 1)),
        "sf too small": lambda: ops.quantize_act(X, sf=_u8(ops.sf_bytes(M, K) - 1)),
        "g_a fp64": lambda: ops.quantize_act(X, g_a=torch.zeros(1, dtype=torch.float64)),
        "bf16 out for fp32": lambda: ops.gemm_prequant(ac, asf, ga, M, K, qw, out=torch.zeros((M, N), dtype=bf16),
                                                       out_fp32=True),
        "out too small": lambda: ops.gemm_prequant(ac, asf, ga, M, K, qw, out=torch.zeros((M, N - 1), dtype=bf16)),
        "out strided": lambda: ops.linear_fused(X, qw, out=torch.zeros((M, 2 * N), dtype=bf16)[:, :N]),
        "K mismatch": lambda: ops.gemm_prequant(ac, asf, ga, M, K, _weight(N, 2 * K)),
        "a_codes too small": lambda: ops.gemm_prequant(ac[:-1], asf, ga, M, K, qw),
        "a_sf too small": lambda: ops.gemm_prequant(ac, asf[:-1], ga, M, K, qw),
        "input not contiguous": lambda: ops.linear_fused(torch.zeros((M, 2 * K), dtype=bf16)[:, :K], qw),
        "ws strided": lambda: ops.linear_fused(X, qw, ws=_u8(1 << 22)[::2]),
        "linear K mismatch": lambda: ops.linear(X, _weight(N, 2 * K)),
        "noalloc out dtype": lambda: ops.linear_fused_noalloc(X, qw, out=torch.zeros((M, N), dtype=f32)),
        "swiglu on plain weight": lambda: ops.linear_swiglu(X, qw),
        "h too small": lambda: ops.linear_swiglu(X, qg, h=torch.zeros((M, F - 1), dtype=bf16)),
        "h fp32": lambda: ops.gemm_prequant_swiglu(ac, asf, ga, M, K, qg, h=h.float()),
        "h_codes too small": lambda: ops.linear_swiglu(X, qg, h_codes=_u8(M * F // 2 - 1)),
        "gated weight with odd rows": lambda: ops.quantize_weights_gated(torch.zeros((3, K), dtype=bf16)),
        "odd gate_up": lambda: ops.swiglu_quantize(torch.zeros((M, 2 * F + 1), dtype=bf16)),
        "kv out too small": lambda: ops.fp8_kv_quantize(X, ga, out=torch.zeros((M - 1, K), dtype=u8)),
        "kv out dtype": lambda: ops.fp8_kv_quantize(X, ga, out=torch.zeros((M, K), dtype=torch.int16)),
        "kv scale fp64": lambda: ops.fp8_kv_quantize(X, torch.ones(1, dtype=torch.float64)),
        "kv calibrate scale dtype": lambda: ops.fp8_kv_calibrate(X, scale=torch.zeros(1, dtype=bf16)),
    }


@pytest.mark.parametrize("case", sorted(_bad_calls()))
def test_malformed_buffers_raise_before_the_library(rec, case):
    with pytest.raises(ValueError):
        _bad_calls()[case]()
    assert rec.calls == []
