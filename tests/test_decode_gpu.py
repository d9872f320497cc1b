"""Decode-sized linears (M <= 128 tokens), where the GEMM divides each output
tile's K steps among several CTAs (split-K) and sums the fp32 partials in a
fixed order: every output against the oracle on all rows (all columns, or
sampled columns plus every module boundary for wide fused weights), bf16 =
RNE(fp32), run-to-run bit equality, the unsplit GEMM on the same quantized
activation within the same tolerance, and the launch that does the sum.  No
byte around the outputs and workspaces (where the split-K partials live) may
change."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import DEV, Guarded, bf16_of_f32, check_gemm, host

pytestmark = pytest.mark.gpu

# (M, N, K, module widths): single and fused modules, ragged M and N, K with a
# partial last stage (1344 = 21 blocks of 64) and the MLP down projection's K
CASES = [
    (1, 5120, 5120, None),
    (7, 1024, 5120, None),
    (16, 2112, 1344, [1024, 1024, 64]),
    (33, 1000, 5120, [600, 400]),
    (64, 16480, 5120, [2048, 2048, 6144, 6144, 48, 48]),
    (128, 1280, 17408, None),
    (100, 5120, 2048, [4096, 1024]),
    (3, 1002, 5120, [500, 502]),  # N % 4 != 0: scalar partial and output stores
    # from 64 rows the partials go through shared memory, a row per store:
    (64, 5120, 6144, None),       # 6 splits, two-column stores
    (100, 1001, 5120, [500, 501]),  # 7 splits, odd N (one-column stores), 4 rows in the last lane quarter
]


def _weight(N, K, widths, seed):
    widths = widths or [N]
    sig = [0.02 * (1.0 + 0.7 * i) for i in range(len(widths))]
    W = torch.cat([wl.weight_normal(w, K, s, seed + i) for i, (w, s) in enumerate(zip(widths, sig))], 0)
    return W, wl.segments_from_widths(widths)


def _columns(N, segs, rng, n_random=1536):
    if N <= 4096:
        return np.arange(N)
    edges = [c for a, b in segs for c in (a, a + 1, b - 2, b - 1) if 0 <= c < N]
    return np.unique(np.concatenate([rng.integers(0, N, n_random), edges]))


@pytest.mark.parametrize("M,N,K,widths", CASES)
def test_decode_linear_matches_oracle(M, N, K, widths):
    seed = M + N + K
    X = wl.activation_normal(M, K, seed)
    W, segs = _weight(N, K, widths, seed)
    xb, wb = wl.bf16_bits(X), wl.bf16_bits(W)
    qw = ops.quantize_weights(W.to(DEV), segs)
    Xd = X.to(DEV)
    gws = Guarded(ops.workspace_bytes(M, N, K, len(segs)), torch.uint8)
    ws = gws.t
    g32 = Guarded((M, N), torch.float32, fill=float("nan"))
    g16 = Guarded((M, N), torch.bfloat16, fill=float("nan"))
    ops.linear_fused(Xd, qw, out=g32.t, out_fp32=True, ws=ws)
    ops.linear_fused(Xd, qw, out=g16.t, ws=ws)
    out32 = host(g32.check("fp32 output"))
    out16 = host(g16.check("bf16 output").view(torch.int16)).view(np.uint16)
    gws.check("workspace (activation codes, scales, split-K partials)")
    again = host(ops.linear_fused(Xd, qw, out_fp32=True, ws=ws))
    assert ops.get_status() == 0

    cols = _columns(N, segs, np.random.default_rng(seed))
    ca, sa, ga = oracle.quantize_tensor(xb)
    gseg = oracle.segment_scales(wb, segs)
    grow = oracle.rows_scale(segs, gseg, N)[cols]
    cw, sw = oracle.quantize(np.ascontiguousarray(wb[cols]), grow)
    C, B = oracle.linear_full(ca, sa, ga, cw, sw, grow)
    check_gemm(out32[:, cols], C, B, f"split-K M={M} N={N} K={K}")
    assert np.array_equal(out16, bf16_of_f32(out32))
    assert np.array_equal(again, out32)

    # the unsplit GEMM over the same quantized activation agrees within the tolerance
    g_ws, c_ws, sf_ws = ops.linear_workspace_views(ws, M, K)
    plain = host(ops.gemm_prequant(c_ws, sf_ws, g_ws, M, K, qw, out_fp32=True))
    assert ops.get_status() == 0
    check_gemm(plain[:, cols], C, B, "unsplit")
    # the workspace form splits like the linear: the same bits on the same operands
    gpw = Guarded(max(ops.gemm_workspace_bytes(M, N, K), 16), torch.uint8)
    gpo = Guarded((M, N), torch.float32, fill=float("nan"))
    ops.gemm_prequant(c_ws, sf_ws, g_ws, M, K, qw, out=gpo.t, out_fp32=True, ws=gpw.t)
    pre = host(gpo.check("pre-quantized GEMM output"))
    gpw.check("split-K workspace")
    assert ops.get_status() == 0
    assert np.array_equal(pre, out32)


def test_split_sum_is_its_own_launch():
    """K = 5120 at N = 5120 splits K (one more launch adds the partials);
    K = 256 has one stage and cannot split.  Counted as the linear's launches
    minus those of quantizing the same input."""
    W, _ = _weight(5120, 5120, None, 1)
    qw = ops.quantize_weights(W.to(DEV))
    qs = ops.quantize_weights(W[:, :256].contiguous().to(DEV))

    def gemm_launches(M, K, q):
        X = wl.activation_normal(M, K, 1).to(DEV)
        ops.linear(X, q)
        ops.quantize_act(X)
        torch.cuda.synchronize()
        n0 = ops.launch_count()
        ops.linear(X, q)
        n1 = ops.launch_count()
        ops.quantize_act(X)
        return (n1 - n0) - (ops.launch_count() - n1)

    assert gemm_launches(16, 256, qs) == 1
    assert gemm_launches(1, 5120, qw) == 2
    assert gemm_launches(16, 5120, qw) == 2
    assert ops.get_status() == 0


def test_zero_activation_and_single_row():
    """An all-zero input gives exact zeros through the split sum; one row of
    an outlier-heavy input still matches."""
    K, N = 5120, 1024
    W, segs = _weight(N, K, [512, 512], 5)
    qw = ops.quantize_weights(W.to(DEV), segs)
    z = torch.zeros((3, K), dtype=torch.bfloat16, device=DEV)
    out = host(ops.linear_fused(z, qw, out_fp32=True))
    assert ops.get_status() == 0
    assert np.all(out == 0.0)
    X = wl.activation_normal(1, K, 6, n_outliers=16, scale=400.0)
    out1 = host(ops.linear_fused(X.to(DEV), qw, out_fp32=True))
    ca, sa, ga = oracle.quantize_tensor(wl.bf16_bits(X))
    cw, sw, gseg = oracle.quantize_segments(wl.bf16_bits(W), segs)
    C, B = oracle.linear_full(ca, sa, ga, cw, sw, oracle.rows_scale(segs, gseg, N))
    check_gemm(out1, C, B, "single row")
