"""Seeded random shapes against the oracle.

nvfp4_linear_fused: M from one row to more than two CTA-pair tiles (split-K
with per-row and with staged partials, the single-CTA and the CTA-pair
GEMM), ragged N, K of one to forty 64-wide steps, one to four module
segments of random widths.  Each case runs the bf16 and the fp32 output,
checks the activation's codes, scales and global scale and the weight's bit
for bit, compares sampled outputs (with every tail and segment-boundary
column of a few rows) with the oracle at 1e-5 sum|a*b| + 1e-6, and checks
that no byte around the outputs and the workspace was written.

Decode sizes with split-K: M up to 128 with K of 1536 to 17408, so that the
split count is 3-8 for most cases, per-row partials below 64 rows and
staged ones above; every row against the oracle, bf16 = RNE(fp32), run to
run and pre-quantized forms bit-identical (the decode suite's checker).

nvfp4_linear_swiglu: random M, K and F (a multiple of 128) through both
gated kernels, h against silu(gate) up of the oracle's GEMM and h's codes,
scales and global scale bit for bit.  nvfp4_quantize_act: random rows and K
(a multiple of 16), codes, scales (padding included) and global scale bit
for bit."""
import numpy as np
import pytest

from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import full_size_check
from test_decode_gpu import test_decode_linear_matches_oracle as decode_check
from test_quant_gpu import _assert_same
from test_swiglu_fused_gpu import _check as _check_swiglu, _gate_up

pytestmark = pytest.mark.gpu


def _cases(n=24, seed=2026):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        # rows: a third decode-sized, a third around the 64-row staged split-K
        # threshold and the 128-row single-CTA limit, a third CTA-pair sized
        band = i % 3
        if band == 0:
            M = int(rng.integers(1, 40))
        elif band == 1:
            M = int(rng.integers(56, 140))
        else:
            M = int(rng.integers(129, 600))
        K = 64 * int(rng.integers(1, 41))
        N = int(rng.integers(2, 3000))
        nseg = int(min(N, rng.integers(1, 5)))
        cuts = np.sort(rng.choice(np.arange(1, N), size=nseg - 1, replace=False)) if nseg > 1 else []
        edges = [0, *[int(c) for c in cuts], N]
        widths = [b - a for a, b in zip(edges[:-1], edges[1:])]
        out.append((M, N, K, widths, 100 + i))
    return out


@pytest.mark.parametrize("M,N,K,widths,seed", _cases())
def test_random_shape_linear_fused(M, N, K, widths, seed):
    X = wl.activation_normal(M, K, seed, n_outliers=min(4, K // 16))
    sig = [0.005 * (1.0 + 3.0 * ((seed * 7 + j) % 4)) for j in range(len(widths))]
    W = np.concatenate([wl.weight_normal(w, K, s, seed * 10 + j).float().numpy() for j, (w, s) in
                        enumerate(zip(widths, sig))], 0)
    ratio = full_size_check(X, wl.to_bf16(W), wl.segments_from_widths(widths), seed)
    assert ratio <= 1.0


def _gated_cases(n=8, seed=77):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        M = int(rng.integers(1, 128)) if i % 2 == 0 else int(rng.integers(129, 420))
        K = 64 * int(rng.integers(1, 25))
        F = 128 * int(rng.integers(1, 9))
        out.append((M, K, F, bool(i % 4 == 1), 300 + i))
    return out


@pytest.mark.parametrize("M,K,F,single_cta,seed", _gated_cases())
def test_random_shape_linear_swiglu(M, K, F, single_cta, seed):
    X = wl.activation_normal(M, K, seed, n_outliers=min(4, K // 16))
    W = _gate_up(F, K, seed + 1)
    _check_swiglu(M, K, F, X, W, np.arange(M), np.arange(F), single_cta)


def _quant_cases(n=12, seed=91):
    rng = np.random.default_rng(seed)
    return [(int(rng.integers(1, 700)), 16 * int(rng.integers(1, 200)), 500 + i) for i in range(n)]


@pytest.mark.parametrize("M,K,seed", _quant_cases())
def test_random_shape_quantize_act(M, K, seed):
    _assert_same(wl.activation_normal(M, K, seed, n_outliers=min(4, K // 16), scale=30.0))


def _decode_cases(n=16, seed=4242):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        M = int(rng.integers(1, 64)) if i % 2 == 0 else int(rng.integers(64, 129))
        K = 64 * int(rng.integers(24, 273))
        N = int(rng.integers(64, 6000))
        nseg = int(rng.integers(1, 4))
        cuts = np.sort(rng.choice(np.arange(1, N), size=nseg - 1, replace=False)) if nseg > 1 else []
        edges = [0, *[int(c) for c in cuts], N]
        widths = [b - a for a, b in zip(edges[:-1], edges[1:])] if nseg > 1 else None
        out.append((M, N, K, widths))
    return out


@pytest.mark.parametrize("M,N,K,widths", _decode_cases())
def test_random_shape_decode_split_k(M, N, K, widths):
    decode_check(M, N, K, widths)
