"""Helpers shared by the GPU parity tests: move oracle outputs to the device,
sample outputs, and apply the GEMM tolerance."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl

DEV = "cuda"


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).reshape(-1).view(np.uint8)).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def oracle_weight_on_device(w_bits: np.ndarray, segments) -> tuple[ops.QuantizedWeight, tuple]:
    """Quantize a fused weight with the oracle and upload codes, swizzled
    scales and per-segment scales as a QuantizedWeight."""
    N, K = w_bits.shape
    codes, scales, gseg = oracle.quantize_segments(w_bits, segments)
    qw = ops.QuantizedWeight(dev_u8(codes).view(N, K // 2), dev_u8(oracle.swizzle(scales, K)),
                             torch.from_numpy(gseg.copy()).to(DEV), list(segments), N, K)
    return qw, (codes, scales, gseg)


def oracle_act_on_device(x_bits: np.ndarray):
    M, K = x_bits.shape
    codes, scales, g = oracle.quantize_tensor(x_bits)
    return (dev_u8(codes).view(M, K // 2), dev_u8(oracle.swizzle(scales, K)),
            torch.tensor([g], dtype=torch.float32, device=DEV)), (codes, scales, g)


def check_gemm(out: np.ndarray, C: np.ndarray, B: np.ndarray, what: str = "") -> float:
    """|gpu - oracle| <= 1e-5 * sum|a*b| + 1e-6 per element; returns the
    largest error / tolerance ratio."""
    out = out.astype(np.float64)
    tol = oracle.gemm_tolerance(B)
    err = np.abs(out - C)
    ratio = float(np.max(err / tol)) if err.size else 0.0
    bad = err > tol
    if np.any(bad):
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"gpu={out[tuple(i)]!r} oracle={C[tuple(i)]!r} tol={tol[tuple(i)]!r}")
    return ratio


def bf16_of_f32(a: np.ndarray) -> np.ndarray:
    """bf16 bits of fp32 values, round to nearest even (torch CPU)."""
    return wl.bf16_bits(torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16))


def sample_outputs(M: int, N: int, segments, rng: np.random.Generator, n_random: int = 4096,
                   n_rows_edges: int = 64):
    """Random (m, n) pairs plus, for a few rows, every N-tail column (the
    ragged last 192-column tile), both columns around every segment boundary
    and the last rows."""
    ms = list(rng.integers(0, M, n_random))
    ns = list(rng.integers(0, N, n_random))
    edge_cols = set(range(max(0, N - 200), N)) | set(range(0, min(N, 8)))
    for a, b in segments:
        for c in (a - 1, a, a + 1, b - 2, b - 1):
            if 0 <= c < N:
                edge_cols.add(c)
    rows = list(rng.integers(0, M, n_rows_edges)) + [M - 1, max(0, M - 128)]
    for r in rows:
        for c in sorted(edge_cols):
            ms.append(r)
            ns.append(c)
    return np.array(ms, dtype=np.int64), np.array(ns, dtype=np.int64)
