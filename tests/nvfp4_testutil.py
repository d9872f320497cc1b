"""Helpers shared by the GPU parity tests: move oracle outputs to the device,
sample outputs, and apply the GEMM tolerance."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl

DEV = "cuda"

GUARD_BYTES = 4096
SENTINEL = 0xA5


class Guarded:
    """A device buffer with GUARD_BYTES of sentinel bytes on each side: the
    bounds check that stands in for a memory sanitizer.  `t` is the buffer a
    call may write (16-byte aligned, contiguous); check() asserts that no
    byte around it changed."""

    def __init__(self, shape, dtype, fill=None, device=DEV):
        shape = tuple(shape) if isinstance(shape, (tuple, list)) else (int(shape),)
        n = 1
        for d in shape:
            n *= int(d)
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((2 * GUARD_BYTES + nbytes,), SENTINEL, dtype=torch.uint8, device=device)
        self.t = self.raw[GUARD_BYTES: GUARD_BYTES + nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what: str = ""):
        if self.raw.is_cuda:
            torch.cuda.synchronize()
        head = self.raw[:GUARD_BYTES]
        tail = self.raw[self.raw.numel() - GUARD_BYTES:]
        bad_head = int((head != SENTINEL).sum())
        bad_tail = int((tail != SENTINEL).sum())
        assert bad_head == 0 and bad_tail == 0, (
            f"{what}: {bad_head} bytes before and {bad_tail} bytes after the buffer were written")
        return self.t


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


def check_gemm_bf16(out_bits: np.ndarray, C: np.ndarray, B: np.ndarray, what: str = "") -> float:
    """bf16 outputs: the fp32 tolerance plus half a bf16 ulp of the output."""
    v = oracle.bf16_bits_to_f32(out_bits).astype(np.float64)
    a = np.maximum(np.abs(v), 1e-38)
    ulp = np.exp2(np.floor(np.log2(a)) - 7)
    tol = oracle.gemm_tolerance(B) + 0.5 * ulp
    err = np.abs(v - C)
    bad = err > tol
    assert not np.any(bad), f"{what}: {int(bad.sum())} outside tolerance, e.g. gpu={v[bad][:3]} oracle={C[bad][:3]}"
    return float(np.max(err / tol)) if err.size else 0.0


def oracle_sampled(xb, wb, segments, ms, ns):
    """Oracle outputs at the sampled (m, n) pairs: the tensor-wide global
    scales come from the whole operands, the codes and block scales only
    from the rows the samples use."""
    g_a = oracle.global_scale(oracle.amax(xb))
    gseg = oracle.segment_scales(wb, segments)
    grow = oracle.rows_scale(segments, gseg, wb.shape[0])
    um, im = np.unique(ms, return_inverse=True)
    un, inn = np.unique(ns, return_inverse=True)
    ac, asc = oracle.quantize(np.ascontiguousarray(xb[um]), g_a)
    wc, wsc = oracle.quantize(np.ascontiguousarray(wb[un]), grow[un])
    C, B = oracle.linear_sampled(ac, asc, g_a, wc, wsc, grow[un], im, inn)
    return C, B, (um, ac, asc, np.float32(g_a)), (un, wc, wsc, gseg)


def full_size_check(X, W, segments, seed):
    """nvfp4_linear_fused at full size (bf16 and fp32 outputs) against the
    oracle on sampled outputs; the quantized operands of the sampled rows
    are checked bit for bit and the bytes around the outputs and the
    workspace must be untouched.  Returns the largest error / tolerance
    ratio."""
    M, K = X.shape
    N = W.shape[0]
    xb, wb = wl.bf16_bits(X), wl.bf16_bits(W)
    qw = ops.quantize_weights(W.to(DEV), segments)
    Xd = X.to(DEV)
    gws = Guarded(ops.workspace_bytes(M, N, K, len(segments)), torch.uint8)
    ws = gws.t
    g16 = Guarded((M, N), torch.bfloat16)
    g32 = Guarded((M, N), torch.float32)
    ops.linear_fused(Xd, qw, out=g16.t, ws=ws)
    ops.linear_fused(Xd, qw, out=g32.t, ws=ws, out_fp32=True)
    out, out32 = g16.check("bf16 output"), g32.check("fp32 output")
    gws.check("workspace")
    assert ops.get_status() == 0
    rng = np.random.default_rng(seed)
    ms, ns = sample_outputs(M, N, segments, rng)
    C, B, (um, ac, asc, ga), (un, wc, wsc, gseg) = oracle_sampled(xb, wb, segments, ms, ns)
    # quantized operands of the sampled rows are the oracle's, bit for bit
    g_ws, c_ws, sf_ws = ops.linear_workspace_views(ws, M, K)
    assert float(host(g_ws)[0]) == float(ga)
    assert np.array_equal(host(qw.g_w), gseg)
    assert np.array_equal(host(c_ws)[um], ac)
    assert np.array_equal(oracle.unswizzle(host(sf_ws), M, K)[um], asc)
    assert np.array_equal(host(qw.codes)[un], wc)
    sf_w = host(qw.sf)
    assert np.array_equal(oracle.unswizzle(sf_w, N, K)[un], wsc)
    o32 = host(out32)[ms, ns]
    r32 = check_gemm(o32, C, B, "fp32 sampled")
    o16 = host(out.view(torch.int16)).view(np.uint16)[ms, ns]
    check_gemm_bf16(o16, C, B, "bf16 sampled")
    assert np.array_equal(o16, bf16_of_f32(o32))
    return r32
