"""ctypes binding of libnvfp4.so (declared in include/nvfp4.h).

Argument marshalling only: every step of the quantize / GEMM path runs in the
library's CUDA kernels.  torch supplies device memory (output and workspace
allocation) and the current CUDA stream.  There is no CPU fallback: if the
library is missing or the device is not an sm_100 GPU, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

NVFP4_STATIC_SCALE = 1
NVFP4_OUT_FP32 = 2
NVFP4_AMAX_GIVEN = 4
NVFP4_DEBUG_INJECT_STALL = 1 << 30
NVFP4_SINGLE_CTA = 1 << 29
MAX_SEGMENTS = 16

STATUS_NAMES = {
    0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_UNSUPPORTED_SHAPE", 3: "NVFP4_ERR_MISALIGNED",
    4: "NVFP4_ERR_CUDA", 5: "NVFP4_ERR_TIMEOUT", 6: "NVFP4_ERR_NONFINITE", 7: "NVFP4_ERR_WORKSPACE",
    8: "NVFP4_ERR_NO_DEVICE",
}

EXPORTED = [
    "nvfp4_sf_bytes", "nvfp4_quant_workspace_bytes", "nvfp4_workspace_bytes", "nvfp4_linear_act_scale_offset",
    "nvfp4_quantize_weights", "nvfp4_quantize_act", "nvfp4_gemm_prequant", "nvfp4_linear_fused",
    "nvfp4_gemm_workspace_bytes", "nvfp4_gemm_prequant_ws",
    "nvfp4_linear", "nvfp4_swiglu_quantize", "nvfp4_get_status", "nvfp4_status_string",
    "nvfp4_device_supported", "nvfp4_launch_count", "nvfp4_linear_fused_noalloc",
    "nvfp4_quantize_weights_gated", "nvfp4_linear_swiglu", "nvfp4_gemm_prequant_swiglu",
    "nvfp4_fp8_kv_calibrate", "nvfp4_fp8_kv_quantize",
]


class Nvfp4Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({status_string(code)})")


class Segment(ctypes.Structure):
    _fields_ = [("n_begin", ctypes.c_int64), ("n_end", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libnvfp4.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with nvfp4_w4a4_quantized_act_b200.build.build()")
    L = ctypes.CDLL(LIB_PATH)
    i64, sz, vp, u8p, fp = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    segp = ctypes.POINTER(Segment)
    sig = {
        "nvfp4_sf_bytes": (sz, [i64, i64]),
        "nvfp4_quant_workspace_bytes": (sz, [ctypes.c_int]),
        "nvfp4_workspace_bytes": (sz, [i64, i64, i64, ctypes.c_int]),
        "nvfp4_linear_act_scale_offset": (sz, []),
        "nvfp4_quantize_weights": (ctypes.c_int, [vp, i64, i64, i64, segp, ctypes.c_int, u8p, u8p, fp, vp, sz, vp]),
        "nvfp4_quantize_act": (ctypes.c_int, [vp, i64, i64, i64, u8p, u8p, fp, ctypes.c_uint, vp, sz, vp]),
        "nvfp4_gemm_workspace_bytes": (sz, [i64, i64, i64]),
        "nvfp4_gemm_prequant_ws": (ctypes.c_int, [u8p, u8p, fp, i64, i64, u8p, u8p, i64, segp, fp, ctypes.c_int,
                                                  vp, ctypes.c_uint, vp, sz, vp]),
        "nvfp4_gemm_prequant": (ctypes.c_int, [u8p, u8p, fp, i64, i64, u8p, u8p, i64, segp, fp, ctypes.c_int, vp,
                                               ctypes.c_uint, vp]),
        "nvfp4_linear_fused": (ctypes.c_int, [vp, i64, i64, u8p, u8p, i64, segp, fp, ctypes.c_int, vp,
                                              ctypes.c_uint, vp, sz, vp]),
        "nvfp4_linear": (ctypes.c_int, [vp, i64, i64, u8p, u8p, fp, i64, vp, ctypes.c_uint, vp, sz, vp]),
        "nvfp4_swiglu_quantize": (ctypes.c_int, [vp, i64, i64, i64, vp, u8p, u8p, fp, vp, sz, vp]),
        "nvfp4_get_status": (ctypes.c_int, [vp]),
        "nvfp4_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "nvfp4_device_supported": (ctypes.c_int, []),
        "nvfp4_launch_count": (ctypes.c_uint64, []),
        "nvfp4_linear_fused_noalloc": (ctypes.c_int, [vp, i64, i64, u8p, u8p, i64, segp, fp, ctypes.c_int, vp,
                                                      ctypes.c_uint, vp]),
        "nvfp4_quantize_weights_gated": (ctypes.c_int, [vp, i64, i64, i64, u8p, u8p, fp, vp, sz, vp]),
        "nvfp4_linear_swiglu": (ctypes.c_int, [vp, i64, i64, u8p, u8p, i64, fp, vp, u8p, u8p, fp, ctypes.c_uint,
                                               vp, sz, vp]),
        "nvfp4_gemm_prequant_swiglu": (ctypes.c_int, [u8p, u8p, fp, i64, i64, u8p, u8p, i64, fp, vp, vp, sz, vp]),
        "nvfp4_fp8_kv_calibrate": (ctypes.c_int, [vp, i64, i64, i64, fp, vp, sz, vp]),
        "nvfp4_fp8_kv_quantize": (ctypes.c_int, [vp, i64, i64, i64, fp, u8p, i64, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().nvfp4_status_string(int(code)).decode()


def _check(rc: int, where: str):
    if rc != 0:
        raise Nvfp4Error(rc, where)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _segs(segments):
    arr = (Segment * len(segments))(*[Segment(int(a), int(b)) for a, b in segments])
    return arr, len(segments)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("nvfp4 ops take CUDA tensors only (there is no CPU path)")


def _input_2d(X, name, contiguous=False):
    """A bf16 [rows, cols] tensor that a kernel reads row by row (unit column
    stride; fully contiguous where the call takes no leading dimension)."""
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1 or (contiguous and not X.is_contiguous()):
        raise ValueError(f"{name} must be a 2-D bf16 tensor with unit column stride"
                         f"{' and contiguous' if contiguous else ''} (got {X.dtype}, shape {tuple(X.shape)}, "
                         f"strides {X.stride()})")


def _nbytes(t):
    return t.numel() * t.element_size()


def _buffer(t, nbytes, name, dtype=None):
    """A caller-supplied buffer that a kernel accesses as `nbytes` of
    contiguous memory.  The library receives only its address, so its size
    is checked here."""
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if _nbytes(t) < nbytes:
        raise ValueError(f"{name} holds {_nbytes(t)} bytes, the call needs {int(nbytes)}")


def _same_k(K, w):
    if K != w.K:
        raise ValueError(f"K = {K} does not match the weight's K = {w.K}")


def _gated(w):
    if not w.gated:
        raise ValueError("this call needs a gated weight from quantize_weights_gated")


def device_supported() -> bool:
    return bool(lib().nvfp4_device_supported())


def launch_count() -> int:
    return int(lib().nvfp4_launch_count())


def get_status(stream=None) -> int:
    """Synchronize the stream and return/clear the device status word."""
    return int(lib().nvfp4_get_status(_stream(stream)))


def sf_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_sf_bytes(rows, K))


def quant_workspace_bytes(nseg: int = 1) -> int:
    return int(lib().nvfp4_quant_workspace_bytes(nseg))


def workspace_bytes(M: int, N: int, K: int, nseg: int = 1) -> int:
    return int(lib().nvfp4_workspace_bytes(M, N, K, nseg))


def act_scale_offset() -> int:
    return int(lib().nvfp4_linear_act_scale_offset())


def _empty_u8(n, device):
    return torch.empty(max(int(n), 1), dtype=torch.uint8, device=device)


@dataclass
class QuantizedWeight:
    """A (possibly fused) NVFP4 weight: codes [N, K/2], swizzled scales,
    one FP32 global scale per module segment."""
    codes: torch.Tensor
    sf: torch.Tensor
    g_w: torch.Tensor
    segments: list
    N: int
    K: int
    gated: bool = False  # gate/up interleaved in 128-row blocks (nvfp4_quantize_weights_gated)


def quantize_weights(W: torch.Tensor, segments=None, stream=None) -> QuantizedWeight:
    """nvfp4_quantize_weights: per-module dynamic scales over row segments."""
    _require_cuda(W)
    _input_2d(W, "W")
    N, K = W.shape
    segments = [(0, N)] if segments is None else [(int(a), int(b)) for a, b in segments]
    dev = W.device
    codes = _empty_u8(N * K // 2, dev)
    sf = _empty_u8(sf_bytes(N, K), dev)
    g_w = torch.empty(len(segments), dtype=torch.float32, device=dev)
    ws = _empty_u8(quant_workspace_bytes(len(segments)), dev)
    arr, n = _segs(segments)
    _check(lib().nvfp4_quantize_weights(_p(W), N, K, W.stride(0), arr, n, _p(codes), _p(sf), _p(g_w), _p(ws),
                                        _nbytes(ws), _stream(stream)), "nvfp4_quantize_weights")
    return QuantizedWeight(codes[: N * K // 2].view(N, K // 2), sf, g_w, segments, N, K)


def quantize_act(X: torch.Tensor, g_a: torch.Tensor | None = None, static_scale: bool = False, codes=None,
                 sf=None, ws=None, stream=None, amax_given: bool = False):
    """nvfp4_quantize_act -> (codes [M, K/2] u8, swizzled sf u8, g_a fp32[1])."""
    _require_cuda(X, g_a, codes, sf, ws)
    _input_2d(X, "X")
    M, K = X.shape
    dev = X.device
    if codes is None:
        codes = _empty_u8(M * K // 2, dev)
    _buffer(codes, M * K // 2, "codes")
    if sf is None:
        sf = _empty_u8(sf_bytes(M, K), dev)
    _buffer(sf, sf_bytes(M, K), "sf")
    if g_a is None:
        if static_scale:
            raise ValueError("static_scale needs the calibrated scale g_a")
        g_a = torch.empty(1, dtype=torch.float32, device=dev)
    _buffer(g_a, 4, "g_a", torch.float32)
    if ws is None:
        ws = _empty_u8(quant_workspace_bytes(1), dev)
    _buffer(ws, 0, "ws")
    flags = (NVFP4_STATIC_SCALE if static_scale else 0) | (NVFP4_AMAX_GIVEN if amax_given else 0)
    _check(lib().nvfp4_quantize_act(_p(X), M, K, X.stride(0), _p(codes), _p(sf), _p(g_a), flags, _p(ws),
                                    _nbytes(ws), _stream(stream)), "nvfp4_quantize_act")
    return codes.view(-1)[: M * K // 2].view(M, K // 2), sf, g_a


def gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().nvfp4_gemm_workspace_bytes(M, N, K))


def gemm_prequant(a_codes, a_sf, g_a, M: int, K: int, w: QuantizedWeight, out=None, out_fp32=False, stream=None,
                  debug_flags: int = 0, ws=None):
    """nvfp4_gemm_prequant on already-quantized activations; with a workspace
    (ws, gemm_workspace_bytes(M, N, K) bytes) nvfp4_gemm_prequant_ws, which may
    split K at decode sizes."""
    _require_cuda(a_codes, a_sf, g_a, out, ws)
    _same_k(K, w)
    _buffer(a_codes, M * K // 2, "a_codes")
    _buffer(a_sf, sf_bytes(M, K), "a_sf")
    _buffer(g_a, 4, "g_a", torch.float32)
    dt = torch.float32 if out_fp32 else torch.bfloat16
    if out is None:
        out = torch.empty((M, w.N), dtype=dt, device=a_codes.device)
    _buffer(out, M * w.N * out.element_size(), "out", dt)
    arr, n = _segs(w.segments)
    flags = (NVFP4_OUT_FP32 if out_fp32 else 0) | debug_flags
    if ws is not None:
        _buffer(ws, 0, "ws")
        _check(lib().nvfp4_gemm_prequant_ws(_p(a_codes), _p(a_sf), _p(g_a), M, K, _p(w.codes), _p(w.sf), w.N, arr,
                                            _p(w.g_w), n, _p(out), flags, _p(ws), _nbytes(ws), _stream(stream)),
               "nvfp4_gemm_prequant_ws")
        return out
    _check(lib().nvfp4_gemm_prequant(_p(a_codes), _p(a_sf), _p(g_a), M, K, _p(w.codes), _p(w.sf), w.N, arr,
                                     _p(w.g_w), n, _p(out), flags, _stream(stream)), "nvfp4_gemm_prequant")
    return out


def linear_fused(X: torch.Tensor, w: QuantizedWeight, out=None, out_fp32=False, ws=None, static_scale=False,
                 stream=None, single_cta=False):
    """nvfp4_linear_fused: quantize X on the fly, fused-module GEMM with one
    global scale per module segment."""
    _require_cuda(X, out, ws)
    _input_2d(X, "X", contiguous=True)
    M, K = X.shape
    _same_k(K, w)
    dt = torch.float32 if out_fp32 else torch.bfloat16
    if out is None:
        out = torch.empty((M, w.N), dtype=dt, device=X.device)
    _buffer(out, M * w.N * out.element_size(), "out", dt)
    if ws is None:
        ws = _empty_u8(workspace_bytes(M, w.N, K, len(w.segments)), X.device)
    _buffer(ws, 0, "ws")
    arr, n = _segs(w.segments)
    flags = (NVFP4_OUT_FP32 if out_fp32 else 0) | (NVFP4_STATIC_SCALE if static_scale else 0)
    flags |= NVFP4_SINGLE_CTA if single_cta else 0
    _check(lib().nvfp4_linear_fused(_p(X), M, K, _p(w.codes), _p(w.sf), w.N, arr, _p(w.g_w), n, _p(out), flags,
                                    _p(ws), _nbytes(ws), _stream(stream)), "nvfp4_linear_fused")
    return out


def linear(X: torch.Tensor, w: QuantizedWeight, out=None, out_fp32=False, ws=None, stream=None):
    """nvfp4_linear: single-module linear (uses g_w[0])."""
    _require_cuda(X, out, ws)
    _input_2d(X, "X", contiguous=True)
    M, K = X.shape
    _same_k(K, w)
    dt = torch.float32 if out_fp32 else torch.bfloat16
    if out is None:
        out = torch.empty((M, w.N), dtype=dt, device=X.device)
    _buffer(out, M * w.N * out.element_size(), "out", dt)
    if ws is None:
        ws = _empty_u8(workspace_bytes(M, w.N, K, 1), X.device)
    _buffer(ws, 0, "ws")
    flags = NVFP4_OUT_FP32 if out_fp32 else 0
    _check(lib().nvfp4_linear(_p(X), M, K, _p(w.codes), _p(w.sf), _p(w.g_w), w.N, _p(out), flags, _p(ws),
                              _nbytes(ws), _stream(stream)), "nvfp4_linear")
    return out


def linear_workspace_views(ws: torch.Tensor, M: int, K: int):
    """The activation scale, codes and scale factors a linear call left in
    its workspace (for tests): (g_a fp32[1], codes [M, K/2], sf)."""
    off = act_scale_offset()
    g_a = ws[off: off + 4].view(torch.float32)
    codes = ws[1024: 1024 + M * K // 2].view(M, K // 2)
    sf_off = (1024 + M * K // 2 + 1023) // 1024 * 1024
    sf = ws[sf_off: sf_off + sf_bytes(M, K)]
    return g_a, codes, sf


def swiglu_quantize(gate_up: torch.Tensor, h=None, codes=None, sf=None, g_h=None, ws=None, stream=None):
    """nvfp4_swiglu_quantize -> (h bf16 [M, F], codes, sf, g_h)."""
    _require_cuda(gate_up, h, codes, sf, g_h, ws)
    _input_2d(gate_up, "gate_up")
    M, F2 = gate_up.shape
    if F2 % 2:
        raise ValueError(f"gate_up has an odd number of columns ({F2})")
    F = F2 // 2
    dev = gate_up.device
    if h is None:
        h = torch.empty((M, F), dtype=torch.bfloat16, device=dev)
    _buffer(h, M * F * 2, "h", torch.bfloat16)
    if codes is None:
        codes = _empty_u8(M * F // 2, dev)
    _buffer(codes, M * F // 2, "codes")
    if sf is None:
        sf = _empty_u8(sf_bytes(M, F), dev)
    _buffer(sf, sf_bytes(M, F), "sf")
    if g_h is None:
        g_h = torch.empty(1, dtype=torch.float32, device=dev)
    _buffer(g_h, 4, "g_h", torch.float32)
    if ws is None:
        ws = _empty_u8(quant_workspace_bytes(1), dev)
    _buffer(ws, 0, "ws")
    _check(lib().nvfp4_swiglu_quantize(_p(gate_up), M, F, gate_up.stride(0), _p(h), _p(codes), _p(sf), _p(g_h),
                                       _p(ws), _nbytes(ws), _stream(stream)), "nvfp4_swiglu_quantize")
    return h, codes.view(-1)[: M * F // 2].view(M, F // 2), sf, g_h


NOALLOC_MAX_ELEMS = 1 << 22
NOALLOC_MAX_SF_BYTES = 1 << 19


def linear_fused_noalloc(X: torch.Tensor, w: QuantizedWeight, out=None, out_fp32=False, stream=None):
    """nvfp4_linear_fused_noalloc: the fused linear with its activation
    scratch in the library's own fixed device array, for callers that cannot
    allocate device memory where the layer runs (M*K <= 2^22).  `out` may be
    passed to keep the call free of allocations on the Python side too."""
    _require_cuda(X, out)
    _input_2d(X, "X", contiguous=True)
    M, K = X.shape
    _same_k(K, w)
    dt = torch.float32 if out_fp32 else torch.bfloat16
    if out is None:
        out = torch.empty((M, w.N), dtype=dt, device=X.device)
    _buffer(out, M * w.N * out.element_size(), "out", dt)
    arr, n = _segs(w.segments)
    flags = NVFP4_OUT_FP32 if out_fp32 else 0
    _check(lib().nvfp4_linear_fused_noalloc(_p(X), M, K, _p(w.codes), _p(w.sf), w.N, arr, _p(w.g_w), n, _p(out),
                                            flags, _stream(stream)), "nvfp4_linear_fused_noalloc")
    return out


def quantize_weights_gated(W: torch.Tensor, stream=None) -> QuantizedWeight:
    """nvfp4_quantize_weights_gated: W = [gate F | up F] rows -> interleaved
    gate/up NVFP4 weight with one global scale per module."""
    _require_cuda(W)
    _input_2d(W, "W")
    if W.shape[0] % 2:
        raise ValueError(f"W must hold gate and up rows, an even count (got {W.shape[0]})")
    N, K = W.shape
    F = N // 2
    dev = W.device
    codes = _empty_u8(N * K // 2, dev)
    sf = _empty_u8(sf_bytes(N, K), dev)
    g_w = torch.empty(2, dtype=torch.float32, device=dev)
    ws = _empty_u8(quant_workspace_bytes(2), dev)
    _check(lib().nvfp4_quantize_weights_gated(_p(W), F, K, W.stride(0), _p(codes), _p(sf), _p(g_w), _p(ws),
                                              _nbytes(ws), _stream(stream)), "nvfp4_quantize_weights_gated")
    return QuantizedWeight(codes[: N * K // 2].view(N, K // 2), sf, g_w, [(0, F), (F, N)], N, K, gated=True)


def linear_swiglu(X: torch.Tensor, w: QuantizedWeight, h=None, h_codes=None, h_sf=None, g_h=None, ws=None,
                  static_scale=False, stream=None, single_cta=False):
    """nvfp4_linear_swiglu -> (h bf16 [M, F], h_codes [M, F/2], h_sf, g_h)."""
    _require_cuda(X, h, h_codes, h_sf, g_h, ws)
    _gated(w)
    _input_2d(X, "X", contiguous=True)
    M, K = X.shape
    _same_k(K, w)
    F = w.N // 2
    dev = X.device
    if h is None:
        h = torch.empty((M, F), dtype=torch.bfloat16, device=dev)
    _buffer(h, M * F * 2, "h", torch.bfloat16)
    if h_codes is None:
        h_codes = _empty_u8(M * F // 2, dev)
    _buffer(h_codes, M * F // 2, "h_codes")
    if h_sf is None:
        h_sf = _empty_u8(sf_bytes(M, F), dev)
    _buffer(h_sf, sf_bytes(M, F), "h_sf")
    if g_h is None:
        g_h = torch.empty(1, dtype=torch.float32, device=dev)
    _buffer(g_h, 4, "g_h", torch.float32)
    if ws is None:
        ws = _empty_u8(workspace_bytes(M, w.N, K, 2), dev)
    _buffer(ws, 0, "ws")
    flags = (NVFP4_STATIC_SCALE if static_scale else 0) | (NVFP4_SINGLE_CTA if single_cta else 0)
    _check(lib().nvfp4_linear_swiglu(_p(X), M, K, _p(w.codes), _p(w.sf), F, _p(w.g_w), _p(h), _p(h_codes),
                                     _p(h_sf), _p(g_h), flags, _p(ws), _nbytes(ws), _stream(stream)),
           "nvfp4_linear_swiglu")
    return h, h_codes.view(-1)[: M * F // 2].view(M, F // 2), h_sf, g_h


def gemm_prequant_swiglu(a_codes, a_sf, g_a, M: int, K: int, w: QuantizedWeight, h=None, ws=None, stream=None):
    """nvfp4_gemm_prequant_swiglu -> (h bf16 [M, F], ws holding max|h|)."""
    _require_cuda(a_codes, a_sf, g_a, h, ws)
    _gated(w)
    _same_k(K, w)
    _buffer(a_codes, M * K // 2, "a_codes")
    _buffer(a_sf, sf_bytes(M, K), "a_sf")
    _buffer(g_a, 4, "g_a", torch.float32)
    F = w.N // 2
    if h is None:
        h = torch.empty((M, F), dtype=torch.bfloat16, device=a_codes.device)
    _buffer(h, M * F * 2, "h", torch.bfloat16)
    if ws is None:
        ws = _empty_u8(quant_workspace_bytes(1), a_codes.device)
    _buffer(ws, 0, "ws")
    _check(lib().nvfp4_gemm_prequant_swiglu(_p(a_codes), _p(a_sf), _p(g_a), M, K, _p(w.codes), _p(w.sf), F,
                                            _p(w.g_w), _p(h), _p(ws), _nbytes(ws), _stream(stream)),
           "nvfp4_gemm_prequant_swiglu")
    return h, ws


def fp8_kv_calibrate(X: torch.Tensor, scale=None, ws=None, stream=None) -> torch.Tensor:
    """nvfp4_fp8_kv_calibrate -> the calibrated FP8 KV-cache scale (device
    fp32 [1]) of a bf16 [rows, cols] cache tensor."""
    _require_cuda(X, scale, ws)
    _input_2d(X, "X")
    rows, cols = X.shape
    if scale is None:
        scale = torch.empty(1, dtype=torch.float32, device=X.device)
    _buffer(scale, 4, "scale", torch.float32)
    if ws is None:
        ws = _empty_u8(quant_workspace_bytes(1), X.device)
    _buffer(ws, 0, "ws")
    _check(lib().nvfp4_fp8_kv_calibrate(_p(X), rows, cols, X.stride(0), _p(scale), _p(ws), _nbytes(ws),
                                        _stream(stream)), "nvfp4_fp8_kv_calibrate")
    return scale


def fp8_kv_quantize(X: torch.Tensor, scale: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """nvfp4_fp8_kv_quantize -> E4M3 codes (uint8 [rows, cols]) of a bf16 cache
    tensor with a calibrated scale (device fp32)."""
    _require_cuda(X, scale, out)
    _input_2d(X, "X")
    rows, cols = X.shape
    _buffer(scale, 4, "scale", torch.float32)
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=X.device)
    # out may be a strided view (leading dimension out.stride(0)); every byte
    # the kernel writes lies inside its [rows, cols] extent
    if out.dtype != torch.uint8 or out.dim() != 2 or out.stride(1) != 1 or out.shape[0] < rows or \
            out.shape[1] < cols:
        raise ValueError(f"out must be a uint8 [>= {rows}, >= {cols}] tensor with unit column stride "
                         f"(got {out.dtype}, shape {tuple(out.shape)}, strides {out.stride()})")
    _check(lib().nvfp4_fp8_kv_quantize(_p(X), rows, cols, X.stride(0), _p(scale), _p(out), out.stride(0),
                                       _stream(stream)), "nvfp4_fp8_kv_quantize")
    return out
