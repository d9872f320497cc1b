"""The C ABI library builds, loads and exports every symbol the header
declares; host-side argument checks return their status codes before any
CUDA work (these calls need no GPU)."""
import ctypes
import os
import re

import pytest

from nvfp4_w4a4_quantized_act_b200 import build as nbuild
from nvfp4_w4a4_quantized_act_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


@pytest.fixture(scope="module")
def L():
    nbuild.build()
    return ops.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


def test_header_declarations_are_exported(L):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert sorted(ops.EXPORTED) == names


def test_sizes(L):
    assert ops.sf_bytes(8192, 5120) == 8192 * 320
    assert ops.sf_bytes(64, 256) == 128 * 16
    assert ops.sf_bytes(1, 16) == 128 * 4
    assert ops.sf_bytes(5, 17) == 0
    assert ops.quant_workspace_bytes(1) >= 4 and ops.quant_workspace_bytes(0) == 0
    ws = ops.workspace_bytes(8192, 34816, 5120, 2)
    assert ws >= 8192 * 5120 // 2 + 8192 * 320 + 1024
    assert ops.act_scale_offset() == 256


def _act_bytes(M, K):
    codes_end = 1024 + M * K // 2
    sf_off = -(-codes_end // 1024) * 1024
    return sf_off + ops.sf_bytes(M, K)


# split counts of the cost model in nvfp4_api.cu (0.6 us per K stage of a CTA
# against the partials' bytes and the cost of their sum), worked by hand
@pytest.mark.parametrize("M,N,K,splits", [
    (16, 5120, 5120, 5),     # 20 tiles, 20 stages: 5 splits of 4 stages
    (1, 1024, 5120, 7),      # 4 tiles: 7 splits of <= 3 stages (8 would leave 3 per split too)
    (3, 1000, 5120, 7),      # ragged N
    (128, 1280, 17408, 8),   # 68 stages, 5 tiles: 8 splits of <= 9 (staged partials from 64 rows)
    (16, 16480, 5120, 2),    # 65 tiles: at most 148 // 65 = 2
    (64, 16480, 5120, 1),    # the partials would cost more than the stages saved
    (128, 5120, 5120, 4),    # staged partials: 4 splits of 5 stages
    (64, 5120, 5120, 5),     # staged partials: 5 splits of 4 stages
    (33, 5120, 5120, 4),     # per-row partials below 64 rows
    (128, 34816, 5120, 1),   # 136 tiles fill the GPU: no split
    (16, 5120, 256, 1),      # one stage of K: no split
    (129, 5120, 5120, 1),    # more than one 128-row block: CTA-pair GEMM, no split
])
def test_decode_workspace_holds_split_partials(L, M, N, K, splits):
    """M <= 128 linears reserve splits x M x N fp32 partial sums after the
    activation (256-byte aligned); N = 0 sizes the activation alone."""
    act = _act_bytes(M, K)
    assert ops.workspace_bytes(M, 0, K) == act
    if splits == 1:
        assert ops.workspace_bytes(M, N, K) == act
    else:
        assert ops.workspace_bytes(M, N, K) == -(-act // 256) * 256 + splits * M * N * 4
    # the pre-quantized GEMM's workspace is the partials alone
    assert ops.gemm_workspace_bytes(M, N, K) == (splits * M * N * 4 if splits > 1 else 0)


def test_gemm_workspace_argument_errors(L):
    fake = ctypes.c_void_p(1 << 20)
    one = _segarr([(0, 5120)])
    need = ops.gemm_workspace_bytes(16, 5120, 5120)
    assert need > 0 and ops.gemm_workspace_bytes(16, 5120, 96) == 0
    assert L.nvfp4_gemm_prequant_ws(fake, fake, fake, 16, 5120, fake, fake, 5120, one, fake, 1, fake, 0, fake,
                                    need - 4, None) == 7
    mis = ctypes.c_void_p((1 << 20) + 8)
    assert L.nvfp4_gemm_prequant_ws(fake, fake, fake, 16, 5120, fake, fake, 5120, one, fake, 1, fake, 0, mis,
                                    need, None) == 3


def _segarr(pairs):
    return (ops.Segment * len(pairs))(*[ops.Segment(a, b) for a, b in pairs])


def test_argument_errors_return_before_launch(L):
    i64 = ctypes.c_int64
    fake = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced: checks fail first
    mis = ctypes.c_void_p((1 << 20) + 8)
    # null input
    assert L.nvfp4_quantize_act(None, 8, 64, 64, fake, fake, fake, 0, fake, 256, None) == 1
    # K not a multiple of 16
    assert L.nvfp4_quantize_act(fake, 8, 40, 40, fake, fake, fake, 0, fake, 256, None) == 2
    # leading dimension smaller than K
    assert L.nvfp4_quantize_act(fake, 8, 64, 32, fake, fake, fake, 0, fake, 256, None) == 1
    # misaligned input
    assert L.nvfp4_quantize_act(mis, 8, 64, 64, fake, fake, fake, 0, fake, 256, None) == 3
    # unknown flag bit
    assert L.nvfp4_quantize_act(fake, 8, 64, 64, fake, fake, fake, 1 << 7, fake, 256, None) == 1
    # workspace too small
    assert L.nvfp4_quantize_act(fake, 8, 64, 64, fake, fake, fake, 0, fake, 2, None) == 7
    segs_ok = _segarr([(0, 10), (10, 32)])
    # GEMM: K % 64
    assert L.nvfp4_gemm_prequant(fake, fake, fake, 8, 96, fake, fake, 32, segs_ok, fake, 2, fake, 0, None) == 2
    # segments not covering [0, N)
    bad = _segarr([(0, 10), (12, 32)])
    assert L.nvfp4_gemm_prequant(fake, fake, fake, 8, 128, fake, fake, 32, bad, fake, 2, fake, 0, None) == 1
    short = _segarr([(0, 10), (10, 30)])
    assert L.nvfp4_gemm_prequant(fake, fake, fake, 8, 128, fake, fake, 32, short, fake, 2, fake, 0, None) == 1
    # too many segments
    many = _segarr([(i, i + 1) for i in range(17)])
    assert L.nvfp4_gemm_prequant(fake, fake, fake, 8, 128, fake, fake, 17, many, fake, 17, fake, 0, None) == 1
    # negative sizes
    assert L.nvfp4_gemm_prequant(fake, fake, fake, -1, 128, fake, fake, 32, segs_ok, fake, 2, fake, 0, None) == 1
    # linear_fused: workspace too small
    assert L.nvfp4_linear_fused(fake, 8, 128, fake, fake, 32, segs_ok, fake, 2, fake, 0, fake, 16, None) == 7
    # decode-sized linear given only the activation's share (no room for the split-K partials)
    one = _segarr([(0, 5120)])
    act_only = ops.workspace_bytes(16, 0, 5120)
    assert L.nvfp4_linear_fused(fake, 16, 5120, fake, fake, 5120, one, fake, 1, fake, 0, fake, act_only, None) == 7
    # weights: misaligned leading dimension
    assert L.nvfp4_quantize_weights(fake, 32, 64, 68, segs_ok, 2, fake, fake, fake, fake, 256, None) == 3
    # SwiGLU: F % 16
    assert L.nvfp4_swiglu_quantize(fake, 8, 24, 48, fake, fake, fake, fake, fake, 256, None) == 2
    for code in range(9):
        assert ops.status_string(code)


def test_fp8_kv_argument_errors_return_before_launch(L):
    fake = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced: checks fail first
    mis8 = ctypes.c_void_p((1 << 20) + 8)
    mis4 = ctypes.c_void_p((1 << 20) + 4)
    # calibrate: cols % 8, ld < cols, null input, null scale, misaligned X, small workspace
    assert L.nvfp4_fp8_kv_calibrate(fake, 4, 12, 16, fake, fake, 256, None) == 2
    assert L.nvfp4_fp8_kv_calibrate(fake, 4, 16, 8, fake, fake, 256, None) == 1
    assert L.nvfp4_fp8_kv_calibrate(None, 4, 16, 16, fake, fake, 256, None) == 1
    assert L.nvfp4_fp8_kv_calibrate(fake, 4, 16, 16, None, fake, 256, None) == 1
    assert L.nvfp4_fp8_kv_calibrate(mis8, 4, 16, 16, fake, fake, 256, None) == 3
    assert L.nvfp4_fp8_kv_calibrate(fake, 4, 16, 20, fake, fake, 256, None) == 3
    assert L.nvfp4_fp8_kv_calibrate(fake, 4, 16, 16, fake, fake, 2, None) == 7
    # quantize: same shape rules, plus ldo < cols, misaligned out / ldo
    assert L.nvfp4_fp8_kv_quantize(fake, 4, 12, 16, fake, fake, 16, None) == 2
    assert L.nvfp4_fp8_kv_quantize(fake, 4, 16, 16, fake, fake, 8, None) == 1
    assert L.nvfp4_fp8_kv_quantize(fake, 4, 16, 16, None, fake, 16, None) == 1
    assert L.nvfp4_fp8_kv_quantize(fake, 4, 16, 16, fake, None, 16, None) == 1
    assert L.nvfp4_fp8_kv_quantize(fake, 4, 16, 16, fake, mis4, 16, None) == 3
    assert L.nvfp4_fp8_kv_quantize(fake, 4, 16, 16, fake, fake, 20, None) == 3
    # empty tensors are no-ops
    assert L.nvfp4_fp8_kv_quantize(None, 0, 16, 16, fake, None, 16, None) == 0


def test_segment_tables_are_checked_before_launch(L):
    """Segments must be ordered, contiguous and cover [0, N); nseg in
    [1, 16]; the table must exist.  Every case fails before any launch."""
    fake = ctypes.c_void_p(1 << 20)
    cases = {
        "unsorted": [(10, 32), (0, 10)],
        "overlapping": [(0, 20), (10, 32)],
        "gap": [(0, 10), (12, 32)],
        "past N": [(0, 10), (10, 40)],
        "reversed": [(0, 20), (20, 10), (10, 32)],
    }
    for name, pairs in cases.items():
        segs = _segarr(pairs)
        assert L.nvfp4_gemm_prequant(fake, fake, fake, 8, 128, fake, fake, 32, segs, fake, len(pairs), fake, 0,
                                     None) == 1, name
        assert L.nvfp4_linear_fused(fake, 8, 128, fake, fake, 32, segs, fake, len(pairs), fake, 0, fake,
                                    1 << 24, None) == 1, name
        assert L.nvfp4_linear_fused_noalloc(fake, 8, 128, fake, fake, 32, segs, fake, len(pairs), fake, 0,
                                            None) == 1, name
    ok = _segarr([(0, 32)])
    assert L.nvfp4_gemm_prequant(fake, fake, fake, 8, 128, fake, fake, 32, ok, fake, 0, fake, 0, None) == 1
    assert L.nvfp4_gemm_prequant(fake, fake, fake, 8, 128, fake, fake, 32, None, fake, 1, fake, 0, None) == 1
    assert L.nvfp4_quantize_weights(fake, 32, 64, 64, None, 1, fake, fake, fake, fake, 256, None) == 1


def test_noalloc_limits_and_flags(L):
    fake = ctypes.c_void_p(1 << 20)
    one = _segarr([(0, 256)])
    # the calibrated activation scale is not supported without a workspace
    assert L.nvfp4_linear_fused_noalloc(fake, 8, 128, fake, fake, 256, one, fake, 1, fake, 1, None) == 1
    # M * K above the fixed scratch
    assert L.nvfp4_linear_fused_noalloc(fake, 1024, 8192, fake, fake, 256, one, fake, 1, fake, 0, None) == 7
    # K % 64
    assert L.nvfp4_linear_fused_noalloc(fake, 8, 96, fake, fake, 256, one, fake, 1, fake, 0, None) == 2


def test_gated_entry_points_check_arguments_before_launch(L):
    fake = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    qws = ops.quant_workspace_bytes(2)
    # gated weight quantize: F % 128, K % 16, ldw < K, misaligned ldw, workspace, null input
    assert L.nvfp4_quantize_weights_gated(fake, 100, 64, 64, fake, fake, fake, fake, qws, None) == 2
    assert L.nvfp4_quantize_weights_gated(fake, 128, 40, 40, fake, fake, fake, fake, qws, None) == 2
    assert L.nvfp4_quantize_weights_gated(fake, 128, 64, 32, fake, fake, fake, fake, qws, None) == 1
    assert L.nvfp4_quantize_weights_gated(fake, 128, 64, 68, fake, fake, fake, fake, qws, None) == 3
    assert L.nvfp4_quantize_weights_gated(fake, 128, 64, 64, fake, fake, fake, fake, 4, None) == 7
    assert L.nvfp4_quantize_weights_gated(None, 128, 64, 64, fake, fake, fake, fake, qws, None) == 1
    # gated GEMM on quantized activations: F % 128, K % 64, workspace, misaligned h
    assert L.nvfp4_gemm_prequant_swiglu(fake, fake, fake, 8, 128, fake, fake, 100, fake, fake, fake, 256,
                                        None) == 2
    assert L.nvfp4_gemm_prequant_swiglu(fake, fake, fake, 8, 96, fake, fake, 128, fake, fake, fake, 256,
                                        None) == 2
    assert L.nvfp4_gemm_prequant_swiglu(fake, fake, fake, 8, 128, fake, fake, 128, fake, fake, fake, 16,
                                        None) == 7
    assert L.nvfp4_gemm_prequant_swiglu(fake, fake, fake, 8, 128, fake, fake, 128, fake, mis, fake, 256,
                                        None) == 3
    # linear with the SwiGLU epilogue: unknown flag, F % 128, null g_h, misaligned h_codes, workspace
    need = ops.workspace_bytes(8, 256, 128, 2)
    assert L.nvfp4_linear_swiglu(fake, 8, 128, fake, fake, 128, fake, fake, fake, fake, fake, 1 << 12, fake,
                                 need, None) == 1
    assert L.nvfp4_linear_swiglu(fake, 8, 128, fake, fake, 96, fake, fake, fake, fake, fake, 0, fake, need,
                                 None) == 2
    assert L.nvfp4_linear_swiglu(fake, 8, 128, fake, fake, 128, fake, fake, fake, fake, None, 0, fake, need,
                                 None) == 1
    assert L.nvfp4_linear_swiglu(fake, 8, 128, fake, fake, 128, fake, fake, mis, fake, fake, 0, fake, need,
                                 None) == 3
    assert L.nvfp4_linear_swiglu(fake, 8, 128, fake, fake, 128, fake, fake, fake, fake, fake, 0, fake, need - 1,
                                 None) == 7


def _prototypes():
    """name -> (return type, [parameter types]) for every function in the
    header, comments removed, parameter names dropped."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    text = "\n".join(l for l in text.splitlines() if not l.lstrip().startswith("#"))
    text = re.sub(r'extern\s+"C"\s*\{|\}', ";", text)
    out = {}
    for stmt in text.split(";"):
        m = re.fullmatch(r"\s*([A-Za-z_][\w\s\*]*?)\b(nvfp4_[a-z0-9_]+)\s*\(([^)]*)\)\s*", stmt, flags=re.S)
        if not m or stmt.lstrip().startswith("typedef"):
            continue
        ret, name, params = m.groups()
        ps = [p.strip() for p in params.split(",") if p.strip() and p.strip() != "void"]
        types = [re.sub(r"\b[A-Za-z_]\w*$", "", p).strip() if not p.endswith("*") else p for p in ps]
        out[name] = (" ".join(ret.split()), [" ".join(t.split()) for t in types])
    return out


def _ctype_of(c_type):
    if "nvfp4_segment" in c_type and "*" in c_type:
        return ctypes.POINTER(ops.Segment)
    if c_type.replace(" ", "") in ("constchar*", "char*"):
        return ctypes.c_char_p
    if "*" in c_type:
        return ctypes.c_void_p
    return {"int": ctypes.c_int, "unsigned": ctypes.c_uint, "int64_t": ctypes.c_int64, "size_t": ctypes.c_size_t,
            "uint64_t": ctypes.c_uint64}[c_type.replace("const ", "")]


def test_binding_signatures_match_the_header(L):
    """Every ctypes restype/argtypes equals the header prototype's types
    (pointer, segment table, 32/64-bit integer, size): a mismatch would pass
    garbage silently."""
    protos = _prototypes()
    assert sorted(protos) == sorted(ops.EXPORTED)
    for name, (ret, params) in protos.items():
        f = getattr(L, name)
        assert f.restype == _ctype_of(ret), (name, ret, f.restype)
        assert list(f.argtypes) == [_ctype_of(p) for p in params], (name, params, f.argtypes)
