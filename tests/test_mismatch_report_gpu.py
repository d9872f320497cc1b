"""The global-scale mismatch report on a reduced token count.  Serving the
fused weight with the first module's scale multiplies module m's outputs by
rho = g_0 / g_m, so its error lies within rho * (repaired error) of |rho - 1|;
module 0 is untouched; per-module scales (the repair) leave only the NVFP4
quantization error, and re-quantizing every module with one shared scale
lands close to it."""
import numpy as np
import pytest

import oracle
from nvfp4_w4a4_quantized_act_b200 import mismatch_report
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import check_gemm

pytestmark = pytest.mark.gpu


def test_mismatch_report_small():
    r = mismatch_report.run(tokens=1024, rows=128, seed=3)
    assert r["status"] == 0
    mods = r["modules"]
    assert [m["module"] for m in mods] == ["q", "k", "v", "z", "b", "a"]
    assert mods[0]["mismatch_scale"] == 1.0
    assert mods[0]["rel_err_mismatch"] == mods[0]["rel_err_repaired"]
    assert max(abs(m["mismatch_scale"] - 1.0) for m in mods) > 1.0
    for m in mods:
        rho, rep, mis, sh = m["mismatch_scale"], m["rel_err_repaired"], m["rel_err_mismatch"], m["rel_err_shared"]
        assert rep < 0.2, m
        assert abs(mis - abs(rho - 1.0)) <= rho * rep * (1 + 1e-4) + 1e-6, m
        assert sh < 1.5 * rep + 0.01, m


def test_mismatch_report_outputs_match_the_oracle():
    """Each of the report's three served outputs, element by element on the
    sampled rows, against the oracle's GEMM of the same quantization:
    repaired = per-module codes and scales with g_m on module m's rows;
    mismatch = the same codes and block scales with g_0 on every row (the
    fault of "Why Gated DeltaNet Survives 4-Bit Quantization", kipquest.com,
    "The abstract" / "The deep dive"); shared = the weight re-quantized with
    one global scale for all rows."""
    seed = 3
    r = mismatch_report.run(tokens=1024, rows=48, seed=seed, keep_outputs=True)
    assert r["status"] == 0
    lin = wl.gdn_inproj_linear(seed)
    xb = wl.bf16_bits(wl.activation_normal(1024, lin.K, seed))
    wb = wl.bf16_bits(wl.fused_weight(lin, seed))
    N = lin.N
    ca, sa, ga = oracle.quantize_tensor(xb)
    pick = r["rows"]
    ca, sa = ca[pick], sa[pick]
    cw, sw, gseg = oracle.quantize_segments(wb, lin.segments)
    g_rows = {"repaired": oracle.rows_scale(lin.segments, gseg, N),
              "mismatch": np.full(N, gseg[0], dtype=np.float32)}
    for name, grow in g_rows.items():
        C, B = oracle.linear_full(ca, sa, ga, cw, sw, grow)
        check_gemm(r["outputs"][name], C, B, name)
    cs, ss, gs = oracle.quantize_segments(wb, [(0, N)])
    assert np.float32(r["g_shared"]) == gs[0]
    C, B = oracle.linear_full(ca, sa, ga, cs, ss, np.full(N, gs[0], dtype=np.float32))
    check_gemm(r["outputs"]["shared"], C, B, "shared")
