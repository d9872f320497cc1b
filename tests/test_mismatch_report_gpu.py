"""The global-scale mismatch report on a reduced token count.  Serving the
fused weight with the first module's scale multiplies module m's outputs by
rho = g_0 / g_m, so its error lies within rho * (repaired error) of |rho - 1|;
module 0 is untouched; per-module scales (the repair) leave only the NVFP4
quantization error, and re-quantizing every module with one shared scale
lands close to it."""
import pytest

from nvfp4_w4a4_quantized_act_b200 import mismatch_report

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
