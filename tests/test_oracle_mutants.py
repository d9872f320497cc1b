"""The oracle's pins must catch plausible mistakes.

Each mutant below plants one mistake in a private copy of the oracle (its C
source or its Python layer): a wrong constant, a dropped absolute value or
sign, the wrong tie rule, a swapped nibble or operand, a wrong index.  The
copy is imported in a child process, ahead of the real oracle on the path,
and the pin tests (tests/test_oracle.py, tests/test_fp8_kv_oracle.py) run
against it; at least one pin has to fail.  An unmodified copy run the same
way has to pass, so a failure is due to the planted mistake and not to the
mechanism.  Everything here is CPU-only and touches no GPU code.
"""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = [os.path.join(ROOT, "tests", "test_oracle.py"), os.path.join(ROOT, "tests", "test_fp8_kv_oracle.py")]
C = "nvfp4_oracle.c"
PY = "__init__.py"

# name -> (file, exact text, replacement); the text must occur exactly once
MUTANTS = {
    # global and block scales
    "global_divisor_448": (C, "float g = amax / 2688.0f;", "float g = amax / 448.0f;"),
    "zero_amax_scale_0": (C, "if (amax == 0.0f)\n        return 1.0f;\n    float g",
                          "if (amax == 0.0f)\n        return 0.0f;\n    float g"),
    "tensor_amax_signed": (C, "float v = fabsf(oracle_bf16_to_float(x[r * ld + k]));",
                           "float v = oracle_bf16_to_float(x[r * ld + k]);"),
    "block_amax_signed": (C, "float v = fabsf(oracle_bf16_to_float(blk[i]));",
                          "float v = oracle_bf16_to_float(blk[i]);"),
    "block_scale_over_4": (C, "float t = bamax / 6.0f;", "float t = bamax / 4.0f;"),
    "block_scale_times_g": (C, "float s32 = t / g;", "float s32 = t * g;"),
    "divisor_without_g": (C, "float d = s * g;", "float d = s;"),
    "scale_product_order": (C, "float t = bamax / 6.0f;\n            float s32 = t / g;",
                            "float t = bamax;\n            float s32 = t / (6.0f * g);"),
    "quotient_two_divisions": (C, "float y = xv / d;", "float y = xv / s / g;"),
    "kv_scale_nvfp4_divisor": (C, "float s = amax / 448.0f;", "float s = amax / 2688.0f;"),
    "multiply_not_divide": (C, "float y = xv / d;", "float y = xv * d;"),
    "zero_block_drops_sign": (C, "c[j] = signbit(xv) ? 8 : 0;", "c[j] = 0;"),
    "nibbles_swapped": (C, "(uint8_t)(c[0] | (c[1] << 4))", "(uint8_t)(c[1] | (c[0] << 4))"),
    # E2M1 / E4M3 formats and rounding
    "ties_to_lower": (C, "(d == bestd && (codes[i] & 1) == 0 && (codes[best] & 1) == 1)", "(0)"),
    "ties_to_upper": (C, "if (d < bestd || (d == bestd && (codes[i] & 1) == 0 && (codes[best] & 1) == 1))",
                      "if (d <= bestd)"),
    "e2m1_saturates_to_4": (C, "mag = 7;", "mag = 6;"),
    "e2m1_drops_sign": (C, "return (signbit(y) ? 8 : 0) | mag;", "return mag;"),
    "e2m1_subnormal_1": (C, "v = 0.5 * m;", "v = 1.0 * m;"),
    "e2m1_mantissa_quarter": (C, "v = (1.0 + 0.5 * m) * ldexp(1.0, e - 1);", "v = (1.0 + 0.25 * m) * ldexp(1.0, e - 1);"),
    "e4m3_saturates_to_nan": (C, "return 0x7E;", "return 0x7F;"),
    "e4m3_bias_8": (C, "v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);", "v = (1.0 + m / 8.0) * ldexp(1.0, e - 8);"),
    "e4m3_subnormal_exp": (C, "v = (m / 8.0) * ldexp(1.0, -6);", "v = (m / 8.0) * ldexp(1.0, -7);"),
    "e4m3_ieee_top_binade": (C, "if (e == 15 && m == 7)", "if (e == 15)"),
    "e4m3_grid_without_448": (C, "return nearest_even_code(a, vals, codes, 127);",
                              "return nearest_even_code(a, vals, codes, 126);"),
    "e2m1_saturates_from_5": (C, "if (a >= 6.0)\n        mag = 7;", "if (a >= 5.0)\n        mag = 7;"),
    # scale-factor layout
    "sf_tile_row_major": (C, "(rr % 32) * 16 + (rr / 32) * 4 + (c % 4)", "(rr / 4) * 16 + (rr % 4) * 4 + (c % 4)"),
    "sf_tiles_unpadded_k": (C, "int64_t cpad = (K / 16 + 3) / 4 * 4;", "int64_t cpad = K / 16;"),
    "sf_tile_stride_unpadded": (C, "int64_t ct_count = (K / 16 + 3) / 4;", "int64_t ct_count = K / 64;"),
    # dequantization and GEMM
    "dequant_scale_per_32": (C, "double s = oracle_e4m3_decode(scales[r * nb + k / 16]);",
                             "double s = oracle_e4m3_decode(scales[r * nb + k / 32]);"),
    "gemm_a_nibbles_swapped": (C, "int ac = (k & 1) ? (ab >> 4) : (ab & 15);", "int ac = (k & 1) ? (ab & 15) : (ab >> 4);"),
    "gemm_w_takes_g_a": (C, "* (double)g_w_row[n];", "* (double)g_a;"),
    "gemm_bound_signed": (C, "bound += fabs(a * w);", "bound += a * w;"),
    "sampled_w_row_from_m": (C, "uint8_t wb = w_codes[n * (K / 2) + k / 2];", "uint8_t wb = w_codes[m * (K / 2) + k / 2];"),
    "dequant_nibbles_swapped": (C, "int c = (k & 1) ? (byte >> 4) : (byte & 15);", "int c = (k & 1) ? (byte & 15) : (byte >> 4);"),
    "block_stride_8": (C, "const uint16_t *blk = x + r * ld + b * 16;", "const uint16_t *blk = x + r * ld + b * 8;"),
    # MLP intermediate and bf16 rounding
    "silu_exp_sign": (C, "double s = gv / (1.0 + exp(-gv));", "double s = gv / (1.0 + exp(gv));"),
    "swiglu_up_is_gate": (C, "gate_up[r * ld + F + j]", "gate_up[r * ld + j]"),
    "bf16_ties_away": (C, "double r = nearbyint(q);", "double r = round(q);"),
    "bf16_one_bit_short": (C, "int ulp_exp = (e - 1) - 7;", "int ulp_exp = (e - 1) - 6;"),
    "bf16_subnormals_flushed_early": (C, "if (ulp_exp < -133)\n        ulp_exp = -133;", "if (ulp_exp < -126)\n        ulp_exp = -126;"),
    # FP8 KV cache
    "kv_scale_240": (C, "float s = amax / 448.0f;", "float s = amax / 240.0f;"),
    "kv_drops_sign": (C, "return signbit(y) ? (m | 0x80) : m;", "return m;"),
    "kv_multiply_not_divide": (C, "oracle_bf16_to_float(x[r * ld + c]) / s;", "oracle_bf16_to_float(x[r * ld + c]) * s;"),
    "kv_zero_amax_scale_0": (C, "if (amax == 0.0f)\n        return 1.0f;\n    float s",
                             "if (amax == 0.0f)\n        return 0.0f;\n    float s"),
    # per-row and per-segment scales
    "rows_share_row0_scale": (C, "float g = g_row[r];", "float g = g_row[0];"),
    "dequant_row0_scale": (C, "(double)g_row[r];", "(double)g_row[0];"),
    "segment_amax_from_row0": (C, "for (int64_t r = r0; r < r1; r++)", "for (int64_t r = 0; r < r1; r++)"),
    # Python layer
    "gated_interleave_inverted": (PY, "out[gated_stored_row(r, F)] = rows_data[r]",
                                  "out[r] = rows_data[gated_stored_row(r, F)]"),
    "segments_share_tensor_amax": (PY, "global_scale(amax(x_bits, a, b))", "global_scale(amax(x_bits))"),
    "rows_take_first_segment": (PY, "g[a:b] = gs", "g[a:b] = g_seg[0]"),
    "gated_layout_concatenated": (PY, "return (2 * block + module) * 128 + within",
                                  "return module * F + block * 128 + within"),
    "silu_mul_exp_sign": (PY, "return g / (1.0 + np.exp(-g)) * np.asarray(u, dtype=np.float64)",
                          "return g / (1.0 + np.exp(g)) * np.asarray(u, dtype=np.float64)"),
    "full_bound_of_sum": (PY, "return A @ W.T, np.abs(A) @ np.abs(W).T", "return A @ W.T, np.abs(A @ W.T)"),
}


def _run(name, mutation, workdir):
    """Copy the oracle into workdir/<name>/oracle, apply the mutation, run the
    pins in a child process with that copy first on the path.  Returns
    (exit code, tail of the output)."""
    base = os.path.join(workdir, name)
    dst = os.path.join(base, "oracle")
    os.makedirs(dst)
    for f in (C, PY):
        shutil.copy(os.path.join(ROOT, "oracle", f), os.path.join(dst, f))
    if mutation is not None:
        fname, old, new = mutation
        path = os.path.join(dst, fname)
        with open(path) as fh:
            text = fh.read()
        assert text.count(old) == 1, f"{name}: mutation text must occur once in {fname}"
        with open(path, "w") as fh:
            fh.write(text.replace(old, new))
    env = dict(os.environ, PYTHONPATH=base + os.pathsep + ROOT, PYTHONDONTWRITEBYTECODE="1",
               CUDA_VISIBLE_DEVICES="")
    # a line that proves which oracle the child imported, then the pins
    probe = subprocess.run([sys.executable, "-c", "import oracle; print(oracle.__file__)"], cwd=base, env=env,
                           capture_output=True, text=True, timeout=300)
    assert probe.stdout.strip().startswith(dst), f"{name}: child imported {probe.stdout.strip()!r}"
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "not gpu",
                        *PINS], cwd=base, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, (r.stdout + r.stderr)[-1500:]


@pytest.fixture(scope="module")
def results():
    workdir = tempfile.mkdtemp(prefix="oracle_mutants_")
    jobs = {"unmodified": None, **MUTANTS}
    try:
        with ThreadPoolExecutor(max_workers=max(2, min(8, os.cpu_count() or 2))) as ex:
            futs = {k: ex.submit(_run, k, m, workdir) for k, m in jobs.items()}
            yield {k: f.result() for k, f in futs.items()}
    finally:
        shutil.rmtree(workdir, ignore_errors=True)


def test_unmodified_copy_passes_the_pins(results):
    rc, out = results["unmodified"]
    assert rc == 0, out


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(results, name):
    rc, out = results[name]
    # exit code 1: at least one pin failed (not a crash or a collection error)
    assert rc == 1, f"mutant {name} survived the pins (exit {rc}):\n{out}"
