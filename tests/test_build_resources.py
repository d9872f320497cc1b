"""Register, spill and stack budgets of every kernel, from ptxas's resource
report (no GPU: nvcc cross-compiles for sm_100a).

The streaming kernels (amax, quantize, SwiGLU, FP8 KV, split sum, clearing)
must not touch local memory at all.  The GEMMs run at one CTA per SM, so
registers are bounded by their launch bounds; the limits on their stack
frame and spills are the current ones, so a change that starts spilling in
the main loop or the epilogue fails here before it reaches a GPU.
"""
import os
import re
import shutil
import subprocess

import pytest

from nvfp4_w4a4_quantized_act_b200 import build as nbuild

# kernel (demangled-name fragment) -> (max registers, max stack bytes, max spill-store bytes)
BUDGET = {
    "gemm_nvf4_pair_kernel<true>": (128, 0, 0),
    "gemm_nvf4_pair_kernel<false>": (128, 16, 16),
    "gemm_nvf4_kernel<true>": (168, 0, 0),
    "gemm_nvf4_kernel<false>": (168, 0, 0),
    "splitk_finalize_kernel": (255, 0, 0),
    "quantize_kernel": (64, 0, 0),
    "quantize_act_kernel": (64, 0, 0),
    "amax_kernel": (64, 0, 0),
    "swiglu_kernel": (64, 0, 0),
    "kv_quantize_kernel": (64, 0, 0),
    "kv_scale_kernel": (64, 0, 0),
    "zero_words_kernel": (64, 0, 0),
}


def _demangle(names):
    filt = shutil.which("c++filt") or "/usr/bin/c++filt"
    out = subprocess.run([filt], input="\n".join(names), capture_output=True, text=True, check=True).stdout
    return out.splitlines()


@pytest.fixture(scope="module")
def report():
    if not os.path.exists(nbuild.NVCC):
        pytest.skip("nvcc not available")
    flags = [f for f in nbuild.NVCC_FLAGS if f != "-shared"]
    cmd = [nbuild.NVCC, *flags, "-Xptxas", "-v", "-c", "-o", os.devnull, *nbuild.sources()]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    entries = []
    cur = None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '([^']+)' for 'sm_100a'", line)
        if m:
            cur = {"mangled": m.group(1)}
            entries.append(cur)
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            cur["stack"], cur["spill_st"], cur["spill_ld"] = map(int, m.groups())
        m = re.search(r"Used (\d+) registers", line)
        if m:
            cur["regs"] = int(m.group(1))
    for e, name in zip(entries, _demangle([e["mangled"] for e in entries])):
        e["name"] = name
    return entries


def test_every_kernel_has_a_budget(report):
    assert report
    for e in report:
        assert any(k in e["name"] for k in BUDGET), f"no budget for {e['name']}"


@pytest.mark.parametrize("kernel", sorted(BUDGET))
def test_kernel_within_budget(report, kernel):
    hits = [e for e in report if kernel in e["name"]]
    assert hits, f"{kernel} not compiled"
    regs, stack, spill = BUDGET[kernel]
    for e in hits:
        assert e["regs"] <= regs, e
        assert e["stack"] <= stack, e
        assert e["spill_st"] <= spill and e["spill_ld"] <= 4 * spill, e
