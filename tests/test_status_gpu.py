"""Failure detection without a GPU fault: every wait inside the GEMM kernel
is bounded.  NVFP4_DEBUG_INJECT_STALL skips the kernel's loads so its waits
run out (20 ms); the kernel must unwind, latch NVFP4_ERR_TIMEOUT for the host,
and leave the context usable for the next, correct, GEMM."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import check_gemm, host, oracle_act_on_device, oracle_weight_on_device

pytestmark = pytest.mark.gpu


def test_stalled_gemm_times_out_and_context_survives():
    X, W = wl.tiny_linear(0)
    xb, wb = wl.bf16_bits(X), wl.bf16_bits(W)
    (ac, asf, ga), (oc, os_, og) = oracle_act_on_device(xb)
    qw, (wc, ws, wg) = oracle_weight_on_device(wb, [(0, 128)])
    assert ops.get_status() == 0
    out = torch.full((64, 128), 7.0, dtype=torch.float32, device="cuda")
    ops.gemm_prequant(ac, asf, ga, 64, 256, qw, out=out, out_fp32=True, debug_flags=ops.NVFP4_DEBUG_INJECT_STALL)
    assert ops.get_status() == 5  # NVFP4_ERR_TIMEOUT, read and cleared
    assert ops.get_status() == 0
    assert torch.all(out == 7.0)  # nothing was written
    good = ops.gemm_prequant(ac, asf, ga, 64, 256, qw, out_fp32=True)
    assert ops.get_status() == 0
    C, B = oracle.linear_full(oc, os_, og, wc, ws, wg)
    check_gemm(host(good), C, B, "after timeout")
