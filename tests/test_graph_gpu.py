"""Chains of linears whose kernels overlap through programmatic dependent
launch: each layer's output is the next layer's input, so every kernel must
wait for its predecessor before reading.  Eager and CUDA-graph replays of the
same chain give the same bits, at prefill (CTA-pair GEMM) and decode
(split-K) sizes, and the chain's last output matches the oracle applied to
the GPU's own input of that layer."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import ops
from nvfp4_w4a4_quantized_act_b200 import workloads as wl
from nvfp4_testutil import DEV, host

pytestmark = pytest.mark.gpu


def _chain(M, K, depth, seed):
    ws = [ops.quantize_weights(wl.weight_normal(K, K, 0.05, seed + i).to(DEV)) for i in range(depth)]
    X = wl.activation_normal(M, K, seed).to(DEV)
    bufs = [torch.empty((M, K), dtype=torch.bfloat16, device=DEV) for _ in range(depth)]
    wsp = torch.empty(ops.workspace_bytes(M, K, K), dtype=torch.uint8, device=DEV)

    def run():
        src = X
        for w, out in zip(ws, bufs):
            ops.linear(src, w, out=out, ws=wsp)
            src = out
    return ws, X, bufs, run


@pytest.mark.parametrize("M,K", [(4, 1024), (300, 512), (1024, 2048)])
def test_graph_replay_equals_eager(M, K):
    ws, X, bufs, run = _chain(M, K, 4, 7)
    run()
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    eager = [host(b.view(torch.int16)).copy() for b in bufs]
    for b in bufs:
        b.zero_()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        run()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert ops.get_status() == 0
    for e, b in zip(eager, bufs):
        assert np.array_equal(e, host(b.view(torch.int16)))
    # the last layer against the oracle on the GPU's own input to it
    xin = wl.bf16_bits(bufs[-2].cpu())
    ca, sa, ga = oracle.quantize_tensor(xin)
    cw, sw, gw = oracle.quantize_tensor(wl.bf16_bits(wl.weight_normal(K, K, 0.05, 7 + 3)))
    C, B = oracle.linear_full(ca, sa, ga, cw, sw, gw)
    out = oracle.bf16_bits_to_f32(host(bufs[-1].view(torch.int16)).view(np.uint16)).astype(np.float64)
    a = np.maximum(np.abs(out), 1e-38)
    half_ulp = 0.5 * np.exp2(np.floor(np.log2(a)) - 7)
    bad = np.abs(out - C) > oracle.gemm_tolerance(B) + half_ulp
    assert not np.any(bad), f"{int(bad.sum())} outputs outside tolerance"
    del g
