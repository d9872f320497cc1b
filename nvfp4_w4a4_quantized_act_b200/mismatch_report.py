"""Global-scale mismatch report: what serving per-module-calibrated NVFP4
weights through one fused GEMM with a single global scale does to each
module's outputs, and what each repair leaves.

The pages describe the fault: when each module carries its own calibrated
global scale and a serving kernel runs the modules as one GEMM under a single
scale, the outputs go wrong without any error showing, and the gates are the
modules they name as damaged -- kipquest.com, "Why Gated DeltaNet Survives
4-Bit Quantization", sections "The abstract" and "The deep dive".  They give
no error figures; this measures them on synthetic tensors shaped like the GDN
input projection (q, k, v, z, b, a: N = 16480 in six modules whose weight
scales differ by up to 10x), M = 16384 tokens, K = 5120.

Three ways to serve the fused weight:
  repaired  per-module FP32 global scales, each applied to its own columns in
            the GEMM epilogue (nvfp4_linear_fused);
  mismatch  one global scale (the first module's) for every column, the
            pages' fault: module m comes out scaled by g_0 / g_m;
  shared    every module re-quantized with one shared global scale (the
            largest), so one scale is right for all columns.
Per module: relative error ||Y - Y_ref||_F / ||Y_ref||_F over sampled rows,
with Y_ref = X W^T in fp64 from the bf16 inputs (no quantization).

    python -m nvfp4_w4a4_quantized_act_b200.mismatch_report [--tokens 16384] [--rows 256] [--json]

Needs a CUDA device and the built library.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import ops
from . import workloads as wl


def _rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))


def run(tokens: int = 16384, rows: int = 256, seed: int = 3, keep_outputs: bool = False) -> dict:
    """Serve the fused weight the three ways; per module, the relative error
    of each against X W^T.  keep_outputs adds the sampled fp32 outputs
    ('outputs': name -> [rows, N]) and their token indices ('rows')."""
    lin = wl.gdn_inproj_linear(seed)
    segs = lin.segments
    K, N = lin.K, lin.N
    X = wl.activation_normal(tokens, K, seed)
    W = wl.fused_weight(lin, seed)
    dev = "cuda"
    Xd, Wd = X.to(dev), W.to(dev)

    repaired_w = ops.quantize_weights(Wd, segs)
    g = repaired_w.g_w.clone()
    mismatch_w = ops.QuantizedWeight(repaired_w.codes, repaired_w.sf, g[:1].clone(), [(0, N)], N, K)
    shared_w = ops.quantize_weights(Wd, [(0, N)])

    pick = np.sort(np.random.default_rng(seed).choice(tokens, size=min(rows, tokens), replace=False))
    idx = torch.from_numpy(pick).to(dev)
    outs = {}
    for name, qw in (("repaired", repaired_w), ("mismatch", mismatch_w), ("shared", shared_w)):
        y = ops.linear_fused(Xd, qw, out_fp32=True)
        outs[name] = y.index_select(0, idx).cpu().numpy().astype(np.float64)
    status = ops.get_status()
    ref = X.float().numpy()[pick].astype(np.float64) @ W.float().numpy().astype(np.float64).T

    gh = g.cpu().numpy().astype(np.float64)
    g_shared = float(shared_w.g_w.cpu()[0])
    modules = []
    for (a, b), m, gm in zip(segs, lin.modules, gh):
        modules.append({
            "module": m.name, "columns": [a, b], "sigma": m.sigma, "g_w": gm,
            "mismatch_scale": float(gh[0] / gm),
            "rel_err_repaired": _rel_err(outs["repaired"][:, a:b], ref[:, a:b]),
            "rel_err_mismatch": _rel_err(outs["mismatch"][:, a:b], ref[:, a:b]),
            "rel_err_shared": _rel_err(outs["shared"][:, a:b], ref[:, a:b]),
        })
    res = {"tokens": tokens, "K": K, "N": N, "rows_sampled": int(len(pick)), "g_shared": g_shared,
           "status": status, "modules": modules}
    if keep_outputs:
        res["outputs"] = outs
        res["rows"] = pick
    return res


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--tokens", type=int, default=16384)
    ap.add_argument("--rows", type=int, default=256)
    ap.add_argument("--seed", type=int, default=3)
    ap.add_argument("--json", action="store_true")
    a = ap.parse_args()
    r = run(a.tokens, a.rows, a.seed)
    if a.json:
        print(json.dumps(r))
        return
    print(f"GDN input projection, M={r['tokens']} (rows sampled: {r['rows_sampled']}), K={r['K']}, N={r['N']}; "
          f"status {r['status']}")
    print(f"{'module':>6} {'cols':>12} {'sigma':>8} {'g_0/g_m':>8} {'repaired':>9} {'mismatch':>9} {'shared':>9}")
    for m in r["modules"]:
        print(f"{m['module']:>6} {m['columns'][0]:>5}-{m['columns'][1]:<6} {m['sigma']:8.4f} "
              f"{m['mismatch_scale']:8.3f} {m['rel_err_repaired']:9.4f} {m['rel_err_mismatch']:9.4f} "
              f"{m['rel_err_shared']:9.4f}")


if __name__ == "__main__":
    main()
