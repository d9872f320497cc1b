"""Benchmark of the NVFP4 W4A4 linear path on B200.

Workload (default): the full stack of 496 linear layers of a 48 Gated-DeltaNet
/ 16 attention hybrid at hidden size 5120, run on one 8192-token prefill
chunk.  Every input-sharing group of modules is one fused GEMM with a global
scale per module (4 GEMMs a layer, 256 a step):

  GDN layer       in_proj [qkv 8192 | z 6144 | b 48 | a 48] <- X (5120)
                  out      5120 <- Y (6144)
                  gate_up [gate 17408 | up 17408] <- X2 (5120), SwiGLU in the
                           epilogue: h = silu(gate) * up (17408)
                  down     5120 <- h
  attention layer qkv [q+gate 12288 | k 1024 | v 1024] <- X, o 5120 <- Y,
                  gate_up, down as above

A step quantizes every GEMM input on the fly (per-tensor dynamic global
scale), runs the block-scaled FP4 GEMMs with the per-module global-scale
epilogue, and computes + quantizes the MLP intermediate.  Weights are random
N(0, 0.02), quantized once offline (per module).  Activations X, X2 ~ N(0,1)
with 4 outlier channels x50, Y ~ N(0,1); all synthetic and seeded.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

TOKENS = 8192
HIDDEN = 5120
METRIC = "NVFP4 W4A4 linear TFLOPS (quant+GEMM) at prefill shapes; % of FP4 & HBM peak"
WORKLOAD = "496-linear hybrid stack (48 GDN + 16 attention layers, hidden 5120, MLP 17408), one 8192-token prefill chunk"
FP4_PER_BF16 = 4.0  # dense FP4 : dense BF16 tensor throughput on B200 (9 : 2.25 PFLOP/s nominal)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) per GEMM launch, mean over the four GEMM launches of
# one layer, from one ncu capture (the DRAM-bytes capture of these sources).
# Reported only while the GEMM kernel sources and the host functions that set
# up their launches (tile order, grid, tensor-map boxes) still hash to the
# captured value.
GEMM_TRAFFIC = {"source_sha256_12": "248398c47700", "bytes_per_launch": 272.20e6}
_CSRC = os.path.join(ROOT, "nvfp4_w4a4_quantized_act_b200", "csrc")
# (file, None for the whole file, or the functions of it that configure GEMM launches)
GEMM_SOURCES = [(os.path.join(_CSRC, "gemm_kernel.cuh"), None),
                (os.path.join(_CSRC, "gemm_pair_kernel.cuh"), None),
                (os.path.join(_CSRC, "ptx_sm100.cuh"), None),
                (os.path.join(_CSRC, "nvfp4_api.cu"), ("make_codes_map", "make_sf_map", "make_out_map", "run_gemm"))]


def _function_text(text, name):
    """Source of the top-level function `name` (its signature line through the
    first closing brace in column 0)."""
    import re
    m = re.search(r"^[A-Za-z_][^\n;]*\b" + re.escape(name) + r"\(", text, flags=re.M)
    if m is None:
        raise ValueError(f"function {name} not found")
    end = text.index("\n}\n", m.start())
    return text[m.start(): end + 3]


def gemm_source_hash():
    """Hash of the GEMM sources with comments and whitespace removed, so that
    an edit to a comment (or to code outside the listed functions) keeps the
    captured traffic valid."""
    import hashlib
    import re
    h = hashlib.sha256()
    for entry in GEMM_SOURCES:
        path, funcs = entry if isinstance(entry, tuple) else (entry, None)
        with open(path) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        if funcs is not None:
            text = "\n".join(_function_text(text, fn) for fn in funcs)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:12]


def gemm_traffic():
    return GEMM_TRAFFIC["bytes_per_launch"] if gemm_source_hash() == GEMM_TRAFFIC["source_sha256_12"] else None


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["nvfp4", "reference"], default="nvfp4")
    ap.add_argument("--layers", type=int, default=64, help="layers in the stack (64 = the full model)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side", action="store_true",
                    help="skip the side measurements (quantize, FP8 KV cache, decode) after the timed steps")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--side-only", choices=["quantize", "fp8_kv", "decode"], default=None,
                    help="run only this side measurement (one GPU) and print it as one JSON line; "
                         "for profiling the kernels behind it")
    ap.add_argument("--decode-tokens", default="1,16,64,128",
                    help="comma-separated tokens per decode step for the decode measurement")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


# --------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.proc is None:
            return out
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        self.file.close()
        os.unlink(self.file.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                pass
        if sm:
            out["sm_mhz"] = statistics.median(sm)
            out["sm_max_mhz"] = max(mx)
        out["reasons"] = sorted(reasons)
        out["samples"] = len(sm)
        return out


# ------------------------------------------------------------ the stack

def stack_flops(layers) -> float:
    f = 0.0
    for _, lins in layers:
        for lin in lins:
            f += 2.0 * TOKENS * lin.N * lin.K
    return f


class Stack:
    """Quantized weights of the stack plus the reusable activation/output
    buffers of one prefill chunk."""

    def __init__(self, n_layers: int, device, seed: int = 1000):
        from nvfp4_w4a4_quantized_act_b200 import ops
        from nvfp4_w4a4_quantized_act_b200 import workloads as wl
        self.ops = ops
        self.layers = wl.stack_layers()[:n_layers]
        self.weights = []  # per layer: 4 QuantizedWeight
        for li, (kind, lins) in enumerate(self.layers):
            qs = []
            for gi, lin in enumerate(lins):
                parts = [wl.weight_normal_cuda(m.width, lin.K, m.sigma, seed + 97 * li + 11 * gi + j, device)
                         for j, m in enumerate(lin.modules)]
                W = torch.cat(parts, 0) if len(parts) > 1 else parts[0]
                del parts
                if lin.name == "gate_up":
                    qs.append(ops.quantize_weights_gated(W))
                else:
                    qs.append(ops.quantize_weights(W, lin.segments))
                del W
            self.weights.append(qs)
        torch.cuda.synchronize()
        # activations (synthetic, seeded) and buffers
        self.X = wl.activation_normal_cuda(TOKENS, HIDDEN, 11, device=device)
        self.X2 = wl.activation_normal_cuda(TOKENS, HIDDEN, 12, device=device)
        self.Y = wl.activation_normal_cuda(TOKENS, 6144, 13, n_outliers=0, device=device)
        self.outs = {}
        for _, lins in self.layers[:4]:
            for lin in lins:
                if lin.name != "gate_up":
                    self.outs.setdefault((lin.name, lin.N), torch.empty((TOKENS, lin.N), dtype=torch.bfloat16,
                                                                         device=device))
        maxK = max(lin.K for _, lins in self.layers for lin in lins)
        self.a_codes = torch.empty(TOKENS * maxK // 2, dtype=torch.uint8, device=device)
        self.a_sf = torch.empty(ops.sf_bytes(TOKENS, maxK), dtype=torch.uint8, device=device)
        self.g_a = torch.empty(1, dtype=torch.float32, device=device)
        self.qws = torch.empty(ops.quant_workspace_bytes(1), dtype=torch.uint8, device=device)
        self.hws = torch.empty(ops.quant_workspace_bytes(1), dtype=torch.uint8, device=device)
        self.h = torch.empty((TOKENS, 17408), dtype=torch.bfloat16, device=device)
        self.lin_ws = torch.empty(ops.workspace_bytes(TOKENS, 0, maxK), dtype=torch.uint8, device=device)
        self.flops = stack_flops(self.layers)
        self.gemm_flops = [2.0 * TOKENS * lin.N * lin.K for _, lins in self.layers for lin in lins]

    def _input(self, lin):
        if lin.name in ("gdn_out", "attn_o"):
            return self.Y
        if lin.name == "gate_up":
            return self.X2
        return self.X

    def step_split(self, gemm_events=None):
        """One step through nvfp4_quantize_act / nvfp4_gemm_prequant(_swiglu),
        with CUDA events around each GEMM launch."""
        ops = self.ops
        k = 0
        for qs, (_, lins) in zip(self.weights, self.layers):
            for lin, qw in zip(lins, qs):
                if lin.name == "down":
                    # h was written by the gated epilogue, its max|h| is in hws
                    ac, asf, _ = ops.quantize_act(self.h, g_a=self.g_a, codes=self.a_codes, sf=self.a_sf,
                                                  ws=self.hws, amax_given=True)
                else:
                    ac, asf, _ = ops.quantize_act(self._input(lin), g_a=self.g_a, codes=self.a_codes, sf=self.a_sf,
                                                  ws=self.qws)
                if gemm_events is not None:
                    gemm_events[k][0].record()
                if lin.name == "gate_up":
                    ops.gemm_prequant_swiglu(ac, asf, self.g_a, TOKENS, lin.K, qw, h=self.h, ws=self.hws)
                else:
                    ops.gemm_prequant(ac, asf, self.g_a, TOKENS, lin.K, qw, out=self.outs[(lin.name, lin.N)])
                if gemm_events is not None:
                    gemm_events[k][1].record()
                k += 1

    def step_public(self, inputs=None, final_out=None):
        """One step through the user-facing calls (nvfp4_linear_fused for the
        fused projections, nvfp4_linear_swiglu for gate/up + SwiGLU, and
        nvfp4_gemm_prequant on the quantized h for the down projection).
        inputs: (X, X2, Y) to read instead of the stack's own; final_out:
        where the last layer's down projection writes (default: the shared
        down buffer)."""
        ops = self.ops
        X, X2, Y = inputs if inputs is not None else (self.X, self.X2, self.Y)
        last = None
        n_layers = len(self.layers)
        for li, (qs, (_, lins)) in enumerate(zip(self.weights, self.layers)):
            for lin, qw in zip(lins, qs):
                if lin.name == "gate_up":
                    _, hc, hsf, gh = ops.linear_swiglu(X2, qw, h=self.h, h_codes=self.a_codes, h_sf=self.a_sf,
                                                       g_h=self.g_a, ws=self.lin_ws)
                elif lin.name == "down":
                    out = self.outs[(lin.name, lin.N)]
                    if final_out is not None and li == n_layers - 1:
                        out = final_out
                    ops.gemm_prequant(hc, hsf, gh, TOKENS, lin.K, qw, out=out)
                    last = out
                else:
                    src = Y if lin.name in ("gdn_out", "attn_o") else X
                    ops.linear_fused(src, qw, out=self.outs[(lin.name, lin.N)], ws=self.lin_ws)
        return last


# -------------------------------------------------------------- GPU arm

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """TFLOPS of the whole job: the work of every rank over the slowest
    rank's step time."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


def bench_gpu(args, rank, world, local):
    from nvfp4_w4a4_quantized_act_b200 import build as nbuild
    from nvfp4_w4a4_quantized_act_b200 import ops
    nbuild.build()
    if not ops.device_supported():
        raise RuntimeError("the current device is not an sm_100 GPU")
    dev = f"cuda:{local}"
    stack = Stack(args.layers, dev)
    n_gemm = len(stack.gemm_flops)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        stack.step_split()
    torch.cuda.synchronize()
    if ops.get_status() != 0:
        raise RuntimeError("device status set during warm-up")

    clocks = ClockSampler(local)
    l0 = ops.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    # the timed region: the steps alone, no event between kernels
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        stack.step_split()
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    launches = ops.launch_count() - l0
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    status = ops.get_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    # a separate, untimed pass of the same steps with CUDA events around each
    # GEMM launch: the GEMM kernel's own durations for the roofline
    gemm_steps = max(2, min(args.steps, 5))
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_gemm)]
          for _ in range(gemm_steps)]
    for s in range(gemm_steps):
        stack.step_split(ev[s])
    torch.cuda.synchronize()
    gemm_ms = [sum(ev[s][k][0].elapsed_time(ev[s][k][1]) for s in range(gemm_steps)) / gemm_steps
               for k in range(n_gemm)]
    if ops.get_status() != 0:
        raise RuntimeError("device status set during the GEMM-duration pass")

    ms_per_step = elapsed_ms / args.steps
    value = aggregate_throughput(stack.flops, world, ms_per_step)
    gemm_tflops = sum(stack.gemm_flops) / (sum(gemm_ms) * 1e-3) / 1e12
    pk, pk_kind = peaks()
    fp4_peak = pk["bf16_tflops_sustained"] * FP4_PER_BF16

    # quantize kernel throughput: one activation [8192, 5120] at HBM roofline
    quant = kv = decode = None
    if not args.no_side:
        quant = quantize_roofline(stack, pk, pk_kind)
        kv = fp8_kv_roofline(pk, pk_kind)
        decode = decode_roofline(stack, pk, pk_kind, decode_tokens(args))

    e2e = None
    if not args.no_e2e:
        e2e = bench_e2e(stack, args, world)

    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 + e4m3 block scales) x nvfp4 -> fp32 accumulate -> bf16",
        "data": "synthetic (seeded N(0,1) activations with outlier channels; random N(0,0.02) weights)",
        "config": {
            "workload": WORKLOAD if args.layers == 64 else f"{args.layers}-layer prefix of the stack",
            "tokens": TOKENS, "hidden": HIDDEN, "layers": args.layers, "gemms_per_step": n_gemm,
            "linears_per_step": sum(len(m.modules) for _, lins in stack.layers for m in lins),
            "gemm_tflop_per_step": round(stack.flops / 1e12, 2),
            "l2": "no flush: each step streams 13.4 GB of NVFP4 weights, far larger than the 126 MB L2",
            "parallelism": f"replicas x{world} (no collectives)",
        },
        "roofline": {
            "kernel": "gemm_nvf4_pair_kernel (CTA-pair tcgen05 block-scaled FP4 GEMM, 256x256 tiles; "
                      "per-module-scale or SwiGLU epilogue)",
            "bound": "tensor",
            "achieved": round(gemm_tflops, 1),
            "peak": round(fp4_peak, 1),
            "unit": "TFLOP/s",
            "frac": round(gemm_tflops / fp4_peak, 4),
            "traffic": gemm_traffic(),
            "traffic_unit": "bytes per launch (DRAM read+write, ncu, mean of one layer's 4 GEMMs)",
            "algorithmic_bytes_per_launch": round(gemm_alg_bytes(stack), 0),
            "peak_basis": f"{pk_kind} bf16 sustained {pk['bf16_tflops_sustained']} TF/s x {FP4_PER_BF16} "
                          "(nominal dense FP4:BF16 ratio)",
            "frac_of_datasheet_9pf": round(gemm_tflops / 9000.0, 4),
        },
        "quantize_roofline": quant,
        "fp8_kv_roofline": kv,
        "decode_roofline": decode,
        "gemm_share_of_step": round(sum(gemm_ms) / ms_per_step, 4),
        "timing": {"ms_per_step": "CUDA events around the K timed steps only, no event between kernels",
                   "gemm": f"roofline.achieved and gemm_share_of_step from a separate untimed pass of "
                           f"{gemm_steps} steps with CUDA events around each of the {n_gemm} GEMM launches"},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if e2e is not None:
        res["e2e"] = e2e
    return res


def gemm_alg_bytes(stack) -> float:
    """Mean algorithmic bytes per GEMM launch over the step: codes (K/2 per
    row) and scales (K/16 per row) of both operands plus the bf16 output."""
    tot, n = 0.0, 0
    for _, lins in stack.layers:
        for lin in lins:
            out_cols = lin.N // 2 if lin.name == "gate_up" else lin.N
            tot += (TOKENS + lin.N) * lin.K * (0.5 + 1 / 16) + TOKENS * out_cols * 2
            n += 1
    return tot / n


def flush_l2(buf):
    """Write a buffer larger than L2, then read it back: the write evicts the
    timed kernel's data, the read leaves L2 holding clean lines, so the timed
    kernel does not also pay for writing back the flush's dirty lines."""
    buf.zero_()
    buf.view(torch.int32).max()


def _timed_flushed(fn, flush, reps=13, skip=3):
    ts = []
    for i in range(reps):
        flush_l2(flush)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        e.synchronize()
        if i >= skip:
            ts.append(s.elapsed_time(e))
    return statistics.median(ts)


def _timed_rotating(fn, n_inputs, rounds=4, reps=7, skip=2):
    """Median time per call of fn(i), called for i = 0 .. n_inputs-1 `rounds`
    times back to back between two CUDA events: with the inputs together
    larger than L2, no call finds its own input there, and each call's launch
    overlaps the previous one as it would inside a step."""
    ts = []
    for r in range(reps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(rounds):
            for i in range(n_inputs):
                fn(i)
        e.record()
        e.synchronize()
        if r >= skip:
            ts.append(s.elapsed_time(e) / (rounds * n_inputs))
    return statistics.median(ts)


def quantize_roofline(stack, pk, pk_kind):
    """Activation quantization of X [8192, 5120] (the stack's GDN/attention
    input): the dynamic path (clearing + amax + quantize launches, the
    roofline figure) and the calibrated single pass.  Timed as 16 calls back
    to back over 4 distinct inputs and outputs (4 x 107.5 MB, more than the
    126 MB L2), per call = total / 16.  For context: one call with L2 flushed
    before it (launch latency included in its events), and one read of X by a
    plain torch reduction under the same flush."""
    from nvfp4_w4a4_quantized_act_b200 import ops
    from nvfp4_w4a4_quantized_act_b200 import workloads as wl
    X = stack.X
    dev = X.device
    n_in = 4
    xs = [X] + [wl.activation_normal_cuda(TOKENS, HIDDEN, 21 + i, device=dev) for i in range(n_in - 1)]
    bufs = [(torch.empty(TOKENS * HIDDEN // 2, dtype=torch.uint8, device=dev),
             torch.empty(ops.sf_bytes(TOKENS, HIDDEN), dtype=torch.uint8, device=dev),
             torch.empty(1, dtype=torch.float32, device=dev),
             torch.empty(ops.quant_workspace_bytes(1), dtype=torch.uint8, device=dev)) for _ in range(n_in)]

    def call(i, static):
        c, sf, g, ws = bufs[i]
        ops.quantize_act(xs[i], g_a=g, codes=c, sf=sf, ws=ws, static_scale=static)

    for i in range(n_in):  # calibrated scales for the static pass: the inputs' own
        call(i, False)
    torch.cuda.synchronize()
    ms = _timed_rotating(lambda i: call(i, False), n_in)
    ms_static = _timed_rotating(lambda i: call(i, True), n_in)
    if ops.get_status() != 0:
        raise RuntimeError("device status set by the quantize measurement")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ms_one = _timed_flushed(lambda: call(0, False), flush)
    ms_one_static = _timed_flushed(lambda: call(0, True), flush)
    xi = X.view(torch.int32)
    ms_read = _timed_flushed(lambda: xi.max(), flush)
    del xs, bufs, flush
    alg = TOKENS * HIDDEN * (2 + 0.5 + 1 / 16)
    gbs = alg / (ms * 1e-3) / 1e9
    return {"kernel": "zero_words_kernel + amax_kernel + quantize_act_kernel (dynamic per-tensor scale), "
                      "X [8192, 5120] bf16",
            "bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / pk["hbm_gbs"], 4), "us": round(ms * 1e3, 2),
            "algorithmic_bytes": int(alg), "peak_basis": pk_kind,
            "l2": "16 calls back to back over 4 distinct inputs and outputs (4 x 107.5 MB > 126 MB L2)",
            "static_scale_us": round(ms_static * 1e3, 2),
            "static_scale_gbs": round(alg / (ms_static * 1e-3) / 1e9, 1),
            "static_scale_frac": round(alg / (ms_static * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
            "one_call_l2_flushed_us": {"dynamic": round(ms_one * 1e3, 2), "static": round(ms_one_static * 1e3, 2),
                                       "note": "256 MB written and read back before the call; its events "
                                               "include the launch latency"},
            "torch_read_of_x_us": round(ms_read * 1e3, 2),
            "torch_read_of_x_gbs": round(X.numel() * 2 / (ms_read * 1e-3) / 1e9, 1)}


def fp8_kv_roofline(pk, pk_kind):
    """FP8 KV-cache quantization with a calibrated scale, L2 flushed before
    each launch; 3 bytes per element (bf16 in, one E4M3 byte out).  Two
    launches shapes: the K cache of one attention layer at 8192 tokens (8 KV
    heads x 128 = [8192, 1024], what one layer writes), and the K and V caches
    of all 16 attention layers of the chunk as one [262144, 1024] launch (the
    roofline figure: the per-layer launch is short enough that launch and
    ramp-up time are a large part of it)."""
    from nvfp4_w4a4_quantized_act_b200 import ops
    from nvfp4_w4a4_quantized_act_b200 import workloads as wl
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def timed(rows):
        X = wl.activation_normal(rows, 1024, seed=1024, n_outliers=8, scale=20.0).to("cuda")
        scale = ops.fp8_kv_calibrate(X)
        out = torch.empty((rows, 1024), dtype=torch.uint8, device="cuda")
        ts = []
        for i in range(13):
            flush_l2(flush)
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            ops.fp8_kv_quantize(X, scale, out=out)
            e.record()
            e.synchronize()
            if i >= 3:
                ts.append(s.elapsed_time(e))
        del X, out
        return statistics.median(ts)

    ms_layer = timed(TOKENS)
    rows_all = TOKENS * 16 * 2
    ms_all = timed(rows_all)
    alg = rows_all * 1024 * 3
    gbs = alg / (ms_all * 1e-3) / 1e9
    return {"kernel": "kv_quantize_kernel (FP8 E4M3, calibrated per-tensor scale), K+V caches of 16 attention "
                      "layers at 8192 tokens as one [262144, 1024] bf16 launch",
            "bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / pk["hbm_gbs"], 4), "us": round(ms_all * 1e3, 2),
            "algorithmic_bytes": int(alg), "peak_basis": pk_kind, "l2": "256 MB written and read back before each launch",
            "one_layer_k_cache_us": round(ms_layer * 1e3, 2),
            "one_layer_k_cache_gbs": round(TOKENS * 1024 * 3 / (ms_layer * 1e-3) / 1e9, 1)}


def decode_roofline(stack, pk, pk_kind, token_counts=(1, 16, 64, 128)):
    """Decode steps through the same 64-layer stack: M new tokens per step
    (M <= 128 runs the split-K GEMM), every linear through the public calls
    (nvfp4_linear_fused; nvfp4_linear_swiglu for gate/up, whose quantized h
    feeds the down projection through nvfp4_gemm_prequant_ws).  A step streams every NVFP4
    weight once (13.4 GB, far above L2), so it is bound by HBM: the figure is
    weight bytes per step / step time.  Each step is one CUDA graph of 256
    linears (captured once per M, replayed)."""
    from nvfp4_w4a4_quantized_act_b200 import ops
    dev = stack.X.device
    wbytes = sum(qw.codes.numel() + qw.sf.numel() for qs in stack.weights for qw in qs)
    res = {"kernel": "split-K linear chain (quantize with its amax + gemm_nvf4_kernel split-K + split sum) per linear; "
                     "gate/up with SwiGLU, down on its quantized h",
           "bound": "hbm", "unit": "GB/s", "peak": pk["hbm_gbs"], "peak_basis": pk_kind,
           "weight_bytes_per_step": int(wbytes), "linears_per_step": 256, "steps": {}}
    for M in token_counts:
        X, X2, Y = stack.X[:M], stack.X2[:M], stack.Y[:M]
        ws_bytes = max(max(ops.workspace_bytes(M, lin.N, lin.K, len(lin.segments)),
                           ops.gemm_workspace_bytes(M, lin.N, lin.K))
                       for _, lins in stack.layers for lin in lins)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        h = torch.empty((M, 17408), dtype=torch.bfloat16, device=dev)
        hc = torch.empty(M * 17408 // 2, dtype=torch.uint8, device=dev)
        hsf = torch.empty(ops.sf_bytes(M, 17408), dtype=torch.uint8, device=dev)
        gh = torch.empty(1, dtype=torch.float32, device=dev)
        outs = {n: torch.empty((M, n), dtype=torch.bfloat16, device=dev) for n in (5120, 14432, 14336)}

        def step():
            for qs, (_, lins) in zip(stack.weights, stack.layers):
                for lin, qw in zip(lins, qs):
                    if lin.name == "gate_up":
                        ops.linear_swiglu(X2, qw, h=h, h_codes=hc, h_sf=hsf, g_h=gh, ws=ws)
                    elif lin.name == "down":
                        ops.gemm_prequant(hc, hsf, gh, M, lin.K, qw, out=outs[5120], ws=ws)
                    else:
                        src = Y if lin.name in ("gdn_out", "attn_o") else X
                        if lin.N not in outs:
                            outs[lin.N] = torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev)
                        ops.linear_fused(src, qw, out=outs[lin.N], ws=ws)

        l0 = ops.launch_count()
        step()
        launches = ops.launch_count() - l0
        torch.cuda.synchronize()
        if ops.get_status() != 0:
            raise RuntimeError("device status set by the decode step")
        side = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(5):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            graph.replay()
            e.record()
            e.synchronize()
            ts.append(s.elapsed_time(e))
        del graph
        if ops.get_status() != 0:
            raise RuntimeError("device status set by the decode step")
        ms = statistics.median(ts)
        gbs = wbytes / (ms * 1e-3) / 1e9
        res["steps"][str(M)] = {"us_per_step": round(ms * 1e3, 1), "us_per_linear": round(ms * 1e3 / 256, 2),
                                "achieved": round(gbs, 1), "frac": round(gbs / pk["hbm_gbs"], 4),
                                "gpu_launches_per_step": launches}
    return res


def bench_e2e(stack, args, world):
    """Same workload through the user-facing calls, each step's inputs copied
    from pinned host memory and its final output read back, inside the timed
    region.  The copies run on one stream per direction into two alternating
    input sets (and out of two alternating output buffers), so that step i+1's
    inputs and step i-1's output move over PCIe while step i computes, as a
    serving loop would; every step still waits for its own inputs, and the
    timed region ends after the last read-back."""
    dev = stack.X.device
    hX = stack.X.cpu().pin_memory()
    hX2 = stack.X2.cpu().pin_memory()
    hY = stack.Y.cpu().pin_memory()
    sets = [(stack.X, stack.X2, stack.Y),
            (torch.empty_like(stack.X), torch.empty_like(stack.X2), torch.empty_like(stack.Y))]
    last_shape = stack.outs[("down", HIDDEN)].shape
    outs = [torch.empty(last_shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    hOut = [torch.empty(last_shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = hX.numel() * 2 + hX2.numel() * 2 + hY.numel() * 2
    d2h = hOut[0].numel() * 2
    comp = torch.cuda.current_stream()
    # one stream per direction: a read-back waiting for its step must not
    # hold up the next step's inputs behind it
    up = torch.cuda.Stream(device=dev)
    down = torch.cuda.Stream(device=dev)

    def run(n):
        in_free = [None, None]   # compute finished reading input set b
        out_free = [None, None]  # read-back of output buffer b finished
        ready = [None, None]

        def upload(i):
            b = i % 2
            with torch.cuda.stream(up):
                if in_free[b] is not None:
                    up.wait_event(in_free[b])
                for dst, src in zip(sets[b], (hX, hX2, hY)):
                    dst.copy_(src, non_blocking=True)
                ready[b] = up.record_event()

        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)  # overlaps step i
            comp.wait_event(ready[b])
            if out_free[b] is not None:
                comp.wait_event(out_free[b])
            stack.step_public(inputs=sets[b], final_out=outs[b])
            done = comp.record_event()
            in_free[b] = done
            with torch.cuda.stream(down):
                down.wait_event(done)
                hOut[b].copy_(outs[b], non_blocking=True)  # overlaps step i + 1
                out_free[b] = down.record_event()
        comp.wait_stream(up)
        comp.wait_stream(down)

    run(max(1, args.warmup))
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(comp)
    run(args.steps)
    e.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(s.elapsed_time(e), world) / args.steps
    return {"value": round(aggregate_throughput(stack.flops, world, ms), 2), "unit": "TFLOPS",
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "api": "nvfp4_linear_fused / nvfp4_linear_swiglu / nvfp4_gemm_prequant",
            "copies": "pinned host buffers, one copy stream per direction and two alternating input/output "
                      "sets: a step's copies overlap its neighbours' compute"}


# ------------------------------------------------------ CPU oracle legs

def oracle_sample_operands():
    """bf16 bits of the 64 activation rows and 256 gate_up weight rows the
    oracle sample draws its outputs from."""
    from nvfp4_w4a4_quantized_act_b200 import workloads as wl
    x = wl.activation_normal(64, HIDDEN, 11)
    w = wl.weight_normal(256, HIDDEN, 0.02, 1000)
    return wl.bf16_bits(x), wl.bf16_bits(w)


def oracle_sample_time(seconds: float, seed: int = 0, operands=None):
    """Time the oracle on a bounded sample of the stack: quantize the rows it
    needs of one activation and one gate_up weight, then compute sampled
    outputs of that GEMM by fp64 dot products, until `seconds` pass.
    Returns (flops, seconds, outputs)."""
    import oracle
    rng = np.random.default_rng(seed)
    K = HIDDEN
    rows = 64
    xb, wb = operands if operands is not None else oracle_sample_operands()
    flops = 0.0
    outs = 0
    t0 = time.perf_counter()
    while True:
        ca, sa, ga = oracle.quantize_tensor(xb)
        cw, sw, gw = oracle.quantize_tensor(wb)
        ms = rng.integers(0, rows, 1024)
        ns = rng.integers(0, wb.shape[0], 1024)
        oracle.linear_sampled(ca, sa, ga, cw, sw, gw, ms, ns)
        flops += 2.0 * K * len(ms)
        outs += len(ms)
        el = time.perf_counter() - t0
        if el >= seconds:
            return flops, el, outs


def oracle_codec_time():
    """Time the oracle's activation codec on the whole activation-quantize
    workload (X [8192, 5120], Student-t(3) with 1% of channels x100): amax,
    global scale, block scales and codes.  Returns (elements, seconds)."""
    import oracle
    from nvfp4_w4a4_quantized_act_b200 import workloads as wl
    xb = _CODEC_X if _CODEC_X is not None else wl.bf16_bits(wl.act_quant_input())
    t0 = time.perf_counter()
    oracle.quantize_tensor(xb)
    return xb.size, time.perf_counter() - t0


def host_cores() -> int:
    """Cores this process may run on (the container's share of the host)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# The activation the parallel codec timing quantizes, made before the worker
# pool is forked so that every worker reads the parent's copy.
_CODEC_X = None
_SAMPLE_OPERANDS = None


def _pool_gemm_sample(args):
    seconds, seed = args
    return oracle_sample_time(seconds, seed, _SAMPLE_OPERANDS)


def _pool_codec_amax(rows):
    import oracle
    return oracle.amax(_CODEC_X, rows[0], rows[1])


def _pool_codec_quantize(args):
    import oracle
    r0, r1, g = args
    codes, scales = oracle.quantize(np.ascontiguousarray(_CODEC_X[r0:r1]), g)
    return int(codes[:, :1].sum()) + int(scales[:, :1].sum())


class OraclePool:
    """One worker process per host core running the oracle, unchanged, on
    disjoint pieces of the work: sampled GEMM outputs (each worker its own
    seed) and the rows of the activation codec (amax of each worker's rows,
    their maximum, then each worker quantizes its rows with the global
    scale).  The pool is forked before any CUDA call of this process (a fork
    after one is unsafe); workers never touch the GPU."""

    def __init__(self, cores: int | None = None):
        global _CODEC_X, _SAMPLE_OPERANDS
        import multiprocessing as mp
        from nvfp4_w4a4_quantized_act_b200 import workloads as wl
        import oracle
        oracle.build()
        self.cores = cores or host_cores()
        # inputs made here, before the fork: the workers use no torch
        _CODEC_X = wl.bf16_bits(wl.act_quant_input())
        _SAMPLE_OPERANDS = oracle_sample_operands()
        self.pool = mp.get_context("fork").Pool(self.cores)

    def gemm_rate(self, seconds: float, seed0: int = 100):
        """(flops, seconds, outputs) of all workers together: the work of
        every worker over the longest worker's time."""
        res = self.pool.map(_pool_gemm_sample, [(seconds, seed0 + i) for i in range(self.cores)])
        return sum(r[0] for r in res), max(r[1] for r in res), sum(r[2] for r in res)

    def codec_time(self):
        import oracle
        rows = _CODEC_X.shape[0]
        cuts = np.linspace(0, rows, self.cores + 1).astype(int)
        parts = [(int(a), int(b)) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]
        t0 = time.perf_counter()
        a = max(self.pool.map(_pool_codec_amax, parts))
        g = oracle.global_scale(a)
        self.pool.map(_pool_codec_quantize, [(r0, r1, g) for r0, r1 in parts])
        return _CODEC_X.size, time.perf_counter() - t0

    def close(self):
        self.pool.terminate()
        self.pool.join()


def cpu_baseline(seconds: float, pool: OraclePool):
    """The oracle on the host cores: all of them (the baseline's value) and
    one (for reference)."""
    gate_up_flops = 2.0 * TOKENS * 2 * 17408 * HIDDEN
    f1, el1, outs1 = oracle_sample_time(seconds)
    n_codec, t_codec1 = oracle_codec_time()
    fa, ela, outsa = pool.gemm_rate(seconds)
    _, t_codeca = pool.codec_time()
    codec_bytes = n_codec * (2 + 0.5 + 1 / 16)
    return {"value": fa / ela / 1e12, "unit": "TFLOPS", "cores": pool.cores, "kind": "oracle",
            "cores_host": host_cores(), "cpu_model": host_cpu_model(),
            "value_all_cores": fa / ela / 1e12, "value_1core": f1 / el1 / 1e12,
            "sample": f"sampled outputs of a [8192,5120]x[34816,5120]^T gate_up GEMM (K=5120) with on-the-fly "
                      f"quantization of the 64 activation rows and 256 weight rows each batch uses, repeated "
                      f"for {seconds:.0f} s: {outsa} outputs on {pool.cores} worker processes (one per core), "
                      f"{outs1} on one core; C oracle, fp64 dot products",
            "fp64_mac_per_s_with_quantization": {"all_cores": round(fa / 2 / ela, 1), "1core": round(f1 / 2 / el1, 1)},
            "gate_up_full_s_extrapolated": {"all_cores": round(gate_up_flops / (fa / ela), 1),
                                            "1core": round(gate_up_flops / (f1 / el1), 1)},
            "codec": {"gbs": round(codec_bytes / t_codeca / 1e9, 5), "seconds": round(t_codeca, 2),
                      "gbs_1core": round(codec_bytes / t_codec1 / 1e9, 5), "seconds_1core": round(t_codec1, 2),
                      "sample": "the whole [8192,5120] activation, dynamic scale (amax + block quantize); "
                                "rows split across the worker processes; algorithmic bytes 2.5625 per element"}}


def bench_reference(args, rank, world):
    if rank != 0:
        return None
    pool = OraclePool()
    try:
        per_step = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
        for _ in range(args.warmup):
            pool.gemm_rate(per_step / 4)
        tot_f, tot_t = 0.0, 0.0
        for _ in range(args.steps):
            f, t, outs = pool.gemm_rate(per_step)
            tot_f += f
            tot_t += t
    finally:
        pool.close()
    v = tot_f / tot_t / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle GEMM)",
        "data": "synthetic", "config": {"workload": WORKLOAD, "tokens": TOKENS, "hidden": HIDDEN},
        "cpu_baseline": {"value": v, "unit": "TFLOPS", "cores": pool.cores, "kind": "oracle",
                         "cores_host": host_cores(), "cpu_model": host_cpu_model(),
                         "sample": f"each step: {per_step:.1f} s of sampled gate_up outputs with quantization "
                                   f"on {pool.cores} worker processes (one per core)"},
        "e2e": {"value": v, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def decode_tokens(args):
    return tuple(int(t) for t in args.decode_tokens.split(","))


def side_only(args):
    """One side measurement on its own (one GPU), for profiling."""
    from nvfp4_w4a4_quantized_act_b200 import build as nbuild
    from nvfp4_w4a4_quantized_act_b200 import ops
    nbuild.build()
    if not ops.device_supported():
        raise RuntimeError("the current device is not an sm_100 GPU")
    pk, pk_kind = peaks()
    if args.side_only == "fp8_kv":
        return {"side": "fp8_kv", **fp8_kv_roofline(pk, pk_kind)}
    stack = Stack(args.layers, "cuda:0")
    if args.side_only == "quantize":
        return {"side": "quantize", **quantize_roofline(stack, pk, pk_kind)}
    return {"side": "decode", **decode_roofline(stack, pk, pk_kind, decode_tokens(args))}


def main():
    args = parse_args()
    if args.side_only is not None:
        if int(os.environ.get("WORLD_SIZE", "1")) != 1:
            raise SystemExit("--side-only runs on one GPU, without torchrun")
        print(json.dumps(side_only(args)), flush=True)
        return
    if args.impl == "reference":
        # the oracle arm runs on rank 0's host cores only; other ranks exit at once
        rank = int(os.environ.get("RANK", "0"))
        res = bench_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    # the oracle's worker pool is forked before this process makes any CUDA call
    pool = None
    if int(os.environ.get("RANK", "0")) == 0 and not args.no_cpu_baseline:
        pool = OraclePool()
    rank, world, local = dist_setup(args)
    try:
        res = bench_gpu(args, rank, world, local)
        if rank == 0 and res is not None and pool is not None:
            res["cpu_baseline"] = cpu_baseline(args.cpu_seconds, pool)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if pool is not None:
            pool.close()
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
