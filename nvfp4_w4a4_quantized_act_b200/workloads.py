"""Seeded synthetic inputs shaped like the prefill workloads of the NVFP4 W4A4
linear layer.  This module holds input recipes only -- no quantization or
GEMM arithmetic -- and is the one module shared by the oracle-side tests and
the CUDA-side tests and benchmark.

Shapes follow the model the paper quantizes: a 48 Gated-DeltaNet / 16
attention hybrid with hidden size 5120 and MLP width 17408 ("Why Gated
DeltaNet Survives 4-Bit Quantization", kipquest.com, "The abstract" and "The
deep dive").  Outliers follow the deep dive's remark that the residual stream
has a few channels whose magnitude is about 100x the median.

Every generator is seeded; values are drawn in fp32/fp64 with numpy's PCG64
(or torch's CUDA generator for the large stack weights) and rounded to bf16
with round-to-nearest-even.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

HIDDEN = 5120
MLP_WIDTH = 17408


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """fp32/fp64 numpy -> bf16 torch (CPU), round to nearest even."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 torch tensor -> uint16 numpy bit patterns (CPU copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def outlier_columns(K: int, count: int, seed: int) -> np.ndarray:
    """`count` distinct column indices chosen by a seeded permutation."""
    return np.sort(_rng(seed + 7919).permutation(K)[:count])


def activation_normal(M: int, K: int, seed: int, n_outliers: int = 4, scale: float = 50.0,
                      outlier_seed: int | None = None) -> torch.Tensor:
    """X ~ N(0,1) [M,K] with `n_outliers` seeded columns multiplied by `scale`."""
    x = _rng(seed).standard_normal((M, K), dtype=np.float32)
    if n_outliers:
        cols = outlier_columns(K, n_outliers, seed if outlier_seed is None else outlier_seed)
        x[:, cols] *= np.float32(scale)
    return to_bf16(x)


def activation_student_t(M: int, K: int, seed: int, nu: float = 3.0, frac: float = 0.01,
                         scale: float = 100.0) -> torch.Tensor:
    """X ~ Student-t(nu) [M,K] with floor(frac*K) seeded channels x scale."""
    rng = _rng(seed)
    x = rng.standard_t(nu, size=(M, K)).astype(np.float32)
    cols = outlier_columns(K, int(np.floor(frac * K)), seed)
    x[:, cols] *= np.float32(scale)
    return to_bf16(x)


def weight_normal(N: int, K: int, sigma: float, seed: int) -> torch.Tensor:
    w = _rng(seed).standard_normal((N, K), dtype=np.float32) * np.float32(sigma)
    return to_bf16(w)


def weight_normal_cuda(N: int, K: int, sigma: float, seed: int, device="cuda") -> torch.Tensor:
    """Large weights drawn directly on the GPU (torch CUDA generator)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
    w.mul_(sigma)
    return w.to(torch.bfloat16)


def activation_normal_cuda(M: int, K: int, seed: int, n_outliers: int = 4, scale: float = 50.0,
                           device="cuda") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    if n_outliers:
        cols = torch.from_numpy(outlier_columns(K, n_outliers, seed)).to(device)
        x[:, cols] *= scale
    return x.to(torch.bfloat16)


def segments_from_widths(widths) -> list[tuple[int, int]]:
    segs, n0 = [], 0
    for w in widths:
        segs.append((n0, n0 + w))
        n0 += w
    return segs


@dataclass
class Module:
    name: str
    width: int
    sigma: float


@dataclass
class FusedLinear:
    """One GEMM over the concatenation of modules that share an input."""
    name: str
    K: int
    modules: list[Module]
    segments: list[tuple[int, int]] = field(init=False)

    def __post_init__(self):
        self.segments = segments_from_widths([m.width for m in self.modules])

    @property
    def N(self) -> int:
        return self.segments[-1][1]


# --------------------------------------------------------------- workloads

def tiny_linear(seed: int = 0):
    """Single linear: X [64,256] N(0,1) with 4 outlier columns x50,
    W [128,256] N(0,0.02)."""
    X = activation_normal(64, 256, seed)
    W = weight_normal(128, 256, 0.02, seed + 1)
    return X, W


def act_quant_input(seed: int = 1, M: int = 8192, K: int = HIDDEN):
    """Activation-quantize workload: [8192,5120] Student-t(3), 1% channels x100."""
    return activation_student_t(M, K, seed)


def mlp_modules():
    gate_up = FusedLinear("gate_up", HIDDEN, [Module("gate", MLP_WIDTH, 0.02), Module("up", MLP_WIDTH, 0.02)])
    down = FusedLinear("down", MLP_WIDTH, [Module("down", HIDDEN, 0.02)])
    return gate_up, down


def gdn_inproj_sigmas(seed: int = 3, n: int = 6) -> list[float]:
    """Per-module sigma, log-uniform in [0.005, 0.05] with the smallest and
    largest pinned to the ends so the spread is the full 10x."""
    u = _rng(seed + 101).uniform(size=n)
    order = np.argsort(u)
    u[order[0]], u[order[-1]] = 0.0, 1.0
    return [float(0.005 * 10.0 ** ui) for ui in u]


def gdn_inproj_linear(seed: int = 3) -> FusedLinear:
    names = ["q", "k", "v", "z", "b", "a"]
    widths = [2048, 2048, 6144, 6144, 48, 48]
    sig = gdn_inproj_sigmas(seed)
    return FusedLinear("gdn_in_proj", HIDDEN, [Module(n, w, s) for n, w, s in zip(names, widths, sig)])


def fused_weight(lin: FusedLinear, seed: int) -> torch.Tensor:
    """Concatenate per-module N(0, sigma_m) weights (CPU, bf16)."""
    parts = [weight_normal(m.width, lin.K, m.sigma, seed * 1000 + i) for i, m in enumerate(lin.modules)]
    return torch.cat(parts, 0)


def stack_layers():
    """The 496-linear stack at hidden 5120: 48 GDN layers and 16 attention
    layers, every input-sharing group fused into one GEMM (4 GEMMs a layer,
    256 in all).  Returns a list of (layer kind, [FusedLinear x 4])."""
    s = 0.02
    gdn = [
        FusedLinear("gdn_in_proj", HIDDEN, [Module("qkv", 8192, s), Module("z", 6144, s),
                                            Module("b", 48, s), Module("a", 48, s)]),
        FusedLinear("gdn_out", 6144, [Module("out", HIDDEN, s)]),
        FusedLinear("gate_up", HIDDEN, [Module("gate", MLP_WIDTH, s), Module("up", MLP_WIDTH, s)]),
        FusedLinear("down", MLP_WIDTH, [Module("down", HIDDEN, s)]),
    ]
    attn = [
        FusedLinear("attn_qkv", HIDDEN, [Module("q_gate", 12288, s), Module("k", 1024, s),
                                         Module("v", 1024, s)]),
        FusedLinear("attn_o", 6144, [Module("o", HIDDEN, s)]),
        FusedLinear("gate_up", HIDDEN, [Module("gate", MLP_WIDTH, s), Module("up", MLP_WIDTH, s)]),
        FusedLinear("down", MLP_WIDTH, [Module("down", HIDDEN, s)]),
    ]
    layers = []
    for i in range(64):
        # one attention layer after every three GDN layers (48 + 16 = 64)
        layers.append(("attention", attn) if i % 4 == 3 else ("gdn", gdn))
    return layers


def count_stack_linears() -> int:
    return sum(len(m.modules) for _, lin in stack_layers() for m in lin)
