"""Seeded synthetic inputs for the activation-sparse int4 GEMV.

This module only draws random tensors and picks thresholds; it holds none of
the arithmetic of the method (no quantization, selection or GEMV). Both the
CUDA path and the CPU oracle take their inputs from here, so neither ever
feeds the other.

Everything is generated on the CPU with a ``torch.Generator`` seeded per
tensor, then (by the caller) copied to the device. The pages evaluate trained
Llama-3 / Qwen3 models on benchmark text; no weights or datasets are used here:
the tensors below take those models' projection shapes and the value
distributions a decode step sees (weights ~ N(0, 0.02); activations Gaussian or
SiLU-gated, or ReLU-gated for the ReGLU FFN of the SVD-predictor page).
"""
from __future__ import annotations

import dataclasses
import math

import torch

# ---------------------------------------------------------------------------
# Shapes. (K = input channels, N = outputs; W is [N][K] like torch.nn.Linear.)
# ---------------------------------------------------------------------------

TINY = dict(N=512, K=256, group=64)                 # single small GEMV
LLAMA8B_DOWN = dict(N=4096, K=14336, group=128)     # Llama-3-8B FFN down_proj
LLAMA8B_LAYER = {                                   # every projection of one decode layer
    "q": dict(N=4096, K=4096, group=128),
    "k": dict(N=1024, K=4096, group=128),
    "v": dict(N=1024, K=4096, group=128),
    "o": dict(N=4096, K=4096, group=128),
    "gate": dict(N=14336, K=4096, group=128),
    "up": dict(N=14336, K=4096, group=128),
    "down": dict(N=4096, K=14336, group=128),
}
REGLU_FFN = dict(hidden=4096, inter=11008, group=128)
QWEN32B_FFN = dict(hidden=5120, inter=25600, group=128)
SPARSITY_SWEEP = (0.0, 0.3, 0.5, 0.7, 0.9)
QWEN_BATCHES = (1, 2, 4, 8, 16)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weight(N: int, K: int, seed: int, std: float = 0.02) -> torch.Tensor:
    """fp16 [N, K] with entries ~ N(0, std^2)."""
    return (torch.randn(N, K, generator=_gen(seed), dtype=torch.float32) * std).to(torch.float16)


def x_gaussian(B: int, K: int, seed: int) -> torch.Tensor:
    """bf16 [B, K] with entries ~ N(0, 1)."""
    return torch.randn(B, K, generator=_gen(seed), dtype=torch.float32).to(torch.bfloat16)


def x_silu_gated(B: int, K: int, seed: int) -> torch.Tensor:
    """bf16 [B, K] distributed like a SiLU-gated FFN hidden state: SiLU(g) * u
    with g, u ~ N(0, 1) drawn in fp32 (the input a down_proj sees)."""
    gen = _gen(seed)
    g = torch.randn(B, K, generator=gen, dtype=torch.float32)
    u = torch.randn(B, K, generator=gen, dtype=torch.float32)
    return (torch.nn.functional.silu(g) * u).to(torch.bfloat16)


def x_relu_shifted(B: int, K: int, seed: int, zero_frac: float = 0.88) -> torch.Tensor:
    """bf16 [B, K] stand-in for a trained ReGLU hidden state: ReLU(g - beta) * u
    with g, u ~ N(0, 1) and beta the normal quantile that leaves ``zero_frac``
    of the entries exactly zero (random weights alone give only ~50% zeros)."""
    gen = _gen(seed)
    g = torch.randn(B, K, generator=gen, dtype=torch.float32)
    u = torch.randn(B, K, generator=gen, dtype=torch.float32)
    beta = math.sqrt(2.0) * torch.special.erfinv(torch.tensor(2.0 * zero_frac - 1.0)).item()
    return (torch.relu(g - beta) * u).to(torch.bfloat16)


def percentile_threshold(x_row: torch.Tensor, sparsity: float) -> float:
    """Magnitude threshold t such that the active set {|x| > t} leaves out the
    ``round(sparsity * K)`` smallest |x| (ties in bf16 can leave out more).
    sparsity 0 gives t = -1 (every channel active)."""
    a = x_row.float().abs().flatten()
    m = int(round(sparsity * a.numel()))
    if m <= 0:
        return -1.0
    return float(torch.kthvalue(a, m).values.item())


@dataclasses.dataclass
class GemvCase:
    """One synthetic sparse-GEMV problem (CPU tensors)."""
    N: int
    K: int
    group: int
    W: torch.Tensor          # fp16 [N, K]
    x: torch.Tensor          # bf16 [B, K]
    t: list                  # B floats

    @property
    def B(self) -> int:
        return int(self.x.shape[0])


def gemv_case(N: int, K: int, group: int, B: int = 1, sparsity: float = 0.5,
              seed: int = 0, act: str = "gaussian") -> GemvCase:
    """Weights from ``seed``, activations from ``seed + 1``; one percentile
    threshold per batch row."""
    W = weight(N, K, seed)
    if act == "gaussian":
        x = x_gaussian(B, K, seed + 1)
    elif act == "silu":
        x = x_silu_gated(B, K, seed + 1)
    elif act == "relu_shifted":
        x = x_relu_shifted(B, K, seed + 1)
    else:
        raise ValueError(act)
    if act == "relu_shifted":
        t = [0.0] * B
    else:
        t = [percentile_threshold(x[b], sparsity) for b in range(B)]
    return GemvCase(N, K, group, W, x, t)


def bits(t: torch.Tensor):
    """uint16 numpy view of an fp16 / bf16 CPU tensor (the bit patterns)."""
    assert t.dtype in (torch.float16, torch.bfloat16)
    return t.contiguous().view(torch.int16).numpy().view("uint16")
