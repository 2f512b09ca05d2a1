"""Seeded synthetic workloads for the NF4-LoRA linear layer.

This module only draws random numbers and describes shapes.  It holds none of
the method's arithmetic (no quantisation, no codebook, no matrix products), so
that the CPU oracle and the CUDA path can both take their inputs from here
without sharing any of the computation they are compared on.

Recipe (every array is drawn on the host with numpy's PCG64 ``default_rng``):

* ``W``   fp32 ``[d_out, d_in]``, ``N(0, sigma)`` (sigma is a standard
  deviation), seed ``0 + module_index``.  Where a workload asks for heavy-tail
  outliers, 0.1 % of the entries, chosen uniformly without replacement with
  seed ``500 + module_index``, are multiplied by 10.
* ``A``   ``[r, d_in]``, ``N(0, 1/r)``, seed ``100 + module_index``.
* ``B``   ``[d_out, r]``, ``N(0, b_std)`` (0.01 by default), seed
  ``200 + module_index``.
* ``X``   ``[M, d_in]``, ``N(0, 1)``, seed ``300`` (``301`` for the wider input
  of a ``down`` projection).
* ``dY``  ``[M, d_out]``, ``N(0, 1)``, seed ``400 + module_index``.

``A``, ``B``, ``X`` and ``dY`` are drawn in fp32 and rounded to bfloat16 with
round-to-nearest-even (torch's conversion); ``W`` stays fp32 because it is the
input of the quantiser.

The workloads are LLaMA-shaped (7B: hidden 4096, MLP 11008; 65B: hidden 8192,
MLP 22016).  Only the shapes come from those models: no weights, datasets or
benchmark items are involved.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Tuple

import numpy as np
import torch


@dataclass(frozen=True)
class Module:
    name: str
    d_in: int
    d_out: int


@dataclass(frozen=True)
class Workload:
    name: str
    modules: Tuple[Module, ...]
    r: int
    alpha: float
    tokens: Tuple[int, ...]          # the M values (tokens per call)
    sigma: float = 0.02
    outliers: bool = False
    backward: str = "full"           # "full" (dX, dA, dB) or "dx" (dX only)
    quantize_timed: bool = False

    @property
    def scaling(self) -> float:
        return self.alpha / self.r


_L7 = (Module("q_proj", 4096, 4096), Module("k_proj", 4096, 4096),
       Module("v_proj", 4096, 4096), Module("o_proj", 4096, 4096),
       Module("gate_proj", 4096, 11008), Module("up_proj", 4096, 11008),
       Module("down_proj", 11008, 4096))
_L65 = (Module("q_proj", 8192, 8192), Module("k_proj", 8192, 8192),
        Module("v_proj", 8192, 8192), Module("o_proj", 8192, 8192),
        Module("gate_proj", 8192, 22016), Module("up_proj", 8192, 22016),
        Module("down_proj", 22016, 8192))

WORKLOADS = {
    # single 512x512 linear, quantize + fwd + bwd
    "linear512_r8_m16": Workload("linear512_r8_m16", (Module("linear", 512, 512),),
                                 r=8, alpha=16, tokens=(16,)),
    # LLaMA-7B q_proj, decode-like token counts, forward plus dX
    "q_proj4096_r64_m1-4-16": Workload("q_proj4096_r64_m1-4-16",
                                       (Module("q_proj", 4096, 4096),), r=64,
                                       alpha=16, tokens=(1, 4, 16), outliers=True,
                                       backward="dx"),
    # LLaMA-7B SwiGLU MLP linears, batch 2 x seq 2048
    "llama7b_mlp_r64_m4096": Workload("llama7b_mlp_r64_m4096", _L7[4:], r=64,
                                      alpha=16, tokens=(4096,)),
    # one LLaMA-7B decoder layer's seven linears, batch 4 x seq 2048
    "llama7b_layer_r16_m8192": Workload("llama7b_layer_r16_m8192", _L7, r=16,
                                        alpha=16, tokens=(8192,)),
    # LLaMA-65B layer linears, quantize timed, then fwd+bwd at 2048 tokens
    "llama65b_layer_r64_m2048": Workload("llama65b_layer_r64_m2048", _L65, r=64,
                                         alpha=16, tokens=(2048,), sigma=0.015,
                                         outliers=True, quantize_timed=True),
}


def weight(d_out: int, d_in: int, sigma: float = 0.02, outliers: bool = False,
           index: int = 0) -> np.ndarray:
    """fp32 ``[d_out, d_in]`` weight, ``N(0, sigma)`` with optional x10 outliers."""
    rng = np.random.default_rng(0 + index)
    w = rng.standard_normal((d_out, d_in), dtype=np.float32)
    w *= np.float32(sigma)
    if outliers:
        n = d_out * d_in
        k = max(1, n // 1000)
        pos = np.random.default_rng(500 + index).choice(n, size=k, replace=False)
        flat = w.reshape(-1)
        flat[pos] *= np.float32(10.0)
    return w


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


def lora_a(r: int, d_in: int, index: int = 0) -> torch.Tensor:
    rng = np.random.default_rng(100 + index)
    return _bf16(rng.standard_normal((r, d_in), dtype=np.float32) * np.float32(1.0 / r))


def lora_b(d_out: int, r: int, index: int = 0, std: float = 0.01) -> torch.Tensor:
    rng = np.random.default_rng(200 + index)
    return _bf16(rng.standard_normal((d_out, r), dtype=np.float32) * np.float32(std))


def activations(m: int, d_in: int, seed: int = 300) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    return _bf16(rng.standard_normal((m, d_in), dtype=np.float32))


def grad_output(m: int, d_out: int, index: int = 0) -> torch.Tensor:
    rng = np.random.default_rng(400 + index)
    return _bf16(rng.standard_normal((m, d_out), dtype=np.float32))


def x_seed(d_in: int, hidden: int) -> int:
    """Seed of the shared activation: 300 for the model width, 301 for wider inputs."""
    return 300 if d_in == hidden else 301


@dataclass
class LinearCase:
    """All host-side inputs of one adapted linear layer."""
    W: np.ndarray
    A: torch.Tensor
    B: torch.Tensor
    X: torch.Tensor
    dY: torch.Tensor
    r: int
    scaling: float


def linear_case(d_out: int, d_in: int, m: int, r: int, alpha: float, *,
                sigma: float = 0.02, outliers: bool = False, index: int = 0,
                b_std: float = 0.01, x_seed_value: int = 300) -> LinearCase:
    return LinearCase(W=weight(d_out, d_in, sigma, outliers, index),
                      A=lora_a(r, d_in, index), B=lora_b(d_out, r, index, b_std),
                      X=activations(m, d_in, x_seed_value),
                      dY=grad_output(m, d_out, index), r=r, scaling=alpha / r)


def special_blocks(rows: int = 16) -> np.ndarray:
    """A ``[rows, 256]`` fp32 matrix of hand-made 64-blocks that exercise the
    encoder's edge cases: an all-zero block, a constant block, a single-outlier
    block, a block of one sign, subnormal magnitudes and a ramp through zero.
    Remaining blocks are seeded ``N(0, 0.02)``."""
    rng = np.random.default_rng(7)
    w = rng.standard_normal((rows, 256), dtype=np.float32) * np.float32(0.02)
    blocks = w.reshape(-1, 64)
    blocks[0] = 0.0
    blocks[1] = np.float32(0.03125)
    blocks[2] = 0.0
    blocks[2, 17] = np.float32(-0.75)
    blocks[3] = np.abs(blocks[3])
    blocks[4] = -np.abs(blocks[4])
    blocks[5] = np.float32(1e-41) * np.arange(64, dtype=np.float32)
    blocks[6] = np.linspace(-1.0, 1.0, 64, dtype=np.float32)
    blocks[7, 5] = np.float32(3.0e4)
    return w
