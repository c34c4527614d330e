"""Seeded synthetic inputs for the Qift W2A4 linear path.

This module only draws random numbers; it holds none of the method's arithmetic (no rotation,
no quantization, no linear).  Both the CUDA path's tests/benchmarks and the CPU oracle take
their inputs from here, so the two sides see byte-identical data.

Shapes and value distributions stand in for the pages' workloads (LLaMA-2-7B and
LLaMA-3.1-8B linear modules; the Qift abstract studies all 224 linear modules of each model).
No trained weights or text data exist here, so:
  * weights are heavy-tailed Student-t(4) * 0.02 before rotation (the small single-linear
    case uses N(0, 0.02^2)), standing in for pretrained weights that are zero-centred but
    far from Gaussian until the Hadamard rotation;
  * activations are N(0, 1) cast to binary16, with a fixed set of outlier channels scaled by
    20 before the cast (channels drawn without replacement by the same generator).
Generator: numpy PCG64 via ``default_rng(seed)``; a second integer in the seed sequence
separates the matrices of one workload.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def weights(n_out: int, n_in: int, seed, dist: str = "t4", scale: float = 0.02) -> np.ndarray:
    """float32 [n_out, n_in]: ``standard_t(4) * scale`` or ``normal(0, scale)``."""
    rng = np.random.default_rng(seed)
    if dist == "t4":
        w = rng.standard_t(4, size=(n_out, n_in)) * scale
    elif dist == "normal":
        w = rng.normal(0.0, scale, size=(n_out, n_in))
    else:
        raise ValueError(dist)
    return w.astype(np.float32)


def activations(tokens: int, n_in: int, seed, n_outliers: int = 0, outlier_gain: float = 20.0) -> np.ndarray:
    """float16 [tokens, n_in]: N(0,1) with ``n_outliers`` fixed channels scaled before the cast."""
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 1.0, size=(tokens, n_in))
    if n_outliers:
        ch = rng.choice(n_in, size=n_outliers, replace=False)
        x[:, ch] *= outlier_gain
    return x.astype(np.float16)


def outlier_count(n_in: int, fraction: float = 0.01) -> int:
    return int(round(fraction * n_in))


@dataclass(frozen=True)
class Linear:
    """One linear module: W [n_out, n_in] applied to ``tokens`` activation rows."""
    name: str
    n_out: int
    n_in: int
    w_seed: tuple
    x_seed: tuple


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    levelset: str                 # "qift" | "pot" | "std" | "int4" (4-bit weights, W4A4)
    w_block: int                  # Hadamard block on the weights' input dimension
    a_block: int                  # Hadamard block on the activations (same as w_block)
    tokens: int
    out_dtype: str                # "f32" | "f16"
    w_dist: str
    n_outliers: int
    linears: tuple = field(default_factory=tuple)

    def w(self, lin: Linear) -> np.ndarray:
        return weights(lin.n_out, lin.n_in, lin.w_seed, self.w_dist)

    def x(self, lin: Linear, tokens: int | None = None) -> np.ndarray:
        t = self.tokens if tokens is None else tokens
        n_out = self.n_outliers if self.n_outliers >= 0 else outlier_count(lin.n_in)
        return activations(t, lin.n_in, lin.x_seed, n_out)


SINGLE_256x512 = Workload(
    name="single_linear_256x512",
    description="single linear out=256 in=512, 8 tokens, full 512-point Hadamard, Qift, fp32 out",
    levelset="qift", w_block=512, a_block=512, tokens=8, out_dtype="f32", w_dist="normal",
    n_outliers=4,
    linears=(Linear("linear", 256, 512, (0,), (0, 1)),),
)

LLAMA7B_QPROJ_DECODE = Workload(
    name="llama7b_q_proj_decode_T1",
    description="LLaMA-7B q_proj decode GEMV 4096x4096, 1 token, full 4096-point Hadamard, Qift",
    levelset="qift", w_block=4096, a_block=4096, tokens=1, out_dtype="f16", w_dist="t4",
    n_outliers=-1,
    linears=(Linear("q_proj", 4096, 4096, (2,), (102,)),),
)

LLAMA7B_MLP_PREFILL = Workload(
    name="llama7b_mlp_prefill_T2048",
    description="LLaMA-7B MLP prefill: gate/up 11008x4096, down 4096x11008, 2048 tokens, "
                "128-block Hadamard, Qift",
    levelset="qift", w_block=128, a_block=128, tokens=2048, out_dtype="f16", w_dist="t4",
    n_outliers=-1,
    linears=(Linear("gate_proj", 11008, 4096, (3, 0), (103, 0)),
             Linear("up_proj", 11008, 4096, (3, 1), (103, 0)),
             Linear("down_proj", 4096, 11008, (3, 2), (103, 2))),
)

LLAMA31_8B_MLP_DECODE16 = Workload(
    name="llama31_8b_mlp_decode_T16_pot",
    description="LLaMA-3.1-8B MLP decode at 16 tokens: up/gate 14336x4096, down 4096x14336, "
                "128-block Hadamard, power-of-two {+-1,+-4}",
    levelset="pot", w_block=128, a_block=128, tokens=16, out_dtype="f16", w_dist="t4",
    n_outliers=0,
    linears=(Linear("gate_proj", 14336, 4096, (4, 0), (104, 0)),
             Linear("up_proj", 14336, 4096, (4, 1), (104, 0)),
             Linear("down_proj", 4096, 14336, (4, 2), (104, 2))),
)

# The 4-bit layers of the mixed W2/W4 configuration, at the same decode shapes.
LLAMA7B_QPROJ_DECODE_W4 = Workload(
    name="llama7b_q_proj_decode_T1_w4",
    description="LLaMA-7B q_proj decode GEMV 4096x4096, 1 token, full 4096-point Hadamard, 4-bit weights (W4A4)",
    levelset="int4", w_block=4096, a_block=4096, tokens=1, out_dtype="f16", w_dist="t4",
    n_outliers=-1,
    linears=(Linear("q_proj", 4096, 4096, (2,), (102,)),),
)

LLAMA31_8B_MLP_DECODE16_W4 = Workload(
    name="llama31_8b_mlp_decode_T16_w4",
    description="LLaMA-3.1-8B MLP decode at 16 tokens: up/gate 14336x4096, down 4096x14336, "
                "128-block Hadamard, 4-bit weights (W4A4)",
    levelset="int4", w_block=128, a_block=128, tokens=16, out_dtype="f16", w_dist="t4",
    n_outliers=0,
    linears=(Linear("gate_proj", 14336, 4096, (4, 0), (104, 0)),
             Linear("up_proj", 14336, 4096, (4, 1), (104, 0)),
             Linear("down_proj", 4096, 14336, (4, 2), (104, 2))),
)

LLAMA7B_MLP_PREFILL_W4 = Workload(
    name="llama7b_mlp_prefill_T2048_w4",
    description="LLaMA-7B MLP prefill: gate/up 11008x4096, down 4096x11008, 2048 tokens, "
                "128-block Hadamard, 4-bit weights (W4A4)",
    levelset="int4", w_block=128, a_block=128, tokens=2048, out_dtype="f16", w_dist="t4",
    n_outliers=-1,
    linears=(Linear("gate_proj", 11008, 4096, (3, 0), (103, 0)),
             Linear("up_proj", 11008, 4096, (3, 1), (103, 0)),
             Linear("down_proj", 4096, 11008, (3, 2), (103, 2))),
)

WORKLOADS = {w.name: w for w in (SINGLE_256x512, LLAMA7B_QPROJ_DECODE, LLAMA7B_MLP_PREFILL,
                                 LLAMA31_8B_MLP_DECODE16, LLAMA7B_QPROJ_DECODE_W4, LLAMA31_8B_MLP_DECODE16_W4,
                                 LLAMA7B_MLP_PREFILL_W4)}

# Offline quantization of a full 8B-shaped model: 32 layers x 7 linear modules.
MODEL_8B_PROJS = (("q_proj", 4096, 4096), ("k_proj", 1024, 4096), ("v_proj", 1024, 4096),
                  ("o_proj", 4096, 4096), ("gate_proj", 14336, 4096), ("up_proj", 14336, 4096),
                  ("down_proj", 4096, 14336))
MODEL_8B_LAYERS = 32
MODEL_8B_BLOCK = 128


def weights_t4_device(n_out: int, n_in: int, seed: int, device, scale: float = 0.02):
    """float32 [n_out, n_in] Student-t(4) * scale drawn ON the device (torch Philox generator):
    t = z / sqrt(c / 4), z ~ N(0,1), c the sum of four squared N(0,1) draws.  Used where the
    host generator would be too slow (the 6.98 G weights of the 8B-shaped model)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    z = torch.randn(n_out, n_in, generator=g, device=device)
    c = torch.zeros(n_out, n_in, device=device)
    for _ in range(4):
        c.add_(torch.randn(n_out, n_in, generator=g, device=device).square_())
    return z.mul_(torch.rsqrt(c.mul_(0.25))).mul_(scale)


def model_8b_modules():
    """The 224 (layer, proj, n_out, n_in, seed) entries; seed = 1000 + 7*layer + proj index."""
    out = []
    for layer in range(MODEL_8B_LAYERS):
        for j, (name, n_out, n_in) in enumerate(MODEL_8B_PROJS):
            out.append((layer, name, n_out, n_in, 1000 + 7 * layer + j))
    return out
