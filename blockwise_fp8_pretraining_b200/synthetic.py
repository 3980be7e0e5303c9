"""Seeded synthetic inputs shaped like the Qwen3-1.7B linear layers.

This module only draws random tensors; it holds none of the quantization or
GEMM arithmetic, so the CUDA path and the CPU oracle can both be fed from it
without sharing any of the method's code.

Shapes follow the Puro-2B model cards (property table: hidden size 2048,
16 query / 8 key-value heads of dimension 128, feed-forward size 6144,
28 layers; setting table: sequence length 4096, micro-batch 2, so 8192
tokens per micro-batch).  Per layer the four linear weights are

    qkv      [4096, 2048]   (16 q heads + 8 k heads + 8 v heads, 128 rows each)
    o_proj   [2048, 2048]
    gate_up  [12288, 2048]  (gate rows 0..6143, up rows 6144..12287)
    down     [2048, 6144]

Value recipe (drawn in float32, then rounded to bf16 round-to-nearest-even):
  * activations ~ N(0, 1), with a set of outlier input channels (the same
    columns for every row, picked by a seeded permutation) multiplied by a
    factor before rounding;
  * weights ~ N(0, 0.02);
  * output gradients ~ N(0, 1e-3);
  * heavy-tailed activations: Student-t with nu = 3 and a seeded 0.1% of
    positions multiplied by 1e3.
The second parameter of N(., .) is the standard deviation.
"""
from __future__ import annotations

import math

import numpy as np
import torch

TOKENS = 8192          # 2 sequences x 4096 tokens
HIDDEN = 2048
FFN = 6144
QKV_OUT = 4096         # (16 q + 8 k + 8 v) heads x 128, fused
LAYERS = 28

# (name, out_features N, in_features K) of the four linears of one layer.
LAYER_LINEARS = (
    ("qkv", QKV_OUT, HIDDEN),
    ("o_proj", HIDDEN, HIDDEN),
    ("gate_up", 2 * FFN, HIDDEN),
    ("down", HIDDEN, FFN),
)


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, gen: torch.Generator, device="cpu") -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    return (x * std).to(torch.bfloat16)


def activation_bf16(rows: int, cols: int, n_outliers: int, factor: float,
                    gen: torch.Generator, device="cpu") -> torch.Tensor:
    """N(0,1) activations with n_outliers whole input channels scaled."""
    x = torch.randn((rows, cols), generator=gen, dtype=torch.float32, device=device)
    if n_outliers > 0:
        idx = torch.randperm(cols, generator=gen, device=device)[:n_outliers]
        x[:, idx] *= factor
    return x.to(torch.bfloat16)


def outlier_channels(cols: int, fraction: float = 0.01) -> int:
    """Number of outlier channels for a fraction of the input width."""
    return int(math.floor(fraction * cols))


def student_t_bf16(shape, seed: int, nu: float = 3.0, outlier_fraction: float = 1e-3,
                   outlier_scale: float = 1e3) -> torch.Tensor:
    """Heavy-tailed activations: Student-t(nu) with a seeded fraction of the
    positions multiplied by outlier_scale (float32, then bf16)."""
    rng = np.random.default_rng(int(seed))
    x = rng.standard_t(nu, size=shape).astype(np.float32)
    n = x.size
    k = int(round(outlier_fraction * n))
    if k:
        pos = rng.choice(n, size=k, replace=False)
        x.reshape(-1)[pos] *= np.float32(outlier_scale)
    return torch.from_numpy(x).to(torch.bfloat16)


# ------------------------------------------------------------- configurations

def tiny(seed: int = 0, device="cpu") -> dict:
    """Tiny fprop + backward: X [256, 2048] with 4 channels x50,
    W [2048, 2048] ~ N(0, 0.02), dY [256, 2048] ~ N(0, 1e-3)."""
    g = generator(seed, device)
    x = activation_bf16(256, HIDDEN, 4, 50.0, g, device)
    w = normal_bf16((HIDDEN, HIDDEN), 0.02, g, device)
    dy = normal_bf16((256, HIDDEN), 1e-3, g, device)
    return {"x": x, "w": w, "dy": dy}


def attention_projections(seed: int = 0, device="cpu", tokens: int = TOKENS) -> dict:
    """One micro-batch of the attention projections: X [tokens, 2048] with
    1% outlier channels x30, fused QKV W [4096, 2048], o_proj W [2048, 2048]."""
    g = generator(seed, device)
    x = activation_bf16(tokens, HIDDEN, outlier_channels(HIDDEN), 30.0, g, device)
    w_qkv = normal_bf16((QKV_OUT, HIDDEN), 0.02, g, device)
    w_o = normal_bf16((HIDDEN, HIDDEN), 0.02, g, device)
    return {"x": x, "w_qkv": w_qkv, "w_o": w_o}


def mlp(seed: int = 0, device="cpu", tokens: int = TOKENS) -> dict:
    """SwiGLU MLP weights and input: X [tokens, 2048] (1% channels x30),
    gate_up W [12288, 2048], down W [2048, 6144].  The down-projection input
    H = silu(gate) * up is derived by the caller from a gate_up output."""
    g = generator(seed, device)
    x = activation_bf16(tokens, HIDDEN, outlier_channels(HIDDEN), 30.0, g, device)
    w_gu = normal_bf16((2 * FFN, HIDDEN), 0.02, g, device)
    w_down = normal_bf16((HIDDEN, FFN), 0.02, g, device)
    return {"x": x, "w_gate_up": w_gu, "w_down": w_down}


def output_grads(shapes, seed: int = 0, device="cpu") -> list:
    """Output gradients ~ N(0, 1e-3) for each (rows, cols) in shapes."""
    g = generator(seed, device)
    return [normal_bf16(s, 1e-3, g, device) for s in shapes]


def layer(seed: int, device="cpu", tokens: int = TOKENS, gen: torch.Generator | None = None) -> dict:
    """Every tensor one layer's four linears need for fprop, dgrad and
    wgrad: per linear an input activation [tokens, K] (1% channels x30 for
    the hidden-size inputs), a weight [N, K] ~ N(0, 0.02) and an output
    gradient [tokens, N] ~ N(0, 1e-3).  The down projection's input is drawn
    here as silu(g) * u of two N(0, 1) tensors rounded through bf16, the
    same shape and distribution family as a gate_up output passed through
    SwiGLU."""
    g = gen if gen is not None else generator(seed, device)
    out = {}
    for name, n, k in LAYER_LINEARS:
        if name == "down":
            gate = torch.randn((tokens, k), generator=g, device=device).to(torch.bfloat16)
            up = torch.randn((tokens, k), generator=g, device=device).to(torch.bfloat16)
            x = (torch.nn.functional.silu(gate.float()).to(torch.bfloat16).float()
                 * up.float()).to(torch.bfloat16)
        else:
            x = activation_bf16(tokens, k, outlier_channels(k), 30.0, g, device)
        out[name] = {
            "x": x,
            "w": normal_bf16((n, k), 0.02, g, device),
            "dy": normal_bf16((tokens, n), 1e-3, g, device),
        }
    return out


def swiglu_bf16(gate_up: torch.Tensor) -> torch.Tensor:
    """H = silu(gate) * up in bf16 torch ops, gate = first half of the
    columns of a gate_up output, up = second half.  This prepares the
    down-projection input that both sides receive; torch's float32 silu is
    not correctly rounded to bf16 on every input, so it is not the definition
    a fused producer of H is held to."""
    half = gate_up.shape[1] // 2
    gate = gate_up[:, :half]
    up = gate_up[:, half:]
    return (torch.nn.functional.silu(gate.float()).to(torch.bfloat16).float()
            * up.float()).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (CPU copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
