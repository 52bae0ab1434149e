"""Seeded synthetic inputs shaped like the models the model-card pages describe.

This module holds no arithmetic of the quantization method: it only draws
random weights and activations (torch CPU generators, fixed seeds) and lists
the workload shapes and the search grids.  Both the CUDA path and the CPU
oracle receive their inputs from here.

Stand-ins: the pages calibrate and evaluate on text datasets (an OpenR1
sample, WikiText-2, the Pile) and trained checkpoints, none of which exist in
this environment.  Seeded Gaussian weights and Gaussian / heavy-tailed
Student-t activations with the pages' model shapes stand in for them.
"""
from __future__ import annotations

import numpy as np
import torch

# --------------------------------------------------------------------------
# generators
# --------------------------------------------------------------------------


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_weight(n: int, k: int, std: float, seed: int, n_outliers: int = 0,
                  outlier_scale: float = 1.0) -> torch.Tensor:
    """bf16 [n, k] weight ~ N(0, std); ``n_outliers`` input channels chosen by
    a seeded permutation are multiplied by ``outlier_scale`` (before the bf16
    rounding)."""
    g = _gen(seed)
    w = torch.randn(n, k, generator=g, dtype=torch.float32) * std
    if n_outliers:
        ch = torch.randperm(k, generator=g)[:n_outliers]
        w[:, ch] *= outlier_scale
    return w.to(torch.bfloat16)


def normal_activations(m: int, k: int, seed: int, std: float = 1.0) -> torch.Tensor:
    """bf16 [m, k] activations ~ N(0, std)."""
    g = _gen(seed)
    return (torch.randn(m, k, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)


def student_t_calibration(m: int, k: int, seed: int, nu: int = 3) -> torch.Tensor:
    """bf16 [m, k] heavy-tailed calibration activations: x_mj = c_j * z_mj with
    per-channel magnitude c_j = |t_nu| and z ~ N(0, 1).  t_nu is drawn from its
    textbook definition z0 / sqrt(chi2_nu / nu), chi2_nu a sum of nu squared
    standard normals."""
    g = _gen(seed)
    z0 = torch.randn(k, generator=g, dtype=torch.float64)
    chi2 = (torch.randn(nu, k, generator=g, dtype=torch.float64) ** 2).sum(0)
    c = (z0 / torch.sqrt(chi2 / nu)).abs()
    z = torch.randn(m, k, generator=g, dtype=torch.float32)
    return (z * c.to(torch.float32)[None, :]).to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 CPU tensor (the oracle's input format)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------
# search grids (inputs of the AWQ scoring call)
# --------------------------------------------------------------------------


def alpha_grid(n: int = 20) -> np.ndarray:
    """alpha_i = i / n, i = 0..n-1 (0 -> 0.95 for n = 20), float32."""
    return np.array([i / n for i in range(n)], dtype=np.float32)


def shrink_grid(n: int = 10, step: float = 0.05) -> np.ndarray:
    """r_j = 1 - step * j, j = 0..n-1 (1.0 -> 0.55 for n = 10), float32."""
    return np.array([round(1.0 - step * j, 6) for j in range(n)], dtype=np.float32)


# --------------------------------------------------------------------------
# workload shapes
# --------------------------------------------------------------------------

# One Qwen3-1.7B decoder block (hidden 2048, 16 query heads and 8 KV heads of
# width 128, SwiGLU width 6144, 28 blocks): (name, K in, N out).
QWEN3_1P7B_BLOCK = (
    ("q_proj", 2048, 2048),
    ("k_proj", 2048, 1024),
    ("v_proj", 2048, 1024),
    ("o_proj", 2048, 2048),
    ("gate_proj", 2048, 6144),
    ("up_proj", 2048, 6144),
    ("down_proj", 6144, 2048),
)
QWEN3_1P7B_BLOCKS = 28

# Llama-2-7B-shaped linears (K, N, count).
LLAMA2_7B_LINEARS = ((4096, 4096, 4), (4096, 11008, 2), (11008, 4096, 1))

# 27B-scale linears (K, N).
SCALE27B_LINEARS = ((5120, 17408), (17408, 5120), (5120, 10240))


def qwen_block_weights(block: int, seed_base: int = 1000):
    """The seven bf16 weights of one Qwen3-1.7B-shaped block, N(0, 0.02)."""
    out = []
    for i, (name, k, n) in enumerate(QWEN3_1P7B_BLOCK):
        out.append((name, normal_weight(n, k, 0.02, seed_base + 7 * block + i)))
    return out


# Linear names of one decoder block in the block-level scoring's order.
BLOCK_LINEAR_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def qwen_block(block: int, seed_base: int = 1000, std: float = 0.02):
    """One Qwen3-1.7B-shaped decoder block for the block-level scoring: the
    seven bf16 linears (N(0, std), keyed "q" .. "down", [out, in]) and the
    float64 norm gains "ln1", "ln2" [2048] and "q_norm", "k_norm" [128], each
    1 + 0.1 N(0, 1)."""
    out = {}
    for i, (name, k, n) in enumerate(QWEN3_1P7B_BLOCK):
        out[BLOCK_LINEAR_NAMES[i]] = normal_weight(n, k, std, seed_base + 7 * block + i)
    g = _gen(seed_base + 7 * block + 1000)
    for name, width in (("ln1", 2048), ("ln2", 2048), ("q_norm", 128), ("k_norm", 128)):
        out[name] = 1.0 + 0.1 * torch.randn(width, generator=g, dtype=torch.float64)
    return out


def block_input(t: int, hidden: int, seed: int, std: float = 1.0) -> torch.Tensor:
    """float64 [t, hidden] hidden states entering a block ~ N(0, std)."""
    g = _gen(seed)
    return torch.randn(t, hidden, generator=g, dtype=torch.float64) * std


def block_of_shape(cfg: dict, seed: int, std: float = 0.05, n_outliers: int = 0,
                   outlier_scale: float = 1.0):
    """A decoder block of any shape (cfg: hidden, heads, kv_heads, head_dim,
    ffn) for the block-level scoring: bf16 linears N(0, std) keyed "q" ..
    "down" ([out, in]), each with n_outliers input channels scaled by
    outlier_scale (normal_weight), and float64 gains 1 + 0.1 N(0, 1)."""
    h, hq, hkv, d, f = cfg["hidden"], cfg["heads"], cfg["kv_heads"], cfg["head_dim"], cfg["ffn"]
    shapes = {"q": (hq * d, h), "k": (hkv * d, h), "v": (hkv * d, h), "o": (h, hq * d),
              "gate": (f, h), "up": (f, h), "down": (h, f)}
    out = {}
    for i, name in enumerate(BLOCK_LINEAR_NAMES):
        n, k = shapes[name]
        out[name] = normal_weight(n, k, std, seed + i, n_outliers, outlier_scale)
    g = _gen(seed + 100)
    for name, width in (("ln1", h), ("ln2", h), ("q_norm", d), ("k_norm", d)):
        out[name] = 1.0 + 0.1 * torch.randn(width, generator=g, dtype=torch.float64)
    return out
