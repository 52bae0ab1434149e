"""CPU oracle for block-level AWQ candidate scoring: the look-ahead loss of
the "ghostchoir/rebuttal_w4g128_awq_w2" card and its block-output arm.

TEST INFRASTRUCTURE ONLY, like w4_oracle: nothing on the product path may
import it; it shares no code with the CUDA library.

Sources (cited by page title and section):
  [rebuttal] "ghostchoir/rebuttal_w4g128_awq_w2" model card: the 'Model
      Details' table (base model Qwen/Qwen3-1.7B, BF16, 28 blocks, hidden
      2048; row 'Search': AWQ scale exponent on a 20-point grid and a
      10-point global shrink grid, look-ahead scored); the paragraph under it
      (a candidate for block i is scored at the output of block i+1, which
      stays in original precision; the reference is the same path with block
      i unquantized; block 27 has no successor and falls back to its own
      output); the scale-rewrite paragraph (a candidate swaps only the
      linear's weight); the perplexity table's d=0 row (block-wise, the loss
      at block i's own output).
  [q326] "ariacompute/qwen3-1.7b_q326_channel" page: the Qwen3-1.7B shapes
      (16 query heads, 8 key/value heads of width 128, SwiGLU width 6144).

Readings where the pages are silent (the decoder block itself is not on
the pages; these are the published Qwen3 conventions):
  * pre-norm block: h = RMSNorm(x); attention; x1 = x + o_proj(attn);
    h2 = RMSNorm(x1); x2 = x1 + down(SiLU(gate(h2)) * up(h2));
  * RMSNorm(v) = v / sqrt(mean(v^2) + eps) * gamma, eps = 1e-6, also applied
    per head to q and k before the rotary embedding (Qwen3's q/k norms);
  * rotary embedding, rotate-half convention: for i < d/2 the pair
    (x_i, x_{i+d/2}) at position p turns by p * theta^(-2i/d), theta = 1e6;
  * causal softmax attention with scale 1/sqrt(d); query head h reads
    key/value head h // (heads / kv_heads);
  * the AWQ statistic of a linear group is the mean |input| over tokens of
    the activation entering that group in the unquantized forward: the norm
    output for q, k, v (shared), the attention output for o, the second norm
    output for gate, up (shared), the SwiGLU product for down;
  * loss = mean over tokens and hidden units of (candidate path - reference
    path)^2; everything in binary64 here (the pages fix no precision);
  * the search: alpha per linear group at no clipping, then one shrink ratio
    per linear with the rest of the group unclipped, each group scored with
    the rest of block i unquantized; the caller supplies block i's input.
"""
from __future__ import annotations

import numpy as np

from oracle import w4_oracle as W4

QWEN3_1P7B = {"hidden": 2048, "heads": 16, "kv_heads": 8, "head_dim": 128, "ffn": 6144,
              "eps": 1e-6, "rope_theta": 1e6}

LINEARS = ("q", "k", "v", "o", "gate", "up", "down")
GROUPS = {"qkv": ("q", "k", "v"), "o": ("o",), "gate_up": ("gate", "up"), "down": ("down",)}


def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2 over the last axis) + eps) * gamma."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * gamma


def rope(x: np.ndarray, theta: float) -> np.ndarray:
    """Rotary embedding of x [T, heads, d] at positions 0..T-1 (rotate half)."""
    t, _, d = x.shape
    half = d // 2
    inv = theta ** (-2.0 * np.arange(half) / d)
    ang = np.arange(t, dtype=np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(d), causal) v per query head; q [T, H, d], k and v
    [T, Hkv, d]; query head h reads key/value head h // (H / Hkv)."""
    t, h_q, d = q.shape
    group = h_q // k.shape[1]
    out = np.empty_like(q)
    mask = np.triu(np.ones((t, t), dtype=bool), 1)
    for h in range(h_q):
        s = q[:, h] @ k[:, h // group].T / np.sqrt(d)
        s[mask] = -np.inf
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h] = p @ v[:, h // group]
    return out


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def block_forward(x: np.ndarray, w: dict, cfg: dict, inputs: dict | None = None) -> np.ndarray:
    """One decoder block on x [T, hidden] (binary64).  w holds binary64
    matrices "q", "k", "v" [heads*d or kv_heads*d, hidden], "o" [hidden,
    heads*d], "gate", "up" [ffn, hidden], "down" [hidden, ffn] and the norm
    gains "ln1", "ln2" [hidden], "q_norm", "k_norm" [d].  If `inputs` is a
    dict it receives the activation entering each linear group."""
    t = x.shape[0]
    hq, hkv, d, eps = cfg["heads"], cfg["kv_heads"], cfg["head_dim"], cfg["eps"]
    h = rms_norm(x, w["ln1"], eps)
    q = rms_norm((h @ w["q"].T).reshape(t, hq, d), w["q_norm"], eps)
    k = rms_norm((h @ w["k"].T).reshape(t, hkv, d), w["k_norm"], eps)
    v = (h @ w["v"].T).reshape(t, hkv, d)
    a = causal_attention(rope(q, cfg["rope_theta"]), rope(k, cfg["rope_theta"]), v)
    a = a.reshape(t, hq * d)
    x1 = x + a @ w["o"].T
    h2 = rms_norm(x1, w["ln2"], eps)
    act = silu(h2 @ w["gate"].T) * (h2 @ w["up"].T)
    if inputs is not None:
        inputs.update(qkv=h, o=a, gate_up=h2, down=act)
    return x1 + act @ w["down"].T


def block_weights_f64(bits: dict, norms: dict) -> dict:
    """Binary64 block weights from bf16 bit patterns of the linears and
    binary64 norm gains."""
    out = {name: W4.bf16_bits_to_f32(bits[name]).astype(np.float64) for name in LINEARS}
    out.update(norms)
    return out


def candidate_linear(w_bits: np.ndarray, s: np.ndarray, shrink: float, symmetric: bool):
    """Q_r(W diag(s)) diag(1/s) in binary64: the weight a candidate swaps in
    ([rebuttal] scale-rewrite paragraph)."""
    codes, s16, z16 = W4.quantize_rtn(w_bits, symmetric, s, shrink)
    return W4.dequantize(codes, s16, z16).astype(np.float64) / np.asarray(s, np.float64)[None, :]


def scoring_losses(x: np.ndarray, bits_i: dict, norms_i: dict, next_block, group: str,
                   alphas, shrinks, symmetric: bool, cfg: dict, only: str | None = None
                   ) -> np.ndarray:
    """loss[a, r] for every (alpha_a, shrink_r) candidate of one linear group
    of block i ([rebuttal] 'Search' row; look-ahead paragraph).

    x: block i's input [T, hidden] (binary64).  next_block: (bits, norms) of
    block i+1 for the look-ahead loss at its output, or None for the loss at
    block i's own output (the d=0 arm, and block 27's fallback).  Every
    linear of the group takes the same alpha; the shrink goes to every
    linear of the group, or with `only` to that linear alone (the others
    unclipped)."""
    w_ref = block_weights_f64(bits_i, norms_i)
    acts: dict = {}
    out_i = block_forward(x, w_ref, cfg, acts)
    w_next = None if next_block is None else block_weights_f64(*next_block)

    def path(w_block):
        y = block_forward(x, w_block, cfg)
        return y if w_next is None else block_forward(y, w_next, cfg)

    ref = out_i if w_next is None else block_forward(out_i, w_next, cfg)
    stat = np.mean(np.abs(acts[group]), axis=0)
    s_all = W4.awq_scales(stat, alphas)
    losses = np.empty((len(alphas), len(shrinks)), dtype=np.float64)
    for a in range(len(alphas)):
        for j, r in enumerate(shrinks):
            wc = dict(w_ref)
            for name in GROUPS[group]:
                ratio = float(r) if only is None or name == only else 1.0
                wc[name] = candidate_linear(bits_i[name], s_all[a], ratio, symmetric)
            diff = path(wc) - ref
            losses[a, j] = np.mean(diff * diff)
    return losses


def search_block(x: np.ndarray, bits_i: dict, norms_i: dict, next_block, alphas, shrinks,
                 symmetric: bool, cfg: dict) -> dict:
    """The search of one block ([rebuttal] 'Search' row, 'Clipping
    granularity'): for each linear group, alpha* = the least loss over the
    alpha grid at no clipping (shrink 1.0); then for each linear of the group
    its own ratio r* = the least loss over the shrink grid with the group at
    alpha* and the group's other linears unclipped.  Groups are scored one at
    a time with the rest of block i unquantized (a candidate swaps only its
    own weights).  Ties go to the lowest grid index.  Returns {group:
    (alpha index, {linear: shrink index})}."""
    one = np.array([1.0], np.float32)
    out = {}
    for group, names in GROUPS.items():
        col = scoring_losses(x, bits_i, norms_i, next_block, group, alphas, one, symmetric, cfg)
        a_star = int(np.argmin(col[:, 0]))
        al = np.asarray(alphas, np.float32)[a_star:a_star + 1]
        r_star = {}
        for name in names:
            row = scoring_losses(x, bits_i, norms_i, next_block, group, al, shrinks, symmetric,
                                 cfg, only=name)
            r_star[name] = int(np.argmin(row[0]))
        out[group] = (a_star, r_star)
    return out
