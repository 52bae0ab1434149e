"""Pins of the block-level scoring oracle (oracle/block_oracle.py) against
things other than itself: closed forms of RMSNorm, SiLU and uniform
attention, the rotary embedding's relative-position property, causality, the
reduction of grouped-query attention to multi-head attention with repeated
heads, a scalar-loop brute force of a whole tiny block, and special cases of
the candidate losses (weights already on the int4 grid, an identity next
block).  No GPU needed."""
import math

import numpy as np
import pytest

from oracle import block_oracle as B
from oracle import w4_oracle as W4

TINY = {"hidden": 8, "heads": 2, "kv_heads": 1, "head_dim": 4, "ffn": 6, "eps": 1e-6,
        "rope_theta": 1e4}
SMALL = {"hidden": 128, "heads": 4, "kv_heads": 2, "head_dim": 32, "ffn": 256, "eps": 1e-6,
         "rope_theta": 1e6}  # linear widths multiples of the 128-channel group


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_bits(a):
    """bf16 patterns of float values (round to nearest even through float32)."""
    u = np.ascontiguousarray(np.asarray(a, np.float32)).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def _block(cfg, seed, std=0.1, zero=()):
    rng = _rng(seed)
    h, hq, hkv, d, f = cfg["hidden"], cfg["heads"], cfg["kv_heads"], cfg["head_dim"], cfg["ffn"]
    shapes = {"q": (hq * d, h), "k": (hkv * d, h), "v": (hkv * d, h), "o": (h, hq * d),
              "gate": (f, h), "up": (f, h), "down": (h, f)}
    bits = {n: _bf16_bits(np.zeros(sh) if n in zero else rng.normal(0, std, sh))
            for n, sh in shapes.items()}
    norms = {"ln1": 1 + 0.1 * rng.normal(size=h), "ln2": 1 + 0.1 * rng.normal(size=h),
             "q_norm": 1 + 0.1 * rng.normal(size=d), "k_norm": 1 + 0.1 * rng.normal(size=d)}
    return bits, norms


# ------------------------------------------------------------- pieces ----

def test_rms_norm_closed_form():
    x = np.full((2, 5), -3.0)
    g = np.arange(1.0, 6.0)
    y = B.rms_norm(x, g, 1e-6)
    assert np.allclose(y, -3.0 / math.sqrt(9.0 + 1e-6) * g, rtol=1e-15, atol=0)
    v = _rng(1).normal(size=(3, 7))
    assert np.allclose(B.rms_norm(5.0 * v, 1.0, 0.0), B.rms_norm(v, 1.0, 0.0), rtol=1e-13)


def test_silu_values():
    x = np.array([0.0, 1.0, -2.0, 40.0])
    y = B.silu(x)
    assert y[0] == 0.0
    assert y[1] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    assert y[2] == pytest.approx(-2.0 / (1.0 + math.exp(2.0)), rel=1e-15)
    assert y[3] == pytest.approx(40.0, rel=1e-15)


def test_rope_position_zero_norms_and_relative_property():
    rng = _rng(2)
    d, theta = 16, 1e4
    x = rng.normal(size=(6, 1, d))
    y = B.rope(x, theta)
    assert np.array_equal(y[0], x[0])  # position 0: no rotation
    half = d // 2
    pair = lambda a: a[..., :half] ** 2 + a[..., half:] ** 2
    assert np.allclose(pair(y), pair(x), rtol=1e-13)
    # <R_m q, R_n k> depends on m - n only: rotate (q at m, k at n) vs (q at m-n, k at 0)
    q = rng.normal(size=d)
    k = rng.normal(size=d)
    t = 6
    qs = B.rope(np.tile(q, (t, 1, 1)), theta)[:, 0]
    ks = B.rope(np.tile(k, (t, 1, 1)), theta)[:, 0]
    for m in range(t):
        for n in range(m + 1):
            assert qs[m] @ ks[n] == pytest.approx(qs[m - n] @ k, rel=1e-10, abs=1e-12)


def test_attention_zero_queries_average_the_prefix():
    rng = _rng(3)
    v = rng.normal(size=(5, 2, 3))
    k = rng.normal(size=(5, 2, 3))
    out = B.causal_attention(np.zeros((5, 4, 3)), k, v)
    for t in range(5):
        for h in range(4):
            assert np.allclose(out[t, h], v[: t + 1, h // 2].mean(axis=0), rtol=1e-14)


def test_attention_is_causal():
    rng = _rng(4)
    q, k, v = rng.normal(size=(6, 2, 4)), rng.normal(size=(6, 1, 4)), rng.normal(size=(6, 1, 4))
    a = B.causal_attention(q, k, v)
    k2, v2 = k.copy(), v.copy()
    k2[4:] += 5.0
    v2[4:] -= 3.0
    b = B.causal_attention(q, k2, v2)
    assert np.array_equal(a[:4], b[:4]) and not np.allclose(a[4:], b[4:])


def test_attention_brute_force_tiny():
    rng = _rng(5)
    t, hq, hkv, d = 4, 4, 2, 3
    q, k, v = rng.normal(size=(t, hq, d)), rng.normal(size=(t, hkv, d)), rng.normal(size=(t, hkv, d))
    out = B.causal_attention(q, k, v)
    for h in range(hq):
        kv = h // (hq // hkv)
        for i in range(t):
            scores = [sum(q[i, h, c] * k[j, kv, c] for c in range(d)) / math.sqrt(d)
                      for j in range(i + 1)]
            mx = max(scores)
            e = [math.exp(s - mx) for s in scores]
            z = sum(e)
            for c in range(d):
                ref = sum(e[j] * v[j, kv, c] for j in range(i + 1)) / z
                assert out[i, h, c] == pytest.approx(ref, rel=1e-12, abs=1e-14)


def test_gqa_equals_mha_with_repeated_heads():
    rng = _rng(6)
    q, k, v = rng.normal(size=(5, 4, 8)), rng.normal(size=(5, 2, 8)), rng.normal(size=(5, 2, 8))
    a = B.causal_attention(q, k, v)
    b = B.causal_attention(q, np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1))
    assert np.allclose(a, b, rtol=1e-15, atol=0)


# --------------------------------------------------------------- block ----

def _block_brute(x, w, cfg):
    """The tiny block with scalar loops (math module only)."""
    t_, hdim, hq, hkv, d, f, eps, th = (x.shape[0], cfg["hidden"], cfg["heads"], cfg["kv_heads"],
                                        cfg["head_dim"], cfg["ffn"], cfg["eps"], cfg["rope_theta"])

    def norm(vec, g):
        r = math.sqrt(sum(a * a for a in vec) / len(vec) + eps)
        return [vec[i] / r * g[i] for i in range(len(vec))]

    def mat(wm, vec):
        return [sum(wm[o][i] * vec[i] for i in range(len(vec))) for o in range(len(wm))]

    def rot(vec, pos):
        half = d // 2
        out = list(vec)
        for i in range(half):
            a = pos * th ** (-2.0 * i / d)
            out[i] = vec[i] * math.cos(a) - vec[i + half] * math.sin(a)
            out[i + half] = vec[i + half] * math.cos(a) + vec[i] * math.sin(a)
        return out

    wl = {n: w[n].tolist() for n in B.LINEARS}
    hs = [norm(list(x[p]), w["ln1"]) for p in range(t_)]
    qs, ks, vs = [], [], []
    for p in range(t_):
        qf, kf, vf = mat(wl["q"], hs[p]), mat(wl["k"], hs[p]), mat(wl["v"], hs[p])
        qs.append([rot(norm(qf[h * d:(h + 1) * d], w["q_norm"]), p) for h in range(hq)])
        ks.append([rot(norm(kf[h * d:(h + 1) * d], w["k_norm"]), p) for h in range(hkv)])
        vs.append([vf[h * d:(h + 1) * d] for h in range(hkv)])
    out = []
    for p in range(t_):
        att = []
        for h in range(hq):
            kv = h // (hq // hkv)
            sc = [sum(qs[p][h][c] * ks[j][kv][c] for c in range(d)) / math.sqrt(d)
                  for j in range(p + 1)]
            mx = max(sc)
            e = [math.exp(s - mx) for s in sc]
            att += [sum(e[j] * vs[j][kv][c] for j in range(p + 1)) / sum(e) for c in range(d)]
        x1 = [x[p][i] + v for i, v in enumerate(mat(wl["o"], att))]
        h2 = norm(x1, w["ln2"])
        g, u = mat(wl["gate"], h2), mat(wl["up"], h2)
        act = [g[i] / (1 + math.exp(-g[i])) * u[i] for i in range(f)]
        out.append([x1[i] + v for i, v in enumerate(mat(wl["down"], act))])
    return np.array(out)


def test_block_brute_force_tiny():
    bits, norms = _block(TINY, 7, std=0.3)
    w = B.block_weights_f64(bits, norms)
    x = _rng(8).normal(size=(3, TINY["hidden"]))
    assert np.allclose(B.block_forward(x, w, TINY), _block_brute(x, w, TINY), rtol=1e-12,
                       atol=1e-13)


def test_block_with_zero_linears_is_identity():
    bits, norms = _block(SMALL, 9, zero=B.LINEARS)
    x = _rng(10).normal(size=(5, SMALL["hidden"]))
    assert np.array_equal(B.block_forward(x, B.block_weights_f64(bits, norms), SMALL), x)


# ----------------------------------------------------------- scoring ----

def _on_grid_bits(n, k, seed):
    """A weight whose every 128-group already lies on the int4 grid with
    scale 2^-6 (codes 0 and 15 present, asymmetric zero 8)."""
    rng = _rng(seed)
    codes = rng.integers(0, 16, size=(n, k))
    codes[:, ::128] = 0
    codes[:, 1::128] = 15
    return _bf16_bits((codes - 8) * 2.0 ** -6)


def test_scoring_zero_loss_for_weights_on_the_grid():
    """alpha = 0 and shrink 1.0 is plain RTN, which reproduces weights
    already on the grid exactly: that candidate's loss is 0; others are not."""
    cfg = dict(SMALL, ffn=128)
    bits, norms = _block(cfg, 11, std=0.05)
    for name in B.GROUPS["gate_up"]:
        bits[name] = _on_grid_bits(128, 128, 12 if name == "gate" else 13)
    x = _rng(14).normal(size=(6, 128))
    al, sh = np.array([0.0, 0.5], np.float32), np.array([1.0, 0.8], np.float32)
    nxt = _block(cfg, 19, std=0.05)
    for next_block in (None, nxt):  # own output (d=0) and look-ahead through block i+1
        losses = B.scoring_losses(x, bits, norms, next_block, "gate_up", al, sh, False, cfg)
        assert losses[0, 0] == 0.0
        assert np.all(losses[:, 1] > 0) and losses[1, 0] > 0


def test_scoring_identity_next_block_equals_own_output():
    """A next block whose linears are zero is the identity, so the
    look-ahead loss equals the loss at block i's own output (d=0)."""
    bits, norms = _block(SMALL, 15)
    nxt = _block(SMALL, 16, zero=B.LINEARS)
    x = _rng(17).normal(size=(5, SMALL["hidden"]))
    al = np.array([0.0, 0.5], np.float32)
    sh = np.array([1.0, 0.7], np.float32)
    for group in ("qkv", "down"):
        own = B.scoring_losses(x, bits, norms, None, group, al, sh, False, SMALL)
        ahead = B.scoring_losses(x, bits, norms, nxt, group, al, sh, False, SMALL)
        assert np.array_equal(own, ahead)
        assert np.all(own > 0)


def test_scoring_candidate_is_the_scale_rewrite():
    """The swapped-in weight equals Q(W diag(s)) diag(1/s) of the linear's
    own oracle (the quantizer pinned in test_oracle_pins)."""
    bits, _ = _block(SMALL, 18)
    s = np.linspace(0.5, 2.0, SMALL["hidden"]).astype(np.float32)
    wc = B.candidate_linear(bits["up"], s, 0.9, True)
    codes, s16, z16 = W4.quantize_rtn(bits["up"], True, s, 0.9)
    assert np.array_equal(wc, W4.dequantize(codes, s16, z16).astype(np.float64) / s[None, :])


def test_search_picks_rtn_for_weights_on_the_grid():
    """Weights already on the int4 grid are reproduced exactly only by alpha 0
    at shrink 1.0, so the search must pick those for every group and linear,
    with or without a next block."""
    cfg = dict(SMALL, hidden=128, heads=4, kv_heads=2, head_dim=32, ffn=128)
    bits, norms = _block(cfg, 20, std=0.05)
    shapes = {"q": (128, 128), "k": (64, 128), "v": (64, 128), "o": (128, 128),
              "gate": (128, 128), "up": (128, 128), "down": (128, 128)}
    for i, name in enumerate(B.LINEARS):
        bits[name] = _on_grid_bits(*shapes[name], 30 + i)
    x = _rng(21).normal(size=(5, 128))
    al = np.array([0.0, 0.25, 0.5], np.float32)
    sh = np.array([0.9, 1.0, 0.8], np.float32)  # 1.0 not first: the index is checked
    for next_block in (None, _block(cfg, 22, std=0.05)):
        res = B.search_block(x, bits, norms, next_block, al, sh, False, cfg)
        assert set(res) == set(B.GROUPS)
        for group, (a_star, r_star) in res.items():
            assert a_star == 0, group
            assert set(r_star) == set(B.GROUPS[group])
            assert all(j == 1 for j in r_star.values()), (group, r_star)


def test_per_linear_shrink_touches_only_that_linear():
    """With `only`, the other linears of the group stay unclipped: a ratio on
    k alone gives the loss of the group with k clipped, which differs from
    clipping the whole group and, at ratio 1.0, equals no clipping."""
    bits, norms = _block(SMALL, 23)
    x = _rng(24).normal(size=(4, SMALL["hidden"]))
    al = np.array([0.5], np.float32)
    sh = np.array([1.0, 0.7], np.float32)
    whole = B.scoring_losses(x, bits, norms, None, "qkv", al, sh, False, SMALL)
    k_only = B.scoring_losses(x, bits, norms, None, "qkv", al, sh, False, SMALL, only="k")
    assert k_only[0, 0] == whole[0, 0]
    assert k_only[0, 1] != whole[0, 1]
