"""Pins of the CPU oracle against things other than itself: hand-derived
closed forms (tests/golden), the binary16 format definition, exact rational
brute force on tiny inputs, invariants the pages state, and an independent
float16 implementation (numpy's).  No GPU needed.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import w4_oracle as O
from weight_only_int4_quantize_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_bits_to_bf16_exact(a):
    """bf16 bit patterns of float32 values that are exactly representable."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = a.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exact in bfloat16"
    return (u >> 16).astype(np.uint16)


# ---------------------------------------------------------------- fp16 -----

def _fp16_cases():
    out = []
    with open(os.path.join(GOLDEN, "fp16_rne.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            expr, hexbits = line.split()
            out.append((expr, int(hexbits, 16)))
    return out


@pytest.mark.parametrize("expr,expected", _fp16_cases())
def test_fp16_rne_golden(expr, expected):
    v = np.float32(eval(expr, {"__builtins__": {}}))
    got = int(O.f32_to_f16_bits(np.array([v]))[0])
    assert got == expected, f"{expr}: got {got:#06x} want {expected:#06x}"


def test_fp16_widening_matches_definition_all_patterns():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    e = (h >> 10) & 0x1F
    finite = e != 31
    got = O.f16_bits_to_f32(h[finite])
    ref = h[finite].view(np.float16).astype(np.float32)  # independent implementation
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    # rounding a binary16 value back is the identity
    assert np.array_equal(O.f32_to_f16_bits(got), h[finite])


def test_fp16_rounding_matches_numpy_on_structured_sample():
    rng = np.random.default_rng(7)
    exps = np.arange(90, 160, dtype=np.uint32)       # 2^-37 .. 2^32
    mant = rng.integers(0, 1 << 23, size=4000, dtype=np.uint32)
    # plus mantissas sitting exactly on / next to binary16 ties
    tie = np.array([0x1000, 0x0FFF, 0x1001, 0x3000, 0x2FFF, 0x3001, 0x7FF000, 0x7FFFFF], np.uint32)
    mant = np.concatenate([mant, tie, (mant[:500] & ~np.uint32(0x1FFF)) | 0x1000])
    u = (exps[:, None] << 23) | mant[None, :]
    u = np.concatenate([u.ravel(), u.ravel() | (1 << 31)])
    x = u.view(np.float32)
    got = O.f32_to_f16_bits(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------- quantizer -----

def _golden_cases():
    with open(os.path.join(GOLDEN, "rtn_groups.json")) as f:
        return json.load(f)["cases"]


def _case_inputs(case):
    vals = np.array([float(Fraction(v)) for v in case["values"]] * 8, dtype=np.float32)
    w = f32_bits_to_bf16_exact(vals)[None, :]
    s = None
    if case["s"] == "2":
        s = np.full(128, 2.0, np.float32)
    elif case["s"] == "alt12":
        s = np.where(np.arange(128) % 2 == 0, 1.0, 2.0).astype(np.float32)
    return w, s


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_rtn_golden_groups(case):
    w, s = _case_inputs(case)
    codes, s16, z16 = O.quantize_rtn(w, case["symmetric"], s, case["shrink"])
    assert list(codes[0, :16]) == case["codes"]
    assert np.array_equal(codes[0], np.tile(codes[0, :16], 8))
    assert int(s16[0, 0]) == int(case["scale16"], 16)
    if case["zero16"] is None:
        assert z16 is None
    else:
        assert int(z16[0, 0]) == int(case["zero16"], 16)


def test_pack_layout_little_endian_nibbles():
    codes = np.zeros((2, 128), np.uint8)
    codes[0, :8] = [1, 2, 3, 4, 5, 6, 7, 8]
    codes[1, 8:16] = [15, 0, 0, 0, 0, 0, 0, 9]
    # (channel 8 in nibble 0, channel 15 in nibble 7)
    q = O.pack_codes(codes).view(np.uint32)
    assert q.shape == (2, 16)
    # nibbles low->high hold channels 0,2,4,6,1,3,5,7 of the word
    assert q[0, 0] == 0x86427531 and q[0, 1] == 0
    assert q[1, 1] == 0x9000000F
    # nibble pair (i, i+4) masked with 0x000F000F gives channels (2i, 2i+1)
    codes[0, 16:24] = [1, 2, 3, 4, 5, 6, 7, 8]
    w = int(O.pack_codes(codes).view(np.uint32)[0, 2])
    for i in range(4):
        pair = (w >> (4 * i)) & 0x000F000F
        assert (pair & 0xF, pair >> 16) == (2 * i + 1, 2 * i + 2)
    rng = np.random.default_rng(1)
    c = rng.integers(0, 16, size=(5, 256), dtype=np.uint8)
    assert np.array_equal(O.unpack_codes(O.pack_codes(c)), c)


@pytest.mark.parametrize("symmetric", [False, True])
@pytest.mark.parametrize("shrink", [1.0, 0.8, 0.55])
@pytest.mark.parametrize("with_s", [False, True])
def test_quantizer_invariants(symmetric, shrink, with_s):
    w = synth.bits(synth.normal_weight(64, 1024, 0.02, seed=3, n_outliers=8, outlier_scale=20.0))
    s = None
    if with_s:
        x = synth.bits(synth.student_t_calibration(64, 1024, seed=4))
        s = O.awq_scales(O.awq_channel_stat(x), [0.5])[0]
    codes, s16, z16 = O.quantize_rtn(w, symmetric, s, shrink)
    assert codes.min() >= 0 and codes.max() <= 15
    sc = O.f16_bits_to_f32(s16)
    z = np.full(sc.shape, 8.0) if symmetric else O.f16_bits_to_f32(z16).astype(np.float64)
    assert np.all(z == np.round(z)) and z.min() >= 0 and z.max() <= 15
    v = O.bf16_bits_to_f32(w).astype(np.float64)
    if s is not None:
        v = (O.bf16_bits_to_f32(w) * s[None, :]).astype(np.float64)
    vg = v.reshape(64, 8, 128)
    what = O.dequantize(codes, s16, z16).reshape(64, 8, 128).astype(np.float64)
    t = vg / sc[:, :, None] + z[:, :, None]
    inside = (t >= 0) & (t <= 15)
    err = np.abs(vg - what)
    assert np.all(err[inside] <= 0.5 * np.broadcast_to(sc[:, :, None], err.shape)[inside] * (1 + 1e-6))


def _nearest_even_code(v: Fraction, sc: Fraction, z: int) -> int:
    """Brute force: the code q in 0..15 whose grid point (q - z) * sc is
    nearest to v; on an exact tie the one with even (q - z)."""
    best = None
    for q in range(16):
        d = abs(v - (q - z) * sc)
        key = (d, (q - z) % 2)
        if best is None or key < best[0]:
            best = (key, q)
    return best[1]


@pytest.mark.parametrize("symmetric", [False, True])
@pytest.mark.parametrize("shrink", [1.0, 0.7])
def test_codes_brute_force_nearest_grid_point(symmetric, shrink):
    rng = np.random.default_rng(11)
    vals = (rng.standard_normal((4, 256)) * 0.05).astype(np.float32)
    w = f32_bits_to_bf16_exact((vals.view(np.uint32) & 0xFFFF0000).view(np.float32))
    codes, s16, z16 = O.quantize_rtn(w, symmetric, None, shrink)
    sc = O.f16_bits_to_f32(s16)
    v = O.bf16_bits_to_f32(w)
    for n in range(4):
        for k in range(256):
            g = k // 128
            z = 8 if symmetric else int(O.f16_bits_to_f32(z16)[n, g])
            want = _nearest_even_code(Fraction(float(v[n, k])), Fraction(float(sc[n, g])), z)
            assert codes[n, k] == want, (n, k)


def test_zero_point_brute_force():
    """zero = the integer in 0..15 nearest to -min'/scale (ties even)."""
    rng = np.random.default_rng(12)
    vals = (rng.standard_normal((6, 128)) * 0.03 + rng.uniform(-0.05, 0.05, (6, 1))).astype(np.float32)
    w = f32_bits_to_bf16_exact((vals.view(np.uint32) & 0xFFFF0000).view(np.float32))
    for r in (1.0, 0.75):
        _, s16, z16 = O.quantize_rtn(w, False, None, r)
        sc = O.f16_bits_to_f32(s16)
        mn = O.bf16_bits_to_f32(w).min(axis=1)
        for n in range(6):
            t = -Fraction(float(np.float32(r) * mn[n])) / Fraction(float(sc[n, 0]))
            cands = sorted(range(16), key=lambda c: (abs(t - c), c % 2))
            assert int(O.f16_bits_to_f32(z16)[n, 0]) == cands[0]


def test_awq_s_one_equals_rtn_and_shrink_one_equals_no_clip():
    w = synth.bits(synth.normal_weight(32, 512, 0.02, seed=5, n_outliers=4, outlier_scale=20.0))
    for sym in (False, True):
        a = O.quantize_rtn(w, sym)
        b = O.quantize_rtn(w, sym, np.ones(512, np.float32), 1.0)
        for x, y in zip(a, b):
            assert (x is None and y is None) or np.array_equal(x, y)


def test_weight_mse_closed_form_uniform():
    """Uniform data: the quantization error is uniform on [-scale/2, scale/2],
    so MSE = mean(scale^2)/12.  A wrong range divisor (e.g. 16) or a scale
    that ignores the zero point breaks the ratio."""
    rng = np.random.default_rng(3)
    n, k = 256, 1024
    lo = rng.uniform(-1.0, -0.2, (n, k // 128, 1))
    hi = rng.uniform(0.2, 1.0, (n, k // 128, 1))
    v = (lo + (hi - lo) * rng.uniform(0, 1, (n, k // 128, 128))).astype(np.float32)
    w = f32_bits_to_bf16_exact((v.reshape(n, k).view(np.uint32) & 0xFFFF0000).view(np.float32))
    for sym in (False, True):
        codes, s16, z16 = O.quantize_rtn(w, sym)
        what = O.dequantize(codes, s16, z16)
        err = (O.bf16_bits_to_f32(w) - what).astype(np.float64)
        sc = O.f16_bits_to_f32(s16).astype(np.float64)
        ratio = np.mean(err ** 2) / (np.mean(sc ** 2) / 12.0)
        # symmetric grids waste part of the range on the short side, but the
        # error inside the grid is still uniform over one step.
        assert abs(ratio - 1.0) < 0.03, (sym, ratio)


def test_dequant_is_exact():
    rng = np.random.default_rng(2)
    codes = rng.integers(0, 16, (8, 256), dtype=np.uint8)
    s16 = O.f32_to_f16_bits(rng.uniform(1e-4, 0.1, (8, 2)).astype(np.float32))
    z16 = O.f32_to_f16_bits(rng.integers(0, 16, (8, 2)).astype(np.float32))
    what = O.dequantize(codes, s16, z16)
    sc = O.f16_bits_to_f32(s16)
    z = O.f16_bits_to_f32(z16)
    for n in range(8):
        for k in range(0, 256, 7):
            ex = (int(codes[n, k]) - Fraction(float(z[n, k // 128]))) * Fraction(float(sc[n, k // 128]))
            assert Fraction(float(what[n, k])) == ex


# -------------------------------------------------------------- linear -----

def test_linear_exact_rational_small():
    x = synth.bits(synth.normal_activations(2, 256, seed=9))
    w = synth.bits(synth.normal_weight(3, 256, 0.02, seed=10))
    codes, s16, z16 = O.quantize_rtn(w, False)
    what = O.dequantize(codes, s16, z16)
    y = O.linear(x, what)
    xf = O.bf16_bits_to_f32(x)
    for m in range(2):
        for n in range(3):
            ex = sum(Fraction(float(xf[m, k])) * Fraction(float(what[n, k])) for k in range(256))
            assert abs(y[m, n] - float(ex)) <= 1e-14 * max(1.0, abs(float(ex)))


def test_linear_closed_form_constant_weight():
    """Codes z+1 everywhere: w_hat = scale in each row, y[m,n] = scale_n * sum_k x[m,k]."""
    x = synth.bits(synth.normal_activations(3, 128, seed=4))
    s16 = O.f32_to_f16_bits(np.array([[0.5], [0.25], [0.125]], np.float32))
    z16 = O.f32_to_f16_bits(np.full((3, 1), 8.0, np.float32))
    codes = np.full((3, 128), 9, np.uint8)
    y = O.linear(x, O.dequantize(codes, s16, z16))
    rowsum = O.bf16_bits_to_f32(x).astype(np.float64).sum(axis=1)
    assert np.allclose(y, rowsum[:, None] * np.array([0.5, 0.25, 0.125])[None, :], rtol=0, atol=1e-12)


# ----------------------------------------------------------------- AWQ -----

def test_awq_scale_stat_and_pow_brute_force():
    x = synth.bits(synth.student_t_calibration(5, 128, seed=21))
    xf = O.bf16_bits_to_f32(x)
    stat = O.awq_channel_stat(x)
    s = O.awq_scales(stat, [0.0, 0.35, 0.95])
    for j in range(128):
        ex = sum(abs(Fraction(float(xf[m, j]))) for m in range(5)) / 5
        assert stat[j] == float(ex)  # sums of 5 bf16 values are exact in binary64
        for i, a in enumerate((0.0, 0.35, 0.95)):
            ref = np.float32(math.pow(max(float(ex), 1e-8), float(np.float32(a))))
            assert s[i, j] == ref
    assert np.all(s[0] == 1.0)


def test_awq_scales_closed_forms():
    """s = float32(stat ** alpha) where the power has an exact closed form:
    alpha = 1/2 on perfect squares (s = k), alpha = 1/4 and 3/4 on 2^(4k)
    (s = 2^k, 2^(3k)), and two roots exactly halfway between binary32
    neighbours, which the final rounding must send to the even one:
    sqrt((1 + 2^-24)^2) = 1 + 2^-24 -> 1.0 and
    sqrt((1 + 3 2^-24)^2) = 1 + 3 2^-24 -> 1 + 2^-22 (both squares are exact in
    binary64).  A stat below the floor 1e-8 takes the floor."""
    ks = np.array([1.0, 3.0, 7.0, 12.0, 255.0, 4096.0, 0.5, 0.125])
    s = O.awq_scales(ks * ks, [0.5])[0]
    assert np.array_equal(s, ks.astype(np.float32))
    p = np.array([-6, -3, 0, 1, 5, 9], dtype=np.float64)  # 2^-24 stays above the floor
    s = O.awq_scales(2.0 ** (4 * p), [0.25, 0.75])
    assert np.array_equal(s[0], (2.0 ** p).astype(np.float32))
    assert np.array_equal(s[1], (2.0 ** (3 * p)).astype(np.float32))
    t1, t3 = 1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24
    assert Fraction(t1 * t1) == Fraction(t1) ** 2 and Fraction(t3 * t3) == Fraction(t3) ** 2
    s = O.awq_scales(np.array([t1 * t1, t3 * t3]), [0.5])[0]
    assert s[0] == np.float32(1.0)
    assert s[1] == np.float32(1.0 + 2.0 ** -22)
    s = O.awq_scales(np.array([1e-12, 0.0]), [0.5])[0]
    assert np.all(s == np.float32(1e-4))


def _sse_exact(x_bits, w_bits, s, shrink, sym):
    codes, s16, z16 = O.quantize_rtn(w_bits, sym, s, shrink)
    what = O.dequantize(codes, s16, z16)
    xf = O.bf16_bits_to_f32(x_bits)
    wf = O.bf16_bits_to_f32(w_bits)
    m_, k_ = xf.shape
    n_ = wf.shape[0]
    tot = Fraction(0)
    for n in range(n_):
        e = [Fraction(float(wf[n, k])) - Fraction(float(what[n, k])) / Fraction(float(s[k]))
             for k in range(k_)]
        for m in range(m_):
            y = sum(Fraction(float(xf[m, k])) * e[k] for k in range(k_))
            tot += y * y
    return tot


@pytest.mark.parametrize("sym", [False, True])
def test_awq_sse_brute_force_tiny(sym):
    x = synth.bits(synth.student_t_calibration(3, 128, seed=31))
    w = synth.bits(synth.normal_weight(2, 128, 0.02, seed=32, n_outliers=2, outlier_scale=20.0))
    alphas = np.array([0.0, 0.5], np.float32)
    shrinks = np.array([1.0, 0.8], np.float32)
    sse, arg = O.awq_score_grid(x, w, alphas, shrinks, sym)
    s_all = O.awq_scales(O.awq_channel_stat(x), alphas)
    for i in range(2):
        for j in range(2):
            ex = _sse_exact(x, w, s_all[i], float(shrinks[j]), sym)
            assert abs(sse[0, i, j] - float(ex)) <= 1e-12 * float(ex)
    assert sse.min() > 0


def test_awq_alpha_zero_row_is_plain_rtn():
    x = synth.bits(synth.student_t_calibration(16, 256, seed=41))
    w = synth.bits(synth.normal_weight(8, 256, 0.02, seed=42))
    shrinks = synth.shrink_grid(3)
    sse, _ = O.awq_score_grid(x, w, np.array([0.0, 0.25], np.float32), shrinks, False)
    for j, r in enumerate(shrinks):
        codes, s16, z16 = O.quantize_rtn(w, False, None, float(r))
        e = O.bf16_bits_to_f32(w).astype(np.float64) - O.dequantize(codes, s16, z16)
        y = O.bf16_bits_to_f32(x).astype(np.float64) @ e.T
        assert sse[0, 0, j] == pytest.approx(float(np.sum(y * y)), rel=1e-13)


def test_scale_rewrite_equivalence():
    """prev_op /= s, W *= s (deployed) equals x . (Q(W s) diag(1/s))^T (simulated)."""
    x = synth.bits(synth.student_t_calibration(32, 512, seed=51))
    w = synth.bits(synth.normal_weight(16, 512, 0.02, seed=52))
    s = O.awq_scales(O.awq_channel_stat(x), [0.6])[0]
    codes, s16, z16 = O.quantize_rtn(w, False, s, 0.9)
    what = O.dequantize(codes, s16, z16).astype(np.float64)
    xf = O.bf16_bits_to_f32(x).astype(np.float64)
    deployed = (xf / s[None, :]) @ what.T
    simulated = xf @ (what / s[None, :]).T
    assert np.max(np.abs(deployed - simulated)) <= 1e-12 * np.max(np.abs(simulated))


def test_argmin_rules_hand_table():
    shrinks = np.array([1.0, 0.9, 0.8], np.float32)
    t0 = np.array([[5.0, 4.0, 4.0],
                   [3.0, 2.0, 2.0],
                   [3.0, 9.0, 1.0]])
    t1 = np.array([[1.0, 1.0, 1.0],
                   [6.0, 0.5, 7.0],
                   [2.0, 2.0, 2.0]])
    out = O.awq_argmins(np.stack([t0, t1]), shrinks)
    # seg 0: joint min 1.0 at (2,2) -> 8; alpha* at r=1.0: tie 3.0 at rows 1,2 -> 1;
    # shrink* at alpha 1 -> tie 2.0 at 1,2 -> 1; group alpha*: sums col0 = 6,9,5 -> 2,
    # seg-0 shrink at alpha 2 -> 2.
    assert list(out[0]) == [8, 1, 1, 2]
    # seg 1: joint 0.5 at (1,1) -> 4; alpha* col0 -> 0; shrink* at 0 -> tie -> 0; at group alpha 2 -> 0
    assert list(out[1]) == [4, 0, 0, 0]
    # group: summed table [[6,5,5],[9,2.5,9],[5,11,3]] -> joint 2.5 at 4; alpha* 2
    assert list(out[2]) == [4, 2, -1, -1]


def test_segments_add_up():
    x = synth.bits(synth.student_t_calibration(16, 256, seed=61))
    w = synth.bits(synth.normal_weight(12, 256, 0.02, seed=62))
    al = np.array([0.0, 0.5], np.float32)
    sh = np.array([1.0, 0.85], np.float32)
    sse, _ = O.awq_score_grid(x, w, al, sh, False, seg_offsets=[0, 5, 12])
    a, _ = O.awq_score_grid(x, w[:5], al, sh, False)
    b, _ = O.awq_score_grid(x, w[5:], al, sh, False)
    assert np.allclose(sse[0], a[0], rtol=1e-13) and np.allclose(sse[1], b[0], rtol=1e-13)


# ------------------------------------------- per-output-channel clipping ----

def _row_sse_exact(x_bits, w_bits, s, shrink, sym):
    """Exact rational output error of every row at one shrink ratio."""
    codes, s16, z16 = O.quantize_rtn(w_bits, sym, s, shrink)
    what = O.dequantize(codes, s16, z16)
    xf = O.bf16_bits_to_f32(x_bits)
    wf = O.bf16_bits_to_f32(w_bits)
    m_, k_ = xf.shape
    out = []
    for n in range(wf.shape[0]):
        e = [Fraction(float(wf[n, k])) - Fraction(float(what[n, k])) / Fraction(float(s[k]))
             for k in range(k_)]
        tot = Fraction(0)
        for m in range(m_):
            y = sum(Fraction(float(xf[m, k])) * e[k] for k in range(k_))
            tot += y * y
        out.append(tot)
    return out


@pytest.mark.parametrize("sym", [False, True])
def test_clip_rows_sse_brute_force_tiny(sym):
    """Per-row output error of every shrink candidate, and each row's choice,
    against exact rational arithmetic on a tiny linear."""
    x = synth.bits(synth.student_t_calibration(3, 128, seed=71))
    w = synth.bits(synth.normal_weight(4, 128, 0.02, seed=72, n_outliers=3, outlier_scale=20.0))
    s = O.awq_scales(O.awq_channel_stat(x), [0.5])[0]
    shrinks = np.array([1.0, 0.8, 0.6], np.float32)
    sse, choice = O.clip_search_rows(x, w, s, shrinks, sym)
    assert sse.shape == (3, 4) and choice.shape == (4,)
    exact = [_row_sse_exact(x, w, s, float(r), sym) for r in shrinks]
    for j in range(3):
        for n in range(4):
            assert abs(sse[j, n] - float(exact[j][n])) <= 1e-12 * float(exact[j][n])
    for n in range(4):
        col = [exact[j][n] for j in range(3)]
        assert choice[n] == col.index(min(col))


def test_clip_rows_ties_take_the_lowest_index():
    """A grid that lists one ratio twice gives equal errors: the first wins."""
    x = synth.bits(synth.student_t_calibration(8, 256, seed=73))
    w = synth.bits(synth.normal_weight(6, 256, 0.02, seed=74, n_outliers=2, outlier_scale=20.0))
    sse, choice = O.clip_search_rows(x, w, None, np.array([0.7, 1.0, 0.7, 1.0], np.float32), False)
    assert np.array_equal(sse[0], sse[2]) and np.array_equal(sse[1], sse[3])
    assert set(choice.tolist()) <= {0, 1}


def test_clip_rows_invariants():
    """The per-row errors of one ratio add up to that ratio's whole-linear
    error (a sum over output channels), and the per-row choice is never worse
    than the best single ratio."""
    x = synth.bits(synth.student_t_calibration(16, 256, seed=75))
    w = synth.bits(synth.normal_weight(10, 256, 0.02, seed=76, n_outliers=2, outlier_scale=20.0))
    shrinks = synth.shrink_grid(4)
    s = O.awq_scales(O.awq_channel_stat(x), [0.3])[0]
    sse, choice = O.clip_search_rows(x, w, s, shrinks, False)
    xf = O.bf16_bits_to_f32(x).astype(np.float64)
    for j, r in enumerate(shrinks):
        y = xf @ O.candidate_error(w, s, r, False).T
        assert sse[j].sum() == pytest.approx(float(np.sum(y * y)), rel=1e-12)
    assert sse[choice, np.arange(10)].sum() <= sse.sum(axis=1).min()


@pytest.mark.parametrize("sym", [False, True])
def test_quantize_rows_reduces_to_per_linear_quantize(sym):
    """One ratio for every row is the per-linear quantizer; distinct ratios
    quantize each row as that row alone with its ratio."""
    w = synth.bits(synth.normal_weight(5, 384, 0.02, seed=77, n_outliers=2, outlier_scale=20.0))
    x = synth.bits(synth.student_t_calibration(4, 384, seed=78))
    s = O.awq_scales(O.awq_channel_stat(x), [0.4])[0]
    same = O.quantize_pack_rows(w, sym, s, np.full(5, 0.85, np.float32))
    ref = O.quantize_pack(w, sym, s, 0.85)
    for a, b in zip(same, ref):
        assert (a is None and b is None) or np.array_equal(a, b)
    rows = np.array([1.0, 0.55, 0.9, 0.75, 0.6], np.float32)
    mixed = O.quantize_pack_rows(w, sym, s, rows)
    for n in range(5):
        one = O.quantize_pack(w[n:n + 1], sym, s, float(rows[n]))
        assert np.array_equal(mixed[0][n:n + 1], one[0]) and np.array_equal(mixed[1][n:n + 1], one[1])
        if not sym:
            assert np.array_equal(mixed[2][n:n + 1], one[2])


# ------------------------------------------------------------- W4A8 -----

def test_act_int8_brute_force():
    """Every code is the integer nearest x / scale (exact rationals; the
    binary32 quotient may sit a hair across a half), the row's largest
    magnitude maps to +-127, and a zero row stays zero."""
    x = synth.bits(synth.student_t_calibration(4, 256, seed=91))
    x[2] = 0
    q, sc = O.quantize_act_int8(x)
    xf = O.bf16_bits_to_f32(x)
    for m in range(4):
        amax = max(abs(Fraction(float(v))) for v in xf[m])
        if amax == 0:
            assert sc[m] == 0 and np.all(q[m] == 0)
            continue
        assert sc[m] == np.float32(float(amax)) / np.float32(127.0)
        s = Fraction(float(sc[m]))
        for k in range(256):
            r = Fraction(float(xf[m, k])) / s
            assert abs(r - int(q[m, k])) <= Fraction(1, 2) + Fraction(1, 1 << 20)
            assert -127 <= int(q[m, k]) <= 127
        j = int(np.argmax(np.abs(xf[m])))
        assert abs(int(q[m, j])) == 127


@pytest.mark.parametrize("sym", [False, True])
def test_w4a8_linear_exact_rational_small(sym):
    x = synth.bits(synth.normal_activations(3, 256, seed=92))
    w = synth.bits(synth.normal_weight(5, 256, 0.02, seed=93, n_outliers=2, outlier_scale=20.0))
    q, xs = O.quantize_act_int8(x)
    codes, s16, z16 = O.quantize_rtn(w, sym)
    y = O.w4a8_linear(q, xs, codes, s16, z16)
    sc = O.f16_bits_to_f32(s16)
    z = np.full(sc.shape, 8.0) if z16 is None else O.f16_bits_to_f32(z16)
    for m in range(3):
        for n in range(5):
            tot = Fraction(0)
            for k in range(256):
                g = k // 128
                tot += (Fraction(int(codes[n, k])) - Fraction(float(z[n, g]))) * \
                    Fraction(float(sc[n, g])) * int(q[m, k])
            ex = tot * Fraction(float(xs[m]))
            assert abs(y[m, n] - float(ex)) <= 1e-12 * abs(float(ex)) + 1e-300


def test_w4a8_is_w4a16_on_the_quantized_activation():
    """y_a16 - y_a8 = w_hat . (x - q * scale): the W4A8 result is the W4A16
    linear of the dequantized activation (exact identity)."""
    x = synth.bits(synth.normal_activations(4, 384, seed=94))
    w = synth.bits(synth.normal_weight(7, 384, 0.02, seed=95))
    q, xs = O.quantize_act_int8(x)
    codes, s16, z16 = O.quantize_rtn(w, False)
    what = O.dequantize(codes, s16, z16).astype(np.float64)
    y8 = O.w4a8_linear(q, xs, codes, s16, z16)
    xd = q.astype(np.float64) * xs.astype(np.float64)[:, None]
    assert np.allclose(y8, xd @ what.T, rtol=1e-12, atol=1e-300)
    y16 = O.linear(x, what)
    err = O.bf16_bits_to_f32(x).astype(np.float64) - xd
    bound = np.abs(err) @ np.abs(what).T
    assert np.all(np.abs(y16 - y8) <= bound * (1 + 1e-9) + 1e-300)


def test_act_int8_ties_to_even_hand_case():
    """max |x| = 127 gives scale 1.0 exactly, so halves are exact ties; the
    codes follow round-half-to-even: 0.5 -> 0, 1.5 -> 2, 2.5 -> 2, -2.5 -> -2,
    3.5 -> 4 (hand-derived)."""
    vals = np.array([[127.0, 0.5, 1.5, 2.5, -0.5, -2.5, 3.5, -127.0] + [0.0] * 120],
                    np.float32)
    q, sc = O.quantize_act_int8(f32_bits_to_bf16_exact(vals))
    assert sc[0] == np.float32(1.0)
    assert q[0, :8].tolist() == [127, 0, 2, 2, 0, -2, 4, -127]


def test_storage_accounting():
    """Stored bytes per weight of the packed format: 4 bits of code plus an
    fp16 scale (and an fp16 zero when asymmetric) per 128 weights, i.e.
    0.53125 B/weight asymmetric and 0.515625 symmetric; the symmetric rate
    applied to the 27B card's 12.56 GB of int4 linears gives about 24.4e9
    parameters (a plausibility check of a 27B-class model, not a pin of the
    card's own packing, which it does not state)."""
    w = synth.bits(synth.normal_weight(16, 384, 0.02, seed=81))
    for sym, rate in ((False, 0.53125), (True, 0.515625)):
        qw, s16, z16 = O.quantize_pack(w, sym)
        stored = qw.nbytes + s16.nbytes + (0 if z16 is None else z16.nbytes)
        assert stored == rate * w.size
    assert 24.0e9 < 12.56e9 / 0.515625 < 24.8e9
