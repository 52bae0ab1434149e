"""CPU oracle for weight-only int4 group-128 quantization, the W4A16 linear and
AWQ alpha/shrink candidate scoring.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code with the CUDA library (no helpers,
no tables, no constants generators); both sides receive the same seeded inputs
from ``weight_only_int4_quantize_b200.synth``, which holds no arithmetic of
the method.

Precision.  The pages fix no precision for the quantizer, so every decision
that yields an integer (a code, a zero point) is taken in IEEE binary32 with
round-to-nearest-even and no fused multiply-add, exactly as the kernels take
it.  Everything that is a sum (the linear, the AWQ error energy) is taken in
binary64.  numpy float32 arithmetic is IEEE binary32 with one rounding per
operation; ``np.rint`` rounds half to even.

Sources (model-card pages; cited by page title and section):
  [rebuttal] "ghostchoir/rebuttal_w4g128_awq_w2" model card:
      'Model Details' table, rows 'Scheme' and 'Search';
      paragraph on AWQ's scale rewrite (prev_op /= s, W *= s);
      paragraph 'Clipping granularity' (one shrink ratio per linear);
      note under the perplexity table defining RTN.
  [qwen27b] "GotoAI-Inc/Qwen3.6-27B-W4A16" model card, opening paragraph
      (int4, group size 128, symmetric, weight-only, activations 16-bit).
  [awq-ppl] "AWQ INT4-g128 WikiText-2 perplexity delta vs fp16, Llama-2 7B",
      'Methodology' (group size 128; grid size 20 for the alpha search).
  [qsrt] "malaiwah/GLM-5.2-QSRT-Fruit-Instruct" card: 'What is included'
      (W4A8 decode execution), the storage paragraph (W4A8 and W4A16 use
      the same stored weights) and the runtime paragraph (W4A8 for
      decode-sized batches of at most 16 rows).
  [rebuttal-cmp] the same "ghostchoir/rebuttal_w4g128_awq_w2" card, the
      'Comparability caveat' under the perplexity table (the d=0 arm uses
      stock AWQ's per-output-channel clipping search).

Readings where the pages are silent (each is pinned by a test in
tests/test_oracle_pins.py; the exact list with reasons is in the repository's
design notes):
  * a group is 128 consecutive input channels (K) of one output row;
  * asymmetric: scale = max(r*max - r*min, 1e-5) / 15,
    zero = clamp(rint(-(r*min) / scale16), 0, 15);
  * symmetric: scale = max(r*absmax, 1e-5) / 7, implicit zero 8, no zeros
    tensor;
  * the scale is stored as fp16 (round to nearest even) and the codes are
    computed from the STORED scale, so that dequantization reproduces them;
  * code = clamp(rint(v / scale16) + zero, 0, 15), IEEE division, ties to
    even;
  * the AWQ scale multiplies before quantization (v = w * s in binary32) and
    the shrink ratio r scales the group's range in that s-domain;
  * s_j = float32(pow(max(mean_m |x_mj|, 1e-8), alpha)), mean in binary64;
  * stock per-output-channel clipping: every output row takes its own ratio
    from the same shrink grid, the one with the least output error of that
    row, ||x E_n^T||^2 (the linear's output error is a sum over rows, so the
    per-row choices minimise it jointly); ties go to the lowest grid index;
  * W4A8 activations ([qsrt] fixes no format): per token row, symmetric
    int8, scale = max_k |x_mk| / 127 in binary32, code = clamp(rint(x /
    scale), -127, 127) with IEEE division and ties to even; a row of zeros
    has scale 0 and codes 0.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

GROUP = 128

# ----------------------------------------------------------------------------
# Bit formats.  bf16 is the upper half of an IEEE binary32; fp16 is IEEE
# binary16 (1 sign, 5 exponent bits with bias 15, 10 fraction bits).
# ----------------------------------------------------------------------------


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns (uint16) to float32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def _round_shift_rne(a: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Integer a / 2**s rounded to nearest, ties to even (a >= 0, s >= 1)."""
    a = a.astype(np.uint64)
    s = s.astype(np.uint64)
    q = a >> s
    rem = a - (q << s)
    half = np.uint64(1) << (s - np.uint64(1))
    up = (rem > half) | ((rem == half) & ((q & np.uint64(1)) == 1))
    return q + up.astype(np.uint64)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary32 values to binary16, round-to-nearest-even, as bit patterns.

    Written from the binary16 format definition (IEEE 754-2008 s3.6):
    normal numbers (1024 + f) * 2**(e - 25) for biased exponent e in 1..30,
    subnormals f * 2**-24, overflow past the largest finite value 65504
    rounds to infinity.  NaN inputs are outside this oracle's domain.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    sign = (u >> np.uint64(31)) << np.uint64(15)
    e32 = ((u >> np.uint64(23)) & np.uint64(0xFF)).astype(np.int64)
    frac = u & np.uint64(0x7FFFFF)
    # binary32 value = sig * 2**(e32 - 150); subnormal binary32 inputs are far
    # below binary16's smallest subnormal and round to zero.
    sig = np.where(e32 > 0, frac | np.uint64(0x800000), np.uint64(0))
    e_unb = e32 - 127  # unbiased exponent of a normal binary32
    out = np.zeros(x.shape, dtype=np.uint64)

    # binary16 normal range: 2**-14 <= |x|.  Keep 11 significant bits.
    normal = (e32 > 0) & (e_unb >= -14) & (e32 < 255)
    sig16 = _round_shift_rne(sig[normal], np.full(sig[normal].shape, 13))
    e16 = (e_unb[normal] + 15).astype(np.uint64)
    # (e16 - 1) * 1024 + sig16 also absorbs a carry of sig16 into 2048.
    bits = ((e16 - np.uint64(1)) << np.uint64(10)) + sig16
    bits = np.minimum(bits, np.uint64(0x7C00))  # overflow -> infinity
    out[normal] = bits

    # binary16 subnormal range: value / 2**-24 = sig * 2**(e32 - 126).
    sub = (e32 > 0) & (e_unb < -14)
    shift = (126 - e32[sub]).astype(np.uint64)
    big = shift > np.uint64(40)  # far below 2**-25: rounds to zero
    shift = np.minimum(shift, np.uint64(40))
    val = _round_shift_rne(sig[sub], shift)
    val[big] = 0
    out[sub] = val

    inf = e32 == 255
    out[inf] = np.where(frac[inf] == 0, np.uint64(0x7C00), np.uint64(0x7E00))
    return (out | sign).astype(np.uint16)


def f16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of binary16 bit patterns to float32 (format definition)."""
    h = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    s = np.where(h >> 15, -1.0, 1.0)
    e = (h >> 10) & 0x1F
    f = h & 0x3FF
    mag = np.where(e == 0, f * 2.0 ** -24, (1024 + f) * np.exp2(e.astype(np.float64) - 25))
    mag = np.where(e == 31, np.where(f == 0, np.inf, np.nan), mag)
    return (s * mag).astype(np.float32)


# ----------------------------------------------------------------------------
# RTN group quantization and packing.
# ----------------------------------------------------------------------------


def quantize_rtn(w_bits: np.ndarray, symmetric: bool, awq_s: np.ndarray | None = None,
                 shrink: float = 1.0, group: int = GROUP):
    """Round-to-nearest int4 group quantization of one linear's weight.

    [rebuttal] 'Scheme': weight-only, 4-bit, group size 128, asymmetric (zero
    point); the perplexity-table note defines RTN as round-to-nearest group
    quantization.  [qwen27b]: int4, group size 128, symmetric.  The AWQ
    per-input-channel scale enters as Q(W diag(s)) ([rebuttal], scale-rewrite
    paragraph); the shrink ratio r narrows the group range ([rebuttal],
    'Clipping granularity').

    w_bits: [N, K] bfloat16 bit patterns, K a multiple of ``group``.
    Returns (codes uint8 [N, K] in 0..15, scale16 uint16 [N, K/group],
    zero16 uint16 [N, K/group] or None when symmetric).
    """
    w = bf16_bits_to_f32(w_bits)
    n, k = w.shape
    assert k % group == 0
    v = w if awq_s is None else w * np.asarray(awq_s, dtype=np.float32)[None, :]
    vg = v.reshape(n, k // group, group)
    # One ratio per linear, or one per output row (a length-N array).
    r = (np.asarray(shrink, dtype=np.float32).reshape(n, 1) if np.ndim(shrink) == 1
         else np.float32(shrink))
    floor = np.float32(1e-5)
    if symmetric:
        a = r * np.max(np.abs(vg), axis=2)
        scale32 = np.maximum(a, floor) / np.float32(7.0)
    else:
        mx = r * np.max(vg, axis=2)
        mn = r * np.min(vg, axis=2)
        scale32 = np.maximum(mx - mn, floor) / np.float32(15.0)
    scale16 = f32_to_f16_bits(scale32)
    sc = f16_bits_to_f32(scale16)
    if symmetric:
        z = np.full(sc.shape, 8, dtype=np.int64)
    else:
        z = np.clip(np.rint(-mn / sc), 0, 15).astype(np.int64)
    with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
        t = np.rint(vg / sc[:, :, None]).astype(np.float64)
    codes = np.clip(t + z[:, :, None], 0, 15).astype(np.uint8).reshape(n, k)
    zero16 = None if symmetric else f32_to_f16_bits(z.astype(np.float32))
    return codes, scale16, zero16


# Nibble i (bits 4i..4i+3) of packed word w holds the code of input channel
# 8w + PACK_ORDER[i].  Pairs of nibbles (i, i+4) are then the adjacent
# channels (2i, 2i+1).
PACK_ORDER = (0, 2, 4, 6, 1, 3, 5, 7)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Pack [N, K] codes into int32 [N, K/8], eight codes per word in the
    nibble order PACK_ORDER.  The pages give storage sizes only, no layout;
    this is the library's canonical layout."""
    c = np.asarray(codes, dtype=np.uint32)
    n, k = c.shape
    c = c.reshape(n, k // 8, 8)
    word = np.zeros((n, k // 8), dtype=np.uint32)
    for i, j in enumerate(PACK_ORDER):
        word |= c[:, :, j] << np.uint32(4 * i)
    return word.view(np.int32)


def unpack_codes(qweight: np.ndarray) -> np.ndarray:
    """Inverse of pack_codes."""
    w = np.asarray(qweight).view(np.uint32)
    n, kw = w.shape
    out = np.empty((n, kw, 8), dtype=np.uint8)
    for i, j in enumerate(PACK_ORDER):
        out[:, :, j] = (w >> np.uint32(4 * i)) & np.uint32(0xF)
    return out.reshape(n, kw * 8)


def dequantize(codes: np.ndarray, scale16: np.ndarray, zero16: np.ndarray | None,
               group: int = GROUP) -> np.ndarray:
    """w_hat = (q - z) * scale in binary32.  Exact: |q - z| <= 15 has 4
    significant bits and the fp16 scale 11, so the product fits in 24."""
    n, k = codes.shape
    sc = f16_bits_to_f32(scale16)
    z = (np.full(sc.shape, 8.0, dtype=np.float32) if zero16 is None
         else f16_bits_to_f32(zero16))
    q = codes.astype(np.float32).reshape(n, k // group, group)
    return ((q - z[:, :, None]) * sc[:, :, None]).reshape(n, k).astype(np.float32)


def quantize_pack(w_bits, symmetric, awq_s=None, shrink=1.0, group=GROUP):
    """The full quantize+pack step: (qweight int32 [N,K/8], scale16, zero16)."""
    codes, s16, z16 = quantize_rtn(w_bits, symmetric, awq_s, shrink, group)
    return pack_codes(codes), s16, z16


# ----------------------------------------------------------------------------
# The W4A16 linear: y = x . dequant(Wq)^T, activations stay 16-bit ([qwen27b]).
# ----------------------------------------------------------------------------


def linear(x_bits: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """y[m, n] = sum_k x[m, k] * w_hat[n, k], in binary64 (exact inputs)."""
    x = bf16_bits_to_f32(x_bits).astype(np.float64)
    return x @ np.asarray(w_hat, dtype=np.float64).T


def linear_rows(x_bits: np.ndarray, w_hat: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """The same linear for a subset of token rows (large-M sampling)."""
    return linear(np.asarray(x_bits)[rows], w_hat)


# ----------------------------------------------------------------------------
# AWQ candidate scoring over the alpha x shrink grid.
# ----------------------------------------------------------------------------


def awq_channel_stat(x_bits: np.ndarray) -> np.ndarray:
    """stat_j = mean over tokens of |x_mj|, in binary64.  [rebuttal] 'Search'
    names the AWQ scale exponent; the statistic is the per-input-channel
    activation magnitude that s = stat**alpha raises."""
    x = bf16_bits_to_f32(x_bits).astype(np.float64)
    return np.abs(x).sum(axis=0) / x.shape[0]


def awq_scales(stat: np.ndarray, alphas) -> np.ndarray:
    """s[i, j] = float32(max(stat_j, 1e-8) ** alpha_i).  alpha = 0 gives s = 1
    exactly, which reduces AWQ to plain RTN."""
    st = np.maximum(np.asarray(stat, dtype=np.float64), 1e-8)
    out = np.empty((len(alphas), st.shape[0]), dtype=np.float32)
    for i, a in enumerate(alphas):
        out[i] = np.power(st, np.float64(np.float32(a))).astype(np.float32)
    return out


def candidate_error(w_bits, s, shrink, symmetric, group=GROUP) -> np.ndarray:
    """E = W - Q(W diag(s)) diag(1/s) in binary64 ([rebuttal], scale-rewrite
    paragraph: the candidate is simulated by swapping only the weight)."""
    codes, s16, z16 = quantize_rtn(w_bits, symmetric, s, shrink, group)
    w_hat = dequantize(codes, s16, z16, group).astype(np.float64)
    w = bf16_bits_to_f32(w_bits).astype(np.float64)
    return w - w_hat / np.asarray(s, dtype=np.float64)[None, :]


def awq_score_grid(x_bits, w_bits, alphas, shrinks, symmetric, seg_offsets=None,
                   group=GROUP):
    """Squared output error of every (alpha, shrink) candidate.

    [rebuttal] 'Search': AWQ scale exponent on a 20-point grid and a 10-point
    global shrink grid, scored by MSE; [awq-ppl] 'Methodology': grid size 20
    for the alpha search.  The score here is the linear's own output error
    ||X E^T||_F^2 (a sum, so tables of linears that share an input add up).

    seg_offsets: row boundaries splitting W into linears that share x (e.g.
    q, k, v); default one segment.  Returns sse [n_seg, n_alpha, n_shrink]
    (binary64) and the argmins of awq_argmins().
    """
    n = np.asarray(w_bits).shape[0]
    seg = np.asarray([0, n] if seg_offsets is None else seg_offsets, dtype=np.int64)
    x = bf16_bits_to_f32(x_bits).astype(np.float64)
    s_all = awq_scales(awq_channel_stat(x_bits), alphas)
    sse = np.empty((len(seg) - 1, len(alphas), len(shrinks)), dtype=np.float64)
    for i in range(len(alphas)):
        for j, r in enumerate(shrinks):
            e = candidate_error(w_bits, s_all[i], r, symmetric, group)
            y = x @ e.T
            for g in range(len(seg) - 1):
                yg = y[:, seg[g]:seg[g + 1]]
                sse[g, i, j] = np.sum(yg * yg)
    return sse, awq_argmins(sse, shrinks)


def no_clip_column(shrinks) -> int:
    """Index of the shrink ratio 1.0 (no clipping); column 0 if absent."""
    for j, r in enumerate(shrinks):
        if np.float32(r) == np.float32(1.0):
            return j
    return 0


def awq_argmins(sse: np.ndarray, shrinks) -> np.ndarray:
    """Selections over an SSE table [n_seg, n_alpha, n_shrink].

    Per segment row s: [joint flat index (alpha-major), alpha* at shrink 1.0,
    shrink* at that segment's alpha*, shrink* at the group's alpha*].
    Last row (the group of segments sharing one s, since one prev_op is
    divided by s, [rebuttal] scale-rewrite paragraph): [joint index of the
    summed table, alpha* of the summed table at shrink 1.0, -1, -1].
    The shrink search stays per linear ([rebuttal], 'Clipping granularity').
    Equal minima resolve to the lowest index (np.argmin's first occurrence).
    """
    n_seg, n_a, n_r = sse.shape
    c1 = no_clip_column(shrinks)
    total = sse.sum(axis=0)
    a_grp = int(np.argmin(total[:, c1]))
    out = np.full((n_seg + 1, 4), -1, dtype=np.int64)
    for s in range(n_seg):
        t = sse[s]
        a_s = int(np.argmin(t[:, c1]))
        out[s] = [int(np.argmin(t)), a_s, int(np.argmin(t[a_s])), int(np.argmin(t[a_grp]))]
    out[n_seg, 0] = int(np.argmin(total))
    out[n_seg, 1] = a_grp
    return out


def relative_gap(values: np.ndarray) -> float:
    """(second smallest - smallest) / smallest over a flat array: how far the
    winner of an argmin is from a tie."""
    v = np.sort(np.asarray(values, dtype=np.float64).ravel())
    if v.size < 2 or v[0] <= 0:
        return float("inf")
    return float((v[1] - v[0]) / v[0])


def clip_search_rows(x_bits, w_bits, awq_s, shrinks, symmetric, group=GROUP):
    """Stock per-output-channel clipping search ([rebuttal-cmp]; contrasted in
    [rebuttal] 'Clipping granularity' with the one global shrink ratio that a
    look-ahead loss forces).

    For every shrink r_j of the grid: E_j = W - Q_{r_j}(W diag(s)) diag(1/s)
    (s = awq_s, or 1 when None) and the error of each output channel n,
    sse_rows[j, n] = sum_m (x E_j^T)[m, n]^2, in binary64.  Row n takes
    choice[n] = argmin_j sse_rows[j, n], the lowest j on equal values.
    Returns (sse_rows [n_shrink, N] float64, choice int64 [N])."""
    n, k = np.asarray(w_bits).shape
    s = np.ones(k, dtype=np.float32) if awq_s is None else np.asarray(awq_s, dtype=np.float32)
    x = bf16_bits_to_f32(x_bits).astype(np.float64)
    sse = np.empty((len(shrinks), n), dtype=np.float64)
    for j, r in enumerate(shrinks):
        y = x @ candidate_error(w_bits, s, r, symmetric, group).T
        sse[j] = np.sum(y * y, axis=0)
    return sse, np.argmin(sse, axis=0)


def quantize_pack_rows(w_bits, symmetric, awq_s, shrink_rows, group=GROUP):
    """quantize_pack with one shrink ratio per output row (the per-channel
    clipping's deployed weight)."""
    codes, s16, z16 = quantize_rtn(w_bits, symmetric, awq_s,
                                   np.asarray(shrink_rows, dtype=np.float32), group)
    return pack_codes(codes), s16, z16


# ----------------------------------------------------------------------------
# W4A8 decode: the same stored int4 weights against int8 activations ([qsrt]).
# ----------------------------------------------------------------------------


def quantize_act_int8(x_bits: np.ndarray):
    """Per-token symmetric int8 activations.  Returns (codes int8 [M, K],
    scale float32 [M]); x ~ codes * scale per row."""
    x = bf16_bits_to_f32(x_bits)
    amax = np.max(np.abs(x), axis=1)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.rint(x / scale[:, None])
    t = np.where(scale[:, None] > 0, t, 0.0)
    return np.clip(t, -127, 127).astype(np.int8), scale


def w4a8_linear(xq: np.ndarray, xscale: np.ndarray, codes: np.ndarray, scale16: np.ndarray,
                zero16: np.ndarray | None, group: int = GROUP) -> np.ndarray:
    """y[m, n] = xscale_m * sum_g scale_ng * D[m, n, g], where the group dot
    D = sum_{k in g} (q_nk - z_ng) * xq_mk is an exact integer; the scaling
    and the sum over groups in binary64."""
    n, k = codes.shape
    g = k // group
    z = (np.full((n, g), 8, dtype=np.int64) if zero16 is None
         else f16_bits_to_f32(zero16).astype(np.int64))
    w = codes.astype(np.int64).reshape(n, g, group) - z[:, :, None]
    xg = np.asarray(xq, dtype=np.int64).reshape(xq.shape[0], g, group)
    d = np.einsum("mgk,ngk->mng", xg, w)  # exact integers
    sc = f16_bits_to_f32(scale16).astype(np.float64)
    return np.asarray(xscale, dtype=np.float64)[:, None] * np.einsum("mng,ng->mn",
                                                                     d.astype(np.float64), sc)


# ----------------------------------------------------------------------------
# Exact rational helpers for brute-force pins on tiny inputs.
# ----------------------------------------------------------------------------


def exact(a) -> list:
    """Fractions of every element (floats are dyadic rationals)."""
    return [[Fraction(float(v)) for v in row] for row in np.asarray(a, dtype=np.float64)]
