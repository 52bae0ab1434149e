"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
identical seeded inputs.

Bars (written here, checked element by element):
  * quantize + pack: codes, fp16 scales and fp16 zeros bit-exact;
  * AWQ scales s: bit-exact;
  * linear: max|y_gpu - y_ref| / max|y_ref| <= 5e-3 against the binary64
    oracle over the identical dequantized weights;
  * AWQ scoring and the per-output-channel clipping search: SSE within
    SSE_RTOL (per row: ROW_SSE_RTOL) relative; every selected index identical
    to the oracle's (the GPU decides near ties of its fp16 scores again in
    binary64), unless the oracle's own binary64 values are equal to 1e-12,
    which is asserted on those values.
"""
import numpy as np
import pytest
import torch

import weight_only_int4_quantize_b200 as w4
from oracle import w4_oracle as O
from weight_only_int4_quantize_b200 import synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

DEV = "cuda:0"
Y_RTOL = 5e-3           # linear: max-normalized error bound
# AWQ: fp16 tensor-core operands, binary64 sums.  Half the library's tie
# tolerance for tables (5e-4): within it the fp16 values cannot invert the
# order of two candidates that are not both decided again in binary64.
SSE_RTOL = 2.5e-4
GENUINE_TIE_RTOL = 1e-12  # oracle values this close are a tie of the definition itself


def u16(t):
    return t.cpu().numpy().view(np.uint16)


def quantize_both(w_cpu, sym, s=None, r=1.0):
    s_dev = None if s is None else torch.from_numpy(np.ascontiguousarray(s)).to(DEV)
    qw, sc, zr = w4.quantize_pack(w_cpu.to(DEV), sym, s_dev, r)
    torch.cuda.synchronize()
    ref = O.quantize_pack(synth.bits(w_cpu), sym, s, r)
    return (qw, sc, zr), ref


def assert_quant_equal(gpu, ref, sym):
    qw, sc, zr = gpu
    oq, os_, oz = ref
    assert np.array_equal(qw.cpu().numpy(), oq), "packed codes differ"
    assert np.array_equal(u16(sc), os_), "scales differ"
    if sym:
        assert zr is None and oz is None
    else:
        assert np.array_equal(u16(zr), oz), "zeros differ"


def max_rel_err(y_gpu, y_ref):
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    return float(np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref)))


# ------------------------------------------------------------ quantize ----

@pytest.mark.parametrize("sym", [False, True])
def test_quantize_single_linear_2048_outliers(sym):
    w = synth.normal_weight(2048, 2048, 0.02, seed=0, n_outliers=8, outlier_scale=20.0)
    gpu, ref = quantize_both(w, sym)
    assert_quant_equal(gpu, ref, sym)


@pytest.mark.parametrize("n,k", [(1, 128), (3, 384), (17, 256), (1000, 1152), (6144, 2048)])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("r", [1.0, 0.7])
def test_quantize_shapes_shrink(n, k, sym, r):
    w = synth.normal_weight(n, k, 0.02, seed=n * 7 + k, n_outliers=min(8, k // 16),
                            outlier_scale=20.0)
    gpu, ref = quantize_both(w, sym, None, r)
    assert_quant_equal(gpu, ref, sym)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("alpha", [0.0, 0.5, 0.95])
def test_quantize_with_awq_scale(sym, alpha):
    x = synth.student_t_calibration(256, 2048, seed=5)
    w = synth.normal_weight(1024, 2048, 0.02, seed=6)
    s = O.awq_scales(O.awq_channel_stat(synth.bits(x)), [alpha])[0]
    gpu, ref = quantize_both(w, sym, s, 0.85)
    assert_quant_equal(gpu, ref, sym)
    if alpha == 0.0:  # s == 1 reduces to plain RTN, byte for byte
        plain, _ = quantize_both(w, sym, None, 0.85)
        for a, b in zip(gpu, plain):
            assert (a is None and b is None) or torch.equal(a, b)


def test_quantize_shrink_one_is_no_clip():
    w = synth.normal_weight(512, 1024, 0.02, seed=8, n_outliers=8, outlier_scale=20.0)
    for sym in (False, True):
        a, _ = quantize_both(w, sym, None, 1.0)
        s1 = np.ones(1024, np.float32)
        b, _ = quantize_both(w, sym, s1, 1.0)
        for p, q in zip(a, b):
            assert (p is None and q is None) or torch.equal(p, q)


def _near_tie_inputs(sym, groups=64, rows=8, seed=3):
    """Weights and per-channel scales whose products v = w*s put v/scale
    within a few ulp of a half-integer tie (exactly on it, just above and
    just below), so the division-free rounding path must defer to the exact
    division.  w is a power of two per row, so v*2^j keeps the quotients."""
    rng = np.random.default_rng(seed)
    k = 128 * groups
    s = np.empty(k, np.float32)
    for g in range(groups):
        # a random fp16 scale with a full mantissa
        sc = np.float32(np.float16(rng.uniform(0.01, 0.1)))
        base = g * 128
        if sym:
            s[base] = np.float32(7) * sc        # absmax -> scale = sc exactly
            m = rng.integers(-7, 7, 127)  # |m + 1/2| < 7 keeps absmax = 7 * scale
        else:
            s[base] = np.float32(0.0)            # min 0 -> zero 0
            s[base + 1] = np.float32(15) * sc    # max -> scale = sc exactly
            m = rng.integers(0, 15, 127)
        for i, mm in enumerate(m):
            j = base + 1 + i + (0 if sym else 1)
            if j >= base + 128:
                break
            t = np.float32((mm + 0.5) * np.float64(sc))
            u = (int(t.view(np.uint32)) + int(rng.integers(-3, 4))) & 0xFFFFFFFF
            s[j] = np.uint32(u).view(np.float32)
    rowscale = (2.0 ** (np.arange(rows) % 5 - 2)).astype(np.float32)
    w = torch.from_numpy(np.repeat(rowscale[:, None], k, axis=1)).to(torch.bfloat16)
    return w, s


@pytest.mark.parametrize("sym", [False, True])
def test_quantize_near_ties_exact(sym):
    w, s = _near_tie_inputs(sym)
    gpu, ref = quantize_both(w, sym, s, 1.0)
    assert_quant_equal(gpu, ref, sym)


# -------------------------------------------------------------- linear ----

def linear_case(m, n, k, sym, seed, flags=0, std=0.02, n_out=0, out_scale=1.0, rows=None):
    w = synth.normal_weight(n, k, std, seed=seed, n_outliers=n_out, outlier_scale=out_scale)
    x = synth.normal_activations(m, k, seed=seed + 1)
    qw, sc, zr = w4.quantize_pack(w.to(DEV), sym)
    y = w4.w4a16_linear(x.to(DEV), qw, sc, zr, flags=flags)
    torch.cuda.synchronize()
    codes = O.unpack_codes(qw.cpu().numpy())
    # the oracle dequantizes its OWN quantization (bit-equality is tested above)
    oc, os_, oz = O.quantize_rtn(synth.bits(w), sym)
    assert np.array_equal(codes, oc)
    what = O.dequantize(oc, os_, oz)
    xb = synth.bits(x)
    if rows is None:
        y_ref = O.linear(xb, what)
        return max_rel_err(y, y_ref)
    y_ref = O.linear_rows(xb, what, rows)
    return max_rel_err(y[torch.as_tensor(rows, device=DEV)], y_ref)


DECODE_KERNELS = {"auto": 0, "stream": w4.LINEAR_DECODE_STREAM, "tiled": w4.LINEAR_DECODE_TILED}


@pytest.mark.parametrize("kernel", ["auto", "stream", "tiled"])
@pytest.mark.parametrize("m", [1, 2, 3, 5, 8, 9, 15, 16])
@pytest.mark.parametrize("sym", [False, True])
def test_gemv_parity_ragged(m, sym, kernel):
    if kernel == "stream" and m > 8:
        pytest.skip("the streaming decode kernel takes at most 8 tokens")
    assert linear_case(m, 1000, 1024, sym, seed=100 + m, flags=DECODE_KERNELS[kernel]) <= Y_RTOL


@pytest.mark.parametrize("m", [1, 16])
def test_gemv_single_linear_2048_outliers(m):
    assert linear_case(m, 2048, 2048, False, seed=0, n_out=8, out_scale=20.0) <= Y_RTOL


@pytest.mark.parametrize("m,n,k", [(1, 7, 128), (8, 33, 128), (3, 100, 256), (4, 100, 1024),
                                   (2, 16, 2048), (6, 1, 384), (7, 4100, 640)])
@pytest.mark.parametrize("sym", [False, True])
def test_gemv_stream_small_and_split(m, n, k, sym):
    """Decode shapes that exercise the streaming kernel's edges: one group
    (K = 128), ragged 64-row units and 16-row tiles, N = 1, and K split over
    2 or 4 warps of a row block (few row blocks), plus one shape with more
    bundles than the grid has CTAs."""
    err = linear_case(m, n, k, sym, seed=1000 + m * 7 + n + k, flags=w4.LINEAR_DECODE_STREAM)
    assert err <= Y_RTOL


def test_gemv_stream_deterministic():
    """Split-K partial sums are reduced in a fixed order: repeated calls give
    identical bits."""
    w = synth.normal_weight(96, 2048, 0.02, seed=61)
    x = synth.normal_activations(5, 2048, seed=62).to(DEV)
    qw, sc, zr = w4.quantize_pack(w.to(DEV), False)
    y0 = w4.w4a16_linear(x, qw, sc, zr, flags=w4.LINEAR_DECODE_STREAM)
    y1 = w4.w4a16_linear(x, qw, sc, zr, flags=w4.LINEAR_DECODE_STREAM)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


@pytest.mark.parametrize("m", [24, 32])
def test_decode_default_up_to_32_rows(m):
    assert linear_case(m, 700, 1024, False, seed=150 + m) <= Y_RTOL


@pytest.mark.parametrize("m,n,k", [(33, 512, 8192), (64, 300, 17408), (130, 640, 4096),
                                   (300, 256, 6144)])
@pytest.mark.parametrize("sym", [False, True])
def test_prefill_split_k(m, n, k, sym):
    """Few tiles and long K: the prefill GEMM splits K over a cluster and
    adds the partial tiles through distributed shared memory."""
    assert linear_case(m, n, k, sym, seed=160 + m + n) <= Y_RTOL


@pytest.mark.parametrize("m,n,k", [(96, 8448, 4096), (1024, 5120, 17408)])
def test_prefill_split_k_four_way(m, n, k):
    """Four-way K splits of 128 x 256 and of 256 x 128 tiles, which the
    launch's time model picks for these shapes on B200."""
    rows = None if m <= 128 else np.sort(np.random.default_rng(m + n).choice(m, 128, replace=False))
    assert linear_case(m, n, k, False, seed=170 + m, rows=rows) <= Y_RTOL


def test_prefill_split_k_deterministic():
    w = synth.normal_weight(384, 8192, 0.02, seed=171)
    x = synth.normal_activations(48, 8192, seed=172).to(DEV)
    qw, sc, zr = w4.quantize_pack(w.to(DEV), False)
    y0 = w4.w4a16_linear(x, qw, sc, zr)
    y1 = w4.w4a16_linear(x, qw, sc, zr)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


@pytest.mark.parametrize("m", [17, 40, 64])
def test_gemv_forced_chunks(m):
    assert linear_case(m, 520, 640, False, seed=200 + m, flags=w4.LINEAR_FORCE_GEMV) <= Y_RTOL


@pytest.mark.parametrize("m,n,k", [(1, 256, 128), (17, 256, 256), (64, 1000, 640), (128, 256, 4096),
                                   (200, 520, 1024), (300, 4096, 512)])
@pytest.mark.parametrize("sym", [False, True])
def test_gemm_parity_ragged(m, n, k, sym):
    assert linear_case(m, n, k, sym, seed=300 + m + n, flags=w4.LINEAR_FORCE_GEMM) <= Y_RTOL


@pytest.mark.parametrize("k,n", [(4096, 4096), (4096, 11008), (11008, 4096)])
@pytest.mark.parametrize("m", [512, 2048])
def test_gemm_llama2_7b_shapes(k, n, m):
    rows = None if m == 512 else np.sort(np.random.default_rng(m + n).choice(m, 256, replace=False))
    assert linear_case(m, n, k, True, seed=400 + n, rows=rows) <= Y_RTOL


@pytest.mark.parametrize("k,n", [(5120, 17408), (17408, 5120), (5120, 10240)])
@pytest.mark.parametrize("m", [1, 8, 64, 512, 4096])
def test_linear_27b_shapes(k, n, m):
    rows = None if m <= 512 else np.sort(np.random.default_rng(m + n).choice(m, 128, replace=False))
    err = linear_case(m, n, k, True, seed=500 + n, std=0.015, n_out=k // 100, out_scale=10.0,
                      rows=rows)
    assert err <= Y_RTOL


@pytest.mark.parametrize("k,n", [(5120, 17408), (17408, 5120)])
@pytest.mark.parametrize("m", [1, 8])
def test_linear_27b_shapes_streaming_kernel(k, n, m):
    err = linear_case(m, n, k, True, seed=500 + n, std=0.015, n_out=k // 100, out_scale=10.0,
                      flags=w4.LINEAR_DECODE_STREAM)
    assert err <= Y_RTOL


# ----------------------------------------------------------------- AWQ ----

def test_awq_scales_bit_exact():
    x = synth.student_t_calibration(2048, 2048, seed=11)
    alphas = synth.alpha_grid(20)
    s = w4.awq_scales(x.to(DEV), alphas)
    torch.cuda.synchronize()
    ref = O.awq_scales(O.awq_channel_stat(synth.bits(x)), alphas)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def _same_pick(idx, values, what):
    """The GPU's index equals the oracle's (the lowest index of the least
    binary64 value); a different index is accepted only for a genuine tie,
    asserted on the oracle's own values (equal to 1e-12 relative, below the
    rounding of either binary64 computation)."""
    v = np.asarray(values, dtype=np.float64).ravel()
    ref = int(np.argmin(v))
    if idx != ref:
        assert abs(v[idx] - v[ref]) <= GENUINE_TIE_RTOL * v[ref], (
            f"{what}: GPU picked {idx}, oracle {ref} (relative gap "
            f"{(v[idx] - v[ref]) / v[ref]:.3e})")


def check_awq(x, w, alphas, shrinks, sym, seg=None):
    sse, arg = w4.awq_score_grid(x.to(DEV), w.to(DEV), alphas, shrinks, sym, seg_offsets=seg)
    torch.cuda.synchronize()
    sse = sse.cpu().numpy()
    arg = arg.cpu().numpy()
    ref, ref_arg = O.awq_score_grid(synth.bits(x), synth.bits(w), alphas, shrinks, sym, seg)
    rel = np.max(np.abs(sse - ref) / ref)
    assert rel <= SSE_RTOL, f"SSE relative error {rel:.3e}"
    c1 = O.no_clip_column(shrinks)
    n_seg = ref.shape[0]
    total = ref.sum(axis=0)
    for s_ in range(n_seg):
        t = ref[s_]
        _same_pick(arg[s_, 0], t, f"seg {s_} joint")
        _same_pick(arg[s_, 1], t[:, c1], f"seg {s_} alpha*")
        _same_pick(arg[s_, 2], t[arg[s_, 1]], f"seg {s_} shrink*")
        _same_pick(arg[s_, 3], t[arg[n_seg, 1]], f"seg {s_} shrink* at group alpha")
    _same_pick(arg[n_seg, 0], total, "group joint")
    _same_pick(arg[n_seg, 1], total[:, c1], "group alpha*")
    assert arg[n_seg, 2] == -1 and arg[n_seg, 3] == -1
    return rel, ref_arg, arg


@pytest.mark.parametrize("sym", [False, True])
def test_awq_grid_small_full_grid(sym):
    x = synth.student_t_calibration(256, 512, seed=21)
    w = synth.normal_weight(384, 512, 0.02, seed=22, n_outliers=4, outlier_scale=20.0)
    check_awq(x, w, synth.alpha_grid(20), synth.shrink_grid(10), sym)


def test_awq_grid_segments_ragged_tokens():
    x = synth.student_t_calibration(200, 640, seed=31)   # M not a multiple of 128
    w = synth.normal_weight(800, 640, 0.02, seed=32)      # three linears sharing x
    check_awq(x, w, synth.alpha_grid(8), synth.shrink_grid(4), False, seg=[0, 256, 528, 800])


def test_awq_grid_small_calibration_scale():
    """Small activation statistics (x * 2^-7) and small weights (sigma 0.005):
    without the operands' power-of-two normalisation the error operand would
    fall into fp16's subnormal range.  Full 20 x 10 grid, two linears."""
    x = (synth.student_t_calibration(512, 1024, seed=43).float() * 2.0 ** -7).to(torch.bfloat16)
    w = synth.normal_weight(640, 1024, 0.005, seed=44, n_outliers=4, outlier_scale=10.0)
    for sym in (False, True):
        check_awq(x, w, synth.alpha_grid(20), synth.shrink_grid(10), sym, seg=[0, 256, 640])


def test_awq_grid_qwen_k_proj_full_size():
    """One Qwen3-1.7B k_proj (2048 -> 1024) on 2048 heavy-tailed calibration
    tokens, the full 20 x 10 grid."""
    x = synth.student_t_calibration(2048, 2048, seed=41)
    w = synth.normal_weight(1024, 2048, 0.02, seed=42)
    check_awq(x, w, synth.alpha_grid(20), synth.shrink_grid(10), False)


# ------------------------------------ per-output-channel clipping ----

# Per-row errors: each row's sum has only M * K products (no averaging over
# rows), so the fp16 operand rounding (2^-11 relative on each of x/s and the
# error operand) can move one row's value by up to ~4 * 2^-11 ~ 2e-3; below
# half the library's per-row tie tolerance (5e-3).
ROW_SSE_RTOL = 2e-3


def check_clip_rows(x, w, shrinks, sym, alpha):
    s = None
    s_ref = None
    if alpha is not None:
        s = w4.awq_scales(x.to(DEV), [alpha])[0].contiguous()
        s_ref = O.awq_scales(O.awq_channel_stat(synth.bits(x)), [alpha])[0]
        torch.cuda.synchronize()
        assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    sse, choice, rows = w4.awq_clip_search_rows(x.to(DEV), w.to(DEV), shrinks, sym, awq_s=s)
    torch.cuda.synchronize()
    sse = sse.cpu().numpy()
    choice = choice.cpu().numpy()
    ref, ref_choice = O.clip_search_rows(synth.bits(x), synth.bits(w), s_ref, shrinks, sym)
    rel = np.max(np.abs(sse - ref) / ref)
    assert rel <= ROW_SSE_RTOL, f"per-row SSE relative error {rel:.3e}"
    n = ref.shape[1]
    # Every row's pick equals the oracle's, but for genuine ties of the
    # oracle's own binary64 values.
    differ = np.flatnonzero(choice != ref_choice)
    picked = ref[choice[differ], differ]
    best = ref[ref_choice[differ], differ]
    assert np.all(np.abs(picked - best) <= GENUINE_TIE_RTOL * best), (
        f"{len(differ)} of {n} rows differ from the oracle's pick")
    assert np.allclose(rows.cpu().numpy(), np.asarray(shrinks, np.float32)[choice])
    # Deploy: quantize with the chosen ratios, bit-exact against the oracle.
    qw, sc, zr = w4.quantize_pack_rows(w.to(DEV), sym, rows, awq_s=s)
    torch.cuda.synchronize()
    oq, os_, oz = O.quantize_pack_rows(synth.bits(w), sym, s_ref, np.asarray(shrinks, np.float32)[choice])
    assert_quant_equal((qw, sc, zr), (oq, os_, oz), sym)
    return rel


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("alpha", [None, 0.5])
def test_clip_rows_small(sym, alpha):
    x = synth.student_t_calibration(200, 640, seed=81)   # ragged token tile
    w = synth.normal_weight(300, 640, 0.02, seed=82, n_outliers=6, outlier_scale=20.0)
    check_clip_rows(x, w, synth.shrink_grid(10), sym, alpha)


def test_clip_rows_qwen_k_proj_full_size():
    """One Qwen3-1.7B k_proj (2048 -> 1024) on 2048 heavy-tailed calibration
    tokens, the 10-point shrink grid at alpha 0.5."""
    x = synth.student_t_calibration(2048, 2048, seed=83)
    w = synth.normal_weight(1024, 2048, 0.02, seed=84)
    check_clip_rows(x, w, synth.shrink_grid(10), False, 0.5)


@pytest.mark.parametrize("sym", [False, True])
def test_quantize_rows_uniform_equals_per_linear(sym):
    w = synth.normal_weight(257, 1024, 0.02, seed=85, n_outliers=4, outlier_scale=20.0).to(DEV)
    rows = torch.full((257,), 0.8, dtype=torch.float32, device=DEV)
    a = w4.quantize_pack_rows(w, sym, rows)
    b = w4.quantize_pack(w, sym, None, 0.8)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert (u is None and v is None) or torch.equal(u, v)


# ------------------------------------------------------------- W4A8 ----

A8_PERM = (0, 4, 1, 5, 2, 6, 3, 7)  # stored order of the channels of a chunk


def unpermute_act(xq):
    """Channel order of w4_quantize_act_int8's codes back to natural order."""
    m, k = xq.shape
    out = np.empty_like(xq)
    c = xq.reshape(m, k // 8, 8)
    o = out.reshape(m, k // 8, 8)
    for p, ch in enumerate(A8_PERM):
        o[:, :, ch] = c[:, :, p]
    return out


def check_act_int8(x):
    xq, xs, sc = w4.quantize_act_int8(x.to(DEV))
    torch.cuda.synchronize()
    q_ref, sc_ref = O.quantize_act_int8(synth.bits(x))
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), sc_ref.view(np.uint32))
    q = unpermute_act(xq.cpu().numpy())
    assert np.array_equal(q, q_ref)
    m, k = q_ref.shape
    assert np.array_equal(xs.cpu().numpy(), q_ref.astype(np.int64).reshape(m, k // 128, 128).sum(2))
    return (xq, xs, sc), (q_ref, sc_ref)


@pytest.mark.parametrize("m,k", [(1, 128), (5, 2048), (16, 6144), (3, 81920)])
def test_act_int8_bit_exact(m, k):
    x = synth.normal_activations(m, k, seed=90 + m)
    if m > 2:
        xb = x.clone()
        xb[1] = 0  # a zero row: scale 0, codes 0
        x = xb
    check_act_int8(x)


def w4a8_case(m, n, k, sym, seed, std=0.02, n_out=0, out_scale=1.0):
    w = synth.normal_weight(n, k, std, seed=seed, n_outliers=n_out, outlier_scale=out_scale)
    x = synth.normal_activations(m, k, seed=seed + 1)
    (xq, xs, sc), (q_ref, sc_ref) = check_act_int8(x)
    qw, s16, z16 = w4.quantize_pack(w.to(DEV), sym)
    y = w4.w4a8_linear(xq, xs, sc, qw, s16, z16)
    torch.cuda.synchronize()
    oc, os_, oz = O.quantize_rtn(synth.bits(w), sym)
    y_ref = O.w4a8_linear(q_ref, sc_ref, oc, os_, oz)
    return y.float().cpu().numpy().astype(np.float64), y_ref


# W4A8 bar: the group dots are exact on both sides; the GPU's binary32
# scaling and group sum add a few ulps, and y is rounded once to bf16
# (half an ulp, 2^-9 relative), so each element must lie within
# 2^-8 |y_ref| + 1e-4 max|y_ref| of the binary64 oracle.
def assert_w4a8_close(y, y_ref):
    bound = 2.0 ** -8 * np.abs(y_ref) + 1e-4 * np.max(np.abs(y_ref))
    assert np.all(np.abs(y - y_ref) <= bound), float(np.max(np.abs(y - y_ref) / bound))


@pytest.mark.parametrize("m", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("sym", [False, True])
def test_w4a8_linear_ragged(m, sym):
    assert_w4a8_close(*w4a8_case(m, 1000, 1024, sym, seed=1100 + m))


@pytest.mark.parametrize("k,n", [(5120, 17408), (17408, 5120)])
@pytest.mark.parametrize("m", [1, 8])
def test_w4a8_27b_shapes(k, n, m):
    assert_w4a8_close(*w4a8_case(m, n, k, True, seed=1200 + n, std=0.015, n_out=k // 100,
                                 out_scale=10.0))


@pytest.mark.parametrize("m", [1, 4, 16])
def test_w4a8_batched_qwen_block_shared_x(m):
    """The seven Qwen linears, each input quantized once and shared where the
    block shares it (q, k, v; gate, up), in one batched call."""
    xs_by_k = {}
    items, refs = [], []
    for i, (_name, k, n) in enumerate(synth.QWEN3_1P7B_BLOCK):
        if k not in xs_by_k:
            x = synth.normal_activations(m, k, seed=1300 + k)
            xs_by_k[k] = check_act_int8(x)
        (xq, xsm, sc), (q_ref, sc_ref) = xs_by_k[k]
        w = synth.normal_weight(n, k, 0.02, seed=1400 + i)
        qw, s16, z16 = w4.quantize_pack(w.to(DEV), False)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
        items.append((xq, xsm, sc, qw, s16, z16, y))
        oc, os_, oz = O.quantize_rtn(synth.bits(w), False)
        refs.append(O.w4a8_linear(q_ref, sc_ref, oc, os_, oz))
    w4.w4a8_linear_batched(items, m)
    torch.cuda.synchronize()
    for it, ref in zip(items, refs):
        assert_w4a8_close(it[6].float().cpu().numpy().astype(np.float64), ref)


# ------------------------------------------------------ failure path ----

def test_bounded_wait_reports_and_context_survives():
    w4.device_error(clear=True)
    w4.selftest_bounded_wait(20_000_000)  # 20 ms
    torch.cuda.synchronize()
    code = w4.device_error(clear=True)
    assert code & 1 and (code >> 16) == 7
    assert w4.device_error(clear=True) == 0
    # the context is still usable
    assert linear_case(4, 256, 256, False, seed=9) <= Y_RTOL


# ------------------------------------------------------------- batched ----

@pytest.mark.parametrize("sym", [False, True])
def test_quantize_batched_mixed_tensors(sym):
    shapes = [(n, k) for _, k, n in synth.QWEN3_1P7B_BLOCK] + [(3, 384), (17, 256)]
    x = synth.student_t_calibration(64, 2048, seed=71)
    s2048 = O.awq_scales(O.awq_channel_stat(synth.bits(x)), [0.5])[0]
    items, refs = [], []
    for i, (n, k) in enumerate(shapes):
        w = synth.normal_weight(n, k, 0.02, seed=700 + i, n_outliers=4, outlier_scale=20.0)
        s = s2048 if (k == 2048 and i % 2 == 0) else None
        r = (1.0, 0.9, 0.75)[i % 3]
        qw = torch.empty(n, k // 8, dtype=torch.int32, device=DEV)
        sc = torch.empty(n, k // 128, dtype=torch.int16, device=DEV)
        zr = None if sym else torch.empty(n, k // 128, dtype=torch.int16, device=DEV)
        s_dev = None if s is None else torch.from_numpy(s).to(DEV)
        items.append((w.to(DEV), s_dev, r, qw, sc, zr))
        refs.append(O.quantize_pack(synth.bits(w), sym, s, r))
    w4.quantize_pack_batched(items, sym)
    torch.cuda.synchronize()
    for (w_, s_, r_, qw, sc, zr), ref in zip(items, refs):
        assert_quant_equal((qw, sc, zr), ref, sym)


@pytest.mark.parametrize("sym", [False, True])
def test_prefill_grouped_many_linears(sym):
    """More linears than one grouped prefill launch takes (16), mixed K and
    ragged N, at a ragged token count: every result meets the bound."""
    rng = np.random.default_rng(9)
    items, refs = [], []
    for i in range(21):
        k = int(rng.choice([128, 384, 1024]))
        n = int(rng.integers(1, 600))
        w = synth.normal_weight(n, k, 0.02, seed=4000 + i)
        x = synth.normal_activations(130, k, seed=7000 + i)
        qw, sc, zr = w4.quantize_pack(w.to(DEV), sym)
        y = torch.empty(130, n, dtype=torch.bfloat16, device=DEV)
        items.append((x.to(DEV), qw, sc, zr, y))
        oc, os_, oz = O.quantize_rtn(synth.bits(w), sym)
        refs.append(O.linear(synth.bits(x), O.dequantize(oc, os_, oz)))
    w4.w4a16_linear_batched(items, 130)
    torch.cuda.synchronize()
    worst = max(max_rel_err(it[4], ref) for it, ref in zip(items, refs))
    assert worst <= Y_RTOL


def test_linear_batched_more_than_one_launch():
    """More linears than one streaming launch takes (STREAM_BATCH), mixed K
    and ragged N, at 3 tokens: every result meets the bound."""
    rng = np.random.default_rng(5)
    count = w4.STREAM_BATCH + 44
    items, refs = [], []
    for i in range(count):
        k = int(rng.choice([128, 256, 384, 1024]))
        n = int(rng.integers(1, 70))
        w = synth.normal_weight(n, k, 0.02, seed=3000 + i)
        x = synth.normal_activations(3, k, seed=6000 + i)
        qw, sc, zr = w4.quantize_pack(w.to(DEV), False)
        y = torch.empty(3, n, dtype=torch.bfloat16, device=DEV)
        items.append((x.to(DEV), qw, sc, zr, y))
        oc, os_, oz = O.quantize_rtn(synth.bits(w), False)
        refs.append(O.linear(synth.bits(x), O.dequantize(oc, os_, oz)))
    for kernel in ("auto", "stream"):
        for it in items:
            it[4].zero_()
        w4.w4a16_linear_batched(items, 3, DECODE_KERNELS[kernel])
        torch.cuda.synchronize()
        worst = max(max_rel_err(it[4], ref) for it, ref in zip(items, refs))
        assert worst <= Y_RTOL, kernel


@pytest.mark.parametrize("kernel", ["auto", "stream", "tiled"])
@pytest.mark.parametrize("m", [1, 5, 8, 16, 40, 200])
@pytest.mark.parametrize("sym", [False, True])
def test_linear_batched_qwen_block(m, sym, kernel):
    if kernel == "stream" and m > 8:
        pytest.skip("the streaming decode kernel takes at most 8 tokens")
    if kernel == "tiled" and m > 64:
        pytest.skip("the tensor-map decode kernel takes at most 64 tokens")
    shapes = [(n, k) for _, k, n in synth.QWEN3_1P7B_BLOCK] + [(72, 640)]
    items, refs = [], []
    for i, (n, k) in enumerate(shapes):
        w = synth.normal_weight(n, k, 0.02, seed=800 + i)
        x = synth.normal_activations(m, k, seed=900 + i)
        qw, sc, zr = w4.quantize_pack(w.to(DEV), sym)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=DEV)
        items.append((x.to(DEV), qw, sc, zr, y))
        oc, os_, oz = O.quantize_rtn(synth.bits(w), sym)
        refs.append(O.linear(synth.bits(x), O.dequantize(oc, os_, oz)))
    w4.w4a16_linear_batched(items, m, DECODE_KERNELS[kernel])
    torch.cuda.synchronize()
    for (x, qw, sc, zr, y), ref in zip(items, refs):
        assert max_rel_err(y, ref) <= Y_RTOL


# --------------------------------------------- bench configuration ----

def test_bench_configuration_sampled():
    """The bench's launch configuration at full size: 28 Qwen3-1.7B-shaped
    blocks (196 linears, bf16 N(0, 0.02)), one batched quantize+pack and one
    batched decode per token count (M = 1, 4, 8) with programmatic dependent
    launch and static weights, as bench.py times them.  Sampled rows of
    sampled linears are checked against the oracle: codes, scales and zeros
    bit-exact, y within the linear bound."""
    rng = np.random.default_rng(2024)
    g = torch.Generator(device=DEV)
    lin = []
    for b in range(28):
        for i, (_name, k, n) in enumerate(synth.QWEN3_1P7B_BLOCK):
            g.manual_seed(5000 + 7 * b + i)
            w = (torch.randn(n, k, generator=g, device=DEV) * 0.02).to(torch.bfloat16)
            qw = torch.empty(n, k // 8, dtype=torch.int32, device=DEV)
            sc = torch.empty(n, k // 128, dtype=torch.int16, device=DEV)
            zr = torch.empty(n, k // 128, dtype=torch.int16, device=DEV)
            lin.append((k, n, w, qw, sc, zr))
    w4.quantize_pack_batched([(w, None, 1.0, qw, sc, zr) for (k, n, w, qw, sc, zr) in lin], False)
    flags = w4.LINEAR_PDL | w4.LINEAR_STATIC_WEIGHTS
    xs = {}
    ys = {}
    for m in (1, 4, 8):
        for k in {k for k, *_ in lin}:
            g.manual_seed(77 + 10 * m + k)
            xs[(m, k)] = torch.randn(m, k, generator=g, device=DEV).to(torch.bfloat16)
        ys[m] = [torch.empty(m, n, dtype=torch.bfloat16, device=DEV) for (k, n, *_r) in lin]
        w4.w4a16_linear_batched([(xs[(m, k)], qw, sc, zr, y) for (k, n, w, qw, sc, zr), y in
                                 zip(lin, ys[m])], m, flags)
    torch.cuda.synchronize()
    for j in rng.choice(len(lin), 12, replace=False):
        k, n, w, qw, sc, zr = lin[j]
        rows = np.sort(rng.choice(n, 16, replace=False))
        rt = torch.as_tensor(rows, device=DEV)
        wb = synth.bits(w[rt].cpu())
        oq, os_, oz = O.quantize_pack(wb, False)
        assert np.array_equal(qw[rt].cpu().numpy(), oq)
        assert np.array_equal(u16(sc[rt]), os_)
        assert np.array_equal(u16(zr[rt]), oz)
        what = O.dequantize(*O.quantize_rtn(wb, False))
        for m in (1, 4, 8):
            ref = O.linear(synth.bits(xs[(m, k)].cpu()), what)
            y = ys[m][j][:, rt]
            assert max_rel_err(y, ref) <= Y_RTOL, (j, m)
