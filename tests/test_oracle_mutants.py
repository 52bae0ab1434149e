"""Mutation check of the oracle's pins: each plausible mistake is planted in a
copy of the oracle's source (CPU only) and at least one pin must fail on it."""
import os
import types

import numpy as np
import pytest

from tests import test_oracle_pins as P

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "w4_oracle.py")

MUTANTS = [
    ("ties away from zero in codes", "t = np.rint(vg / sc[:, :, None])",
     "t = np.floor(0.5 + vg / sc[:, :, None])"),
    ("asym divisor 16", "np.float32(15.0)", "np.float32(16.0)"),
    ("sym divisor 8", "np.float32(7.0)", "np.float32(8.0)"),
    ("zero-point sign", "np.rint(-mn / sc)", "np.rint(mn / sc)"),
    ("codes from unrounded scale", "t = np.rint(vg / sc[:, :, None])",
     "t = np.rint(vg / scale32[:, :, None])"),
    ("shrink dropped on max", "mx = r * np.max(vg, axis=2)", "mx = np.max(vg, axis=2)"),
    ("shrink dropped on absmax", "a = r * np.max(np.abs(vg), axis=2)", "a = np.max(np.abs(vg), axis=2)"),
    ("AWQ s applied the wrong way", "return w - w_hat / np.asarray(s", "return w - w_hat * np.asarray(s"),
    ("AWQ s not applied before quantization",
     "v = w if awq_s is None else w * np.asarray(awq_s, dtype=np.float32)[None, :]", "v = w"),
    ("linear nibble order", "word |= c[:, :, j] << np.uint32(4 * i)",
     "word |= c[:, :, i] << np.uint32(4 * i)"),
    ("fp16 ties away", "up = (rem > half) | ((rem == half) & ((q & np.uint64(1)) == 1))",
     "up = rem >= half"),
    ("fp16 truncation", "up = (rem > half) | ((rem == half) & ((q & np.uint64(1)) == 1))",
     "up = rem < 0"),
    ("stat over the wrong axis", "np.abs(x).sum(axis=0) / x.shape[0]", "np.abs(x).sum(axis=0) / x.shape[1]"),
    ("dequant adds the zero", "((q - z[:, :, None]) * sc[:, :, None])", "((q + z[:, :, None]) * sc[:, :, None])"),
    ("linear against the untransposed weight", "return x @ np.asarray(w_hat, dtype=np.float64).T",
     "return x @ np.asarray(w_hat, dtype=np.float64).T[::-1, ::-1]"),
    ("range floor dropped", "np.maximum(mx - mn, floor)", "(mx - mn)"),
    ("per-row error summed over tokens' complement", "sse[j] = np.sum(y * y, axis=0)",
     "sse[j] = np.sum(y * y, axis=0)[::-1]"),
    ("per-row choice takes the last minimum", "return sse, np.argmin(sse, axis=0)",
     "return sse, len(shrinks) - 1 - np.argmin(sse[::-1], axis=0)"),
    ("activation scale over 128", "scale = (amax / np.float32(127.0))", "scale = (amax / np.float32(128.0))"),
    ("activation codes rounded away from zero", "t = np.rint(x / scale[:, None])",
     "t = np.trunc(x / scale[:, None] + np.copysign(0.5, x))"),
    ("W4A8 zero point dropped", "w = codes.astype(np.int64).reshape(n, g, group) - z[:, :, None]",
     "w = codes.astype(np.int64).reshape(n, g, group)"),
    ("W4A8 activation scale dropped", "return np.asarray(xscale, dtype=np.float64)[:, None] * np.einsum",
     "return np.ones_like(np.asarray(xscale, dtype=np.float64))[:, None] * np.einsum"),
    ("per-row ratios applied to the wrong rows",
     "np.asarray(shrink, dtype=np.float32).reshape(n, 1)",
     "np.asarray(shrink, dtype=np.float32)[::-1].reshape(n, 1)"),
]


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mod = types.ModuleType("w4_oracle_mutant")
    exec(compile(src.replace(old, new), "w4_oracle_mutant", "exec"), mod.__dict__)
    return mod


def _all_pins():
    yield from ((P.test_fp16_rne_golden, a) for a in P._fp16_cases())
    yield from ((P.test_rtn_golden_groups, (c,)) for c in P._golden_cases())
    yield P.test_pack_layout_little_endian_nibbles, ()
    for sym in (False, True):
        yield P.test_codes_brute_force_nearest_grid_point, (sym, 1.0)
        yield P.test_awq_sse_brute_force_tiny, (sym,)
    yield P.test_zero_point_brute_force, ()
    yield P.test_weight_mse_closed_form_uniform, ()
    yield P.test_dequant_is_exact, ()
    yield P.test_linear_exact_rational_small, ()
    yield P.test_linear_closed_form_constant_weight, ()
    yield P.test_awq_scale_stat_and_pow_brute_force, ()
    for sym in (False, True):
        yield P.test_clip_rows_sse_brute_force_tiny, (sym,)
        yield P.test_quantize_rows_reduces_to_per_linear_quantize, (sym,)
    yield P.test_clip_rows_ties_take_the_lowest_index, ()
    yield P.test_act_int8_brute_force, ()
    yield P.test_act_int8_ties_to_even_hand_case, ()
    for sym in (False, True):
        yield P.test_w4a8_linear_exact_rational_small, (sym,)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(monkeypatch, name, old, new):
    mut = _mutant(old, new)
    monkeypatch.setattr(P, "O", mut)
    for fn, args in _all_pins():
        try:
            with np.errstate(all="ignore"):
                fn(*args)
        except Exception:
            return  # caught
    pytest.fail(f"no pin caught the planted mistake: {name}")
