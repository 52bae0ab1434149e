"""Mutation check of the block-level scoring oracle's pins: each plausible
mistake is planted in a copy of oracle/block_oracle.py (CPU only) and at
least one pin of tests/test_block_oracle_pins.py must fail on it."""
import os
import types

import numpy as np
import pytest

from tests import test_block_oracle_pins as P

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "block_oracle.py")

MUTANTS = [
    ("rotary sign", "x1 * c - x2 * s", "x1 * c + x2 * s"),
    ("rotary frequency", "theta ** (-2.0 * np.arange(half) / d)", "theta ** (-1.0 * np.arange(half) / d)"),
    ("causal mask one step late", "np.triu(np.ones((t, t), dtype=bool), 1)",
     "np.triu(np.ones((t, t), dtype=bool), 2)"),
    ("key head mapping", "s = q[:, h] @ k[:, h // group].T", "s = q[:, h] @ k[:, h % k.shape[1]].T"),
    ("attention scale", "@ k[:, h // group].T / np.sqrt(d)", "@ k[:, h // group].T / d"),
    ("RMSNorm epsilon outside the root", "np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)",
     "(np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps)"),
    ("q norm skipped", 'q = rms_norm((h @ w["q"].T).reshape(t, hq, d), w["q_norm"], eps)',
     'q = (h @ w["q"].T).reshape(t, hq, d)'),
    ("MLP residual dropped", 'return x1 + act @ w["down"].T', 'return act @ w["down"].T'),
    ("SiLU as sigmoid", "return x / (1.0 + np.exp(-x))", "return 1.0 / (1.0 + np.exp(-x))"),
    ("reference not taken through block i+1",
     "ref = out_i if w_next is None else block_forward(out_i, w_next, cfg)", "ref = out_i"),
    ("AWQ statistic over the hidden axis", "stat = np.mean(np.abs(acts[group]), axis=0)",
     "stat = np.mean(np.abs(acts[group]), axis=1)"),
]


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mod = types.ModuleType("block_oracle_mutant")
    exec(compile(src.replace(old, new), "block_oracle_mutant", "exec"), mod.__dict__)
    return mod


def _pins():
    return [getattr(P, n) for n in dir(P) if n.startswith("test_")]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(monkeypatch, name, old, new):
    mut = _mutant(old, new)
    monkeypatch.setattr(P, "B", mut)
    for fn in _pins():
        try:
            with np.errstate(all="ignore"):
                fn()
        except Exception:
            return  # caught
    pytest.fail(f"no pin caught the planted mistake: {name}")
