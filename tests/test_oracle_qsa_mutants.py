"""The QSA oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of oracle/qsa.py (loaded as a separate module
on the CPU) and runs the pin battery of tests/test_oracle_qsa.py against it; at least
one pin must fail for every mutant.
"""
from __future__ import annotations

import os
import types

import pytest

import test_oracle_qsa as T
from oracle import qsa

SRC = os.path.join(os.path.dirname(os.path.abspath(qsa.__file__)), "qsa.py")

# (exact text, replacement, what the mistake is)
MUTANTS = [
    ("out[..., half:rope_dims] = x2 * c + x1 * s", "out[..., half:rope_dims] = x2 * c - x1 * s",
     "wrong sign in the rotation"),
    ("inv_freq = base ** (-2.0 *", "inv_freq = base ** (-1.0 *",
     "rotary frequencies without the factor 2"),
    ("rope_partial(pooled, p0[n] + r * b,", "rope_partial(pooled, p0[n] + r * b + r - 1,",
     "pooled key placed at the block's last token"),
    ("pooled = k[t0:t0 + r].mean(axis=0)\n            out[cu_blocks[n] + b] = rope_partial(pooled, p0[n] + r * b, rope_dims, base)",
     "out[cu_blocks[n] + b] = rope_partial(k[t0:t0 + r], p0[n] + r * b + np.arange(r), rope_dims, base).mean(axis=0)",
     "rotation before pooling (each token at its own position)"),
    ("return max(0, min(int(n_blocks), (int(q_pos) + 1) // r))",
     "return max(0, min(int(n_blocks), int(q_pos) // r + 1))",
     "the block holding the query counted as complete"),
    ("key=lambda b: (-scores[b], b))", "key=lambda b: (-scores[b], -b))",
     "ties go to the later block"),
    ("for h in range(qh.shape[0]):", "for h in range(qh.shape[0] - 1):",
     "one query head dropped"),
    ("return np.array(sorted(order[:budget]), np.int64)", "return np.array(order[:budget], np.int64)",
     "kept blocks in rank order, not block order"),
    ("return np.array([r * int(b) + j for b in blocks for j in range(r)], np.int64)",
     "return np.array([r * int(b) + j + 1 for b in blocks for j in range(r)], np.int64)",
     "expansion off by one token"),
    ("x1, x2 = x[..., :half], x[..., half:rope_dims]",
     "x1, x2 = x[..., half:rope_dims], x[..., :half]",
     "rotation pairs swapped"),
]


def _mutant_module(old: str, new: str):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("qsa_mutant")
    exec(compile(src.replace(old, new), "qsa_mutant.py", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("old,new,what", MUTANTS, ids=[m[2] for m in MUTANTS])
def test_mutant_is_caught(old, new, what):
    Q = _mutant_module(old, new)
    caught = []
    for name, fn in T.BATTERY:
        try:
            fn(Q)
        except (AssertionError, ValueError, IndexError):
            caught.append(name)
    assert caught, f"no pin caught: {what}"


def test_unmutated_copy_passes():
    Q = _mutant_module("R = 4 ", "R = 4 ")
    for _, fn in T.BATTERY:
        fn(Q)
