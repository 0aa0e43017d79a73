"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU, in a
temporary directory), builds it, points the oracle wrapper at the mutant and runs
the pin battery of tests/test_oracle.py.  A mutant that no pin catches would mean
the oracle is not pinned against that kind of error.
"""
from __future__ import annotations

import os
import shutil

import pytest

import oracle
import test_oracle as T

ORACLE_DIR = os.path.dirname(os.path.abspath(oracle.__file__))

# (file, exact text, replacement, what the mistake is)
MUTANTS = [
    ("recurrence.inc", "- alpha * b * kt[i] * kTS[j]", "- b * kt[i] * kTS[j]",
     "alpha dropped from the erase term (the concept code's variant)"),
    ("recurrence.inc", "- alpha * b * kt[i] * kTS[j]", "+ alpha * b * kt[i] * kTS[j]",
     "wrong sign on the erase term"),
    ("recurrence.inc", "+ b * kt[i] * vt[j]", "+ kt[i] * vt[j]",
     "beta dropped from the write term"),
    ("recurrence.inc", "const int hq = h / group;", "const int hq = h % A->H_qk;",
     "wrong q/k head for a value head"),
    ("recurrence.inc", "const REAL alpha = EXP(g[(size_t)t * A->H_v + h]);",
     "const REAL alpha = EXP((REAL)0.5 * g[(size_t)t * A->H_v + h]);",
     "wrong gate mapping"),
    ("recurrence.inc", "ot[j] = scale * acc;", "ot[j] = acc;", "read-out scale ignored"),
    ("recurrence.inc", "acc += S[(size_t)i * dv + j] * qt[i];",
     "acc += S[(size_t)i * dv + j] * kt[i];", "read-out with k instead of q"),
    ("recurrence.inc", "    if (S0)\n        memcpy(S, S0", "    if (0)\n        memcpy(S, S0",
     "initial state ignored"),
    ("recurrence.inc", "for (int i = 0; i < dk; ++i) acc += kt[i] * S[(size_t)i * dv + j];",
     "for (int i = 0; i < dk - 1; ++i) acc += kt[i] * S[(size_t)i * dv + j];",
     "dropped term in k^T S"),
    ("gdn_oracle.c", "O[i * dv + e] = exp(G[i]) * qs + pu;", "O[i * dv + e] = qs + pu;",
     "chunked form: decay missing on Q S"),
    ("gdn_oracle.c", "for (int m = j; m < i; ++m) acc -= Am[i * C + m] * T[m * C + j];",
     "for (int m = j; m < i; ++m) acc += Am[i * C + m] * T[m * C + j];",
     "chunked form: wrong sign in the triangular inverse"),
    ("gdn_oracle.c", "P[i * C + j] = (j <= i) ? exp(G[i] - G[j]) * qk : 0.0;",
     "P[i * C + j] = (j < i) ? exp(G[i] - G[j]) * qk : 0.0;",
     "chunked form: diagonal of the intra-chunk scores dropped"),
]


def _battery():
    return [
        ("golden", lambda: T.test_golden_handworked_oracle("f64", 1e-14)),
        ("brute", lambda: [T.test_bruteforce_exact(*a) for a in
                           [(1, 5, 2, 3), (3, 16, 6, 5)]]),
        ("brute_gva_varlen", T.test_bruteforce_exact_multihead_varlen),
        ("pure_decay", T.test_pure_decay_closed_form),
        ("unit_write", T.test_unit_write_recalls_value),
        ("orthonormal", T.test_orthonormal_keys_store_all_pairs),
        ("chunked", lambda: [T.test_chunked_equals_sequential(C) for C in (1, 16, 64)]),
    ]


@pytest.mark.parametrize("fname,old,new,what", MUTANTS, ids=[m[3] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, fname, old, new, what):
    for f in ("gdn_oracle.c", "recurrence.inc"):
        shutil.copy(os.path.join(ORACLE_DIR, f), tmp_path / f)
    path = tmp_path / fname
    src = path.read_text()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    path.write_text(src.replace(old, new))
    so = oracle.build(force=True, src=str(tmp_path / "gdn_oracle.c"), out=str(tmp_path / "m.so"))
    mutant = oracle.load(so)
    saved = oracle._lib
    oracle._lib = mutant
    caught = []
    try:
        for name, fn in _battery():
            try:
                fn()
            except (AssertionError, ValueError):
                caught.append(name)
    finally:
        oracle._lib = saved
    assert caught, f"no pin caught the mutant: {what}"
