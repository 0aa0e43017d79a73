"""The chunked backward oracle equals the sequential one.

oracle/backward.py is pinned by central finite differences of the forward oracle
(tests/test_oracle.py); the chunked derivation (oracle/backward_chunked.py) must give the
same gradients for every chunk size, on ragged sequences (empty ones, lengths that are
not multiples of the chunk), with grouped heads, an initial state, a final-state gradient
and a read-out scale.  A planted mistake in each backward step must break that equality.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle.backward_chunked as BC
from oracle.backward import backward


def _case(seed, lens, H_qk=2, H_v=4, dk=6, dv=5):
    rng = np.random.default_rng(seed)
    T = int(sum(lens))
    q = rng.standard_normal((T, H_qk, dk))
    k = rng.standard_normal((T, H_qk, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H_v, dv))
    g = -np.log1p(np.exp(rng.standard_normal((T, H_v))))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H_v))))
    S0 = rng.standard_normal((len(lens), H_v, dk, dv)) * 0.3
    d_out = rng.standard_normal((T, H_v, dv))
    dSf = rng.standard_normal((len(lens), H_v, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return q, k, v, g, beta, S0, d_out, dSf, cu


def _rel(a, b):
    den = np.max(np.abs(b))
    return np.max(np.abs(a - b)) / den if den > 0 else np.max(np.abs(a - b))


@pytest.mark.parametrize("chunk", [1, 3, 16, 64])
def test_chunked_backward_equals_sequential(chunk):
    q, k, v, g, beta, S0, d_out, dSf, cu = _case(1, [0, 5, 64, 65, 130])
    want = backward(q, k, v, g, beta, S0, d_out, dSf, cu, scale=0.7)
    got = BC.backward_chunked(q, k, v, g, beta, S0, d_out, dSf, cu, scale=0.7, chunk=chunk)
    for name, a, b in zip(("dq", "dk", "dv", "dg", "dbeta", "dS0"), got, want):
        assert _rel(a, b) < 1e-9, (name, chunk, _rel(a, b))


def test_chunked_backward_strong_decay_and_no_state():
    q, k, v, g, beta, S0, d_out, dSf, cu = _case(2, [200], H_qk=1, H_v=1)
    g = g * 3.0                                     # in-chunk decays down to e^-60 and below
    want = backward(q, k, v, g, beta, None, d_out, None, cu)
    got = BC.backward_chunked(q, k, v, g, beta, None, d_out, None, cu, chunk=64)
    for a, b in zip(got, want):
        assert _rel(a, b) < 1e-9


# planted mistakes, one per backward step, each must break the equality
MUTANTS = [
    ("dU = P.T @ dOs + Kd @ dS1", "dU = P.T @ dOs", "state gradient not fed to U"),
    ("dS0 = (gam[:, None] * q).T @ dOs + gam[-1] * dS1 - W.T @ dU",
     "dS0 = (gam[:, None] * q).T @ dOs + gam[-1] * dS1 + W.T @ dU", "sign of W^T dU"),
    ("dA = np.where(f[\"low_strict\"], -T.T @ dT @ T.T, 0.0)",
     "dA = np.where(f[\"low_strict\"], -T @ dT @ T, 0.0)", "inverse gradient untransposed"),
    ("dG -= ddec", "dG += ddec", "decay-to-end gradient sign"),
    ("dg = np.cumsum(dG[::-1])[::-1]", "dg = np.cumsum(dG)", "forward instead of reverse cumsum"),
    ("dk += dKK @ k + dKK.T @ k", "dk += dKK @ k", "one side of k k^T dropped"),
    ("dbeta += np.einsum(\"id,id->i\", dVb, v)", "dbeta += 0.0", "beta's V term dropped"),
]


@pytest.mark.parametrize("old,new,what", MUTANTS, ids=[m[2] for m in MUTANTS])
def test_mutants_break_the_equality(old, new, what):
    import types
    src = open(BC.__file__).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("bc_mutant")
    mod.__dict__["__package__"] = "oracle"
    exec(compile(src.replace(old, new), "bc_mutant.py", "exec"), mod.__dict__)
    q, k, v, g, beta, S0, d_out, dSf, cu = _case(3, [70, 9])
    want = backward(q, k, v, g, beta, S0, d_out, dSf, cu, scale=0.7)
    got = mod.backward_chunked(q, k, v, g, beta, S0, d_out, dSf, cu, scale=0.7, chunk=16)
    assert max(_rel(a, b) for a, b in zip(got, want)) > 1e-3, what
