"""CPU oracle for the gated delta rule — TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of bench.py
may import this package.  The CUDA library never imports, links or calls it,
and it shares no code with the CUDA path: the only common module is the seeded
input generator ``linear_attention_token_b200.inputs``.

What it computes ("論文解説: Qwen3.8-Next の設計", section "GDNの中身", Eq. (1)
and the one-token concept code beside it):

    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
    o_t = scale * S_t^T q_t          (read after the update),
    alpha_t = exp(g_t).

The arithmetic lives in ``gdn_oracle.c`` (plain C, compiled with gcc, no fast
math); this module only marshals numpy arrays.  Every function here is pinned
by tests/test_oracle.py (exact rational brute force, a hand-worked example,
closed forms and invariants) and by tests/test_oracle_mutants.py.  The backward passes live
in oracle/backward.py (sequential) and oracle/backward_chunked.py (chunked); the QSA
indexer in oracle/qsa.py; the segmented (sequence-parallel) form in oracle/segments.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc (-O2, strict IEEE: no -ffast-math)."""
    deps = [src, os.path.join(os.path.dirname(src), "recurrence.inc")]
    if (not force and os.path.exists(out)
            and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in deps if os.path.exists(d))):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-pthread",
           "-I", os.path.dirname(src), src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def load(path: Optional[str] = None):
    """Load (building first if needed) and return the ctypes handle."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    if _lib is None:
        build()
        _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _declare(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    D = ctypes.c_double
    common = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, D, I]
    lib.gdn_oracle_recurrent_f64.argtypes = common + [I]
    lib.gdn_oracle_recurrent_f32.argtypes = common + [I]
    lib.gdn_oracle_chunked_f64.argtypes = common + [I, I]
    for f in (lib.gdn_oracle_recurrent_f64, lib.gdn_oracle_recurrent_f32, lib.gdn_oracle_chunked_f64):
        f.restype = I
    lib.gdn_oracle_default_threads.restype = I
    return lib


def default_threads() -> int:
    return int(load().gdn_oracle_default_threads())


def _arr(x, dt):
    if x is None:
        return None
    if hasattr(x, "detach"):        # torch tensor -> numpy (exact upcast of bf16/fp32)
        import torch
        x = x.detach().to("cpu", torch.float64 if dt == np.float64 else torch.float32).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=dt))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _run(fn_name, q, k, v, g, beta, S0, cu_seqlens, scale, l2norm, threads, dt, extra=(),
         lib=None):
    lib = lib or load()
    q, k, v, g, beta, S0 = (_arr(x, dt) for x in (q, k, v, g, beta, S0))
    T, H_qk, dk = q.shape
    _, H_v, dv = v.shape
    assert k.shape == q.shape and v.shape[0] == T and g.shape == (T, H_v) and beta.shape == (T, H_v)
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    N = len(cu) - 1
    assert cu[0] == 0 and cu[-1] == T
    if S0 is not None:
        assert S0.shape == (N, H_v, dk, dv)
    out = np.zeros((T, H_v, dv), dtype=dt)
    S_final = np.zeros((N, H_v, dk, dv), dtype=dt)
    rc = getattr(lib, fn_name)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                               _ptr(out), _ptr(S_final), _ptr(cu), N, H_qk, H_v, dk, dv,
                               float(scale), int(bool(l2norm)), *extra, int(threads))
    if rc != 0:
        raise ValueError(f"{fn_name} rejected its arguments (rc={rc})")
    return out, S_final


def recurrent(q, k, v, g, beta, S0=None, cu_seqlens=None, scale: float = 1.0,
              l2norm: bool = False, threads: int = 0, precision: str = "f64", lib=None):
    """Sequential Eq. (1).  Returns (out [T,H_v,dv], S_final [N,H_v,dk,dv]) as numpy.

    ``precision`` "f64" is the parity oracle; "f32" is the timed CPU baseline.
    """
    if precision == "f64":
        return _run("gdn_oracle_recurrent_f64", q, k, v, g, beta, S0, cu_seqlens, scale,
                    l2norm, threads, np.float64, lib=lib)
    if precision == "f32":
        return _run("gdn_oracle_recurrent_f32", q, k, v, g, beta, S0, cu_seqlens, scale,
                    l2norm, threads, np.float32, lib=lib)
    raise ValueError(precision)


def chunked(q, k, v, g, beta, S0=None, cu_seqlens=None, scale: float = 1.0,
            l2norm: bool = False, chunk: int = 64, threads: int = 0, lib=None):
    """The chunked (WY / UT) re-association in fp64, chunk size ``chunk``."""
    return _run("gdn_oracle_chunked_f64", q, k, v, g, beta, S0, cu_seqlens, scale, l2norm,
                threads, np.float64, extra=(int(chunk),), lib=lib)


def decode_step(q, k, v, g, beta, S, scale: float = 1.0, l2norm: bool = False,
                threads: int = 0):
    """One token per sequence: q,k [N,H_qk,dk], v [N,H_v,dv], g,beta [N,H_v], S [N,H_v,dk,dv].

    A decode step is Eq. (1) applied once; it is the recurrence with every
    sequence of length 1.  Returns (out [N,H_v,dv], S_new).
    """
    N = q.shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    return recurrent(q, k, v, g, beta, S0=S, cu_seqlens=cu, scale=scale, l2norm=l2norm,
                     threads=threads)


def decode_multi(q, k, v, g, beta, S, n_commit=None, scale: float = 1.0, l2norm: bool = False,
                 threads: int = 0):
    """T consecutive tokens per sequence: q,k [N,T,H_qk,dk], v [N,T,H_v,dv], g,beta [N,T,H_v],
    S [N,H_v,dk,dv], n_commit [N] or None.

    Eq. (1) applied to each sequence's T tokens in order: the outputs are the
    recurrence's over all T tokens, and the returned state is the recurrence's state
    after the first n_commit[n] tokens (clamped to [0, T]; all T when None).  Returns
    (out [N,T,H_v,dv], S_new) as numpy.
    """
    N, T = q.shape[0], q.shape[1]
    flat = lambda x: _arr(x, np.float64).reshape((N * T,) + tuple(x.shape[2:]))
    cu = np.arange(0, N * T + 1, T, dtype=np.int64)
    out, S_all = recurrent(flat(q), flat(k), flat(v), flat(g), flat(beta), S0=S, cu_seqlens=cu,
                           scale=scale, l2norm=l2norm, threads=threads)
    out = out.reshape((N, T) + out.shape[1:])
    if n_commit is None:
        return out, S_all
    c = np.clip(np.asarray(n_commit.cpu() if hasattr(n_commit, "cpu") else n_commit).astype(np.int64), 0, T)
    # the first c[n] tokens of sequence n, packed
    idx = np.concatenate([n * T + np.arange(c[n]) for n in range(N)]).astype(np.int64)
    cu_c = np.concatenate([[0], np.cumsum(c)]).astype(np.int64)
    pick = lambda x: flat(x)[idx]
    _, S_c = recurrent(pick(q), pick(k), pick(v), pick(g), pick(beta), S0=S, cu_seqlens=cu_c,
                       scale=scale, l2norm=l2norm, threads=threads)
    return out, S_c


def gates_from_logits(a, b):
    """Gate prologue: from unconstrained logits, the decay gate's log g = -softplus(a)
    (so alpha = exp(g) lies in (0, 1)) and the write strength beta = sigmoid(b) (in
    (0, 1)) -- the ranges stated under Eq. (1) of "論文解説: Qwen3.8-Next の設計",
    section "GDNの中身".  fp64; returns numpy (g, beta)."""
    a = _arr(a, np.float64)
    b = _arr(b, np.float64)
    e = np.exp(-np.abs(b))                      # in (0, 1]: no overflow on either side
    return -np.logaddexp(0.0, a), np.where(b >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
