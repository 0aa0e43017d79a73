"""ctypes binding of libgdn (include/gdn.h, include/qsa.h): argument marshalling only.

Every step of the gated delta rule runs in libgdn's CUDA kernels; this module
passes torch device pointers, sizes and the current CUDA stream through the C ABI
and turns status codes into exceptions.  There is no fallback: if libgdn.so is
missing, or a tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT = range(5)
GDN_F32, GDN_BF16 = 0, 1
GDN_FLAG_QK_L2NORM = 1
GDN_FLAG_FORCE_CUDA_CORE = 2
GDN_FLAG_GATE_LOGITS = 4

# QSA indexer constants (include/qsa.h)
GDN_QSA_R, GDN_QSA_DIM, GDN_QSA_ROPE_DIMS, GDN_QSA_HEADS = 4, 128, 64, 4
GDN_QSA_MAX_BUDGET, GDN_QSA_MAX_SEQS, GDN_QSA_MAX_QUERIES = 4096, 4096, 4

# every symbol include/gdn.h and include/qsa.h declare
EXPORTED = ("gdn_prefill_workspace_size", "gdn_prefill", "gdn_decode_step",
            "gdn_get_device_error", "gdn_status_string", "gdn_prefill_static_scratch",
            "gdn_decode_multi", "gdn_backward", "gdn_backward_workspace_size",
            "gdn_qsa_compress", "gdn_qsa_index_workspace_size", "gdn_qsa_index_decode",
            "gdn_qsa_index_multi_workspace_size", "gdn_qsa_index_multi",
            "gdn_set_wait_budget", "gdn_set_prefill_segment_tokens", "gdn_prefill_schedule")

_lib = None


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {gdn_status_string(status)}")


def lib():
    """The loaded libgdn handle (raises if the library has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgdn.so not found at {LIB_PATH}; build it with "
                               "`python -m linear_attention_token_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, U32, F, SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                   ctypes.c_uint32, ctypes.c_float, ctypes.c_size_t)
        L.gdn_prefill_workspace_size.argtypes = [I32, I64, I32, I32, I32]
        L.gdn_prefill_workspace_size.restype = SZ
        L.gdn_prefill.argtypes = [P, P, P, P, P, P, P, P, P, I32, I32, I64, I32, I32, I32, I32,
                                  ctypes.c_int, F, U32, P, SZ, P]
        L.gdn_prefill.restype = ctypes.c_int
        L.gdn_prefill_static_scratch.argtypes = [P, P, P, P, P, P, P, P, P, I32, I32, I64, I32,
                                                 I32, I32, I32, ctypes.c_int, F, U32, P]
        L.gdn_prefill_static_scratch.restype = ctypes.c_int
        L.gdn_decode_step.argtypes = [P, P, P, P, P, P, P, I32, I32, I32, I32, I32, ctypes.c_int,
                                      F, U32, P]
        L.gdn_decode_step.restype = ctypes.c_int
        L.gdn_decode_multi.argtypes = [P, P, P, P, P, P, P, P, I32, I32, I32, I32, I32, I32,
                                       ctypes.c_int, F, U32, P]
        L.gdn_decode_multi.restype = ctypes.c_int
        L.gdn_backward_workspace_size.argtypes = [I32, I64, I32, I32, I32]
        L.gdn_backward_workspace_size.restype = SZ
        L.gdn_backward.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, I32, I32, I64, I32,
                                   I32, I32, I32, ctypes.c_int, F, U32, P, SZ, P]
        L.gdn_backward.restype = ctypes.c_int
        L.gdn_qsa_compress.argtypes = [P, P, P, P, P, I32, I64, F, P]
        L.gdn_qsa_compress.restype = ctypes.c_int
        L.gdn_qsa_index_workspace_size.argtypes = [I32, I64]
        L.gdn_qsa_index_workspace_size.restype = SZ
        L.gdn_qsa_index_decode.argtypes = [P, P, P, P, I32, I64, I32, F, P, P, P, P, SZ, P]
        L.gdn_qsa_index_decode.restype = ctypes.c_int
        L.gdn_qsa_index_multi_workspace_size.argtypes = [I32, I64, I32]
        L.gdn_qsa_index_multi_workspace_size.restype = SZ
        L.gdn_qsa_index_multi.argtypes = [P, P, P, P, I32, I64, I32, I32, F, P, P, P, P, SZ, P]
        L.gdn_qsa_index_multi.restype = ctypes.c_int
        L.gdn_prefill_schedule.argtypes = [I32, I64, I32, I32, I32, ctypes.c_int, I32, SZ, U32,
                                           P, P, P]
        L.gdn_prefill_schedule.restype = ctypes.c_int
        L.gdn_set_wait_budget.argtypes = [U32]
        L.gdn_set_wait_budget.restype = U32
        L.gdn_set_prefill_segment_tokens.argtypes = [I32]
        L.gdn_set_prefill_segment_tokens.restype = ctypes.c_int
        L.gdn_get_device_error.argtypes = [P, P]
        L.gdn_get_device_error.restype = ctypes.c_int
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def gdn_status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != GDN_OK:
        raise GdnError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; libgdn takes float32 or bfloat16")


def _check_dtypes(q, same=(), f32=()):
    """Every (name, tensor) in `same` must have q's dtype and every one in `f32` must be
    float32 (None entries are skipped): a mismatch would otherwise be read as q's type."""
    _dtype_code(q)
    for name, t in same:
        if t is not None and t.dtype != q.dtype:
            raise TypeError(f"{name} must have q's dtype {q.dtype}, got {t.dtype}")
    for name, t in f32:
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32, got {t.dtype}")


def _dev(t: Optional[torch.Tensor], name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libgdn has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def gdn_set_wait_budget(polls: int) -> int:
    """Set the poll limit of every device-side wait of the tensor-core prefill (process-wide);
    returns the previous limit.  0 makes every wait give up at once."""
    return int(lib().gdn_set_wait_budget(int(polls)))


def gdn_set_prefill_segment_tokens(tokens: int) -> None:
    """Prefill schedule override: 0 automatic, -1 one unit per sequence, or a segment
    length in tokens (a multiple of 64)."""
    _check(lib().gdn_set_prefill_segment_tokens(int(tokens)), "gdn_set_prefill_segment_tokens")


PREFILL_KERNELS = {0: "none", 1: "cuda_core", 2: "chain", 3: "cluster"}


def gdn_prefill_schedule(num_seqs: int, T_total: int, H_v: int, dk: int, dv: int,
                         dtype=torch.bfloat16, varlen: bool = False, workspace_bytes=None,
                         flags: int = 0) -> dict:
    """The schedule gdn_prefill would use: {"kernel", "segment_tokens", "launches"}."""
    if workspace_bytes is None:
        workspace_bytes = gdn_prefill_workspace_size(num_seqs, T_total, H_v, dk, dv)
    kern, seg, n = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    _check(lib().gdn_prefill_schedule(num_seqs, T_total, H_v, dk, dv, code, int(varlen),
                                      int(workspace_bytes), int(flags), ctypes.byref(kern),
                                      ctypes.byref(seg), ctypes.byref(n)), "gdn_prefill_schedule")
    return {"kernel": PREFILL_KERNELS[kern.value], "segment_tokens": seg.value, "launches": n.value}


def gdn_prefill_workspace_size(num_seqs: int, T_total: int, H_v: int, dk: int, dv: int) -> int:
    return int(lib().gdn_prefill_workspace_size(num_seqs, T_total, H_v, dk, dv))


def prefill_workspace(num_seqs: int, T_total: int, H_v: int, dk: int, dv: int,
                      device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size gdn_prefill needs (torch allocates it)."""
    n = gdn_prefill_workspace_size(num_seqs, T_total, H_v, dk, dv)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _prefill_shapes(q, k, v, g, beta, S0, cu_seqlens, out, S_final):
    """Sizes (B, T, N, H_qk, H_v, dk, dv) of a prefill call, after checking every operand
    against them: the library reads and writes exactly these extents, so a wrong shape, an
    int64 offset table or a tensor on another device would otherwise be an out-of-bounds
    device access instead of a Python error."""
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
            raise ValueError("cu_seqlens must be 1-D with num_seqs + 1 entries")
        if q.dim() != 3:
            raise ValueError("varlen q must be [T_total, H_qk, dk]")
        T_total, H_qk, dk = q.shape
        B, T, N = 1, T_total, cu_seqlens.numel() - 1
    else:
        if q.dim() == 4:
            B, T, H_qk, dk = q.shape
        elif q.dim() == 3:
            B, (T, H_qk, dk) = 1, q.shape
        else:
            raise ValueError("q must be [B, T, H_qk, dk] or [T, H_qk, dk]")
        N = B
    lead = tuple(q.shape[:-2])
    if v.dim() != q.dim() or tuple(v.shape[:-2]) != lead:
        raise ValueError(f"v {tuple(v.shape)} does not match q {tuple(q.shape)}")
    H_v, dv = v.shape[-2:]
    want = {"k": tuple(q.shape), "g": lead + (H_v,), "beta": lead + (H_v,),
            "out": tuple(v.shape), "S0": (N, H_v, dk, dv), "S_final": (N, H_v, dk, dv)}
    for name, t in (("k", k), ("g", g), ("beta", beta), ("out", out), ("S0", S0),
                    ("S_final", S_final)):
        if t is not None and tuple(t.shape) != want[name]:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want[name]}")
    for name, t in (("k", k), ("v", v), ("g", g), ("beta", beta), ("out", out), ("S0", S0),
                    ("S_final", S_final), ("cu_seqlens", cu_seqlens)):
        if t is not None and t.device != q.device:
            raise ValueError(f"{name} is on {t.device}, q on {q.device}")
    return B, T, N, H_qk, H_v, dk, dv


def gdn_prefill(q, k, v, g, beta, S0=None, cu_seqlens=None, *, out=None, S_final=None,
                scale: float = 1.0, flags: int = 0, workspace=None, want_state: bool = True,
                stream=None):
    """Chunked prefill.  q,k [..., T, H_qk, dk]; v [..., T, H_v, dv]; g,beta [..., T, H_v].

    Dense batch: q is [B, T, H_qk, dk] (or [T, H_qk, dk] for B = 1) and cu_seqlens is None.
    Varlen: q is [T_total, H_qk, dk] and cu_seqlens an int32 CUDA tensor [num_seqs + 1].
    Returns (out, S_final); S_final is None when want_state is False and none was given.
    """
    _check_dtypes(q, (("k", k), ("v", v), ("out", out)),
                  (("g", g), ("beta", beta), ("S0", S0), ("S_final", S_final)))
    B, T, N, H_qk, H_v, dk, dv = _prefill_shapes(q, k, v, g, beta, S0, cu_seqlens, out, S_final)
    T_total = B * T
    if out is None:
        out = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    if S_final is None and want_state:
        S_final = torch.empty(N, H_v, dk, dv, dtype=torch.float32, device=v.device)
    if workspace is None:
        workspace = prefill_workspace(N, T_total, H_v, dk, dv, v.device)
    st = lib().gdn_prefill(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
        _dev(S0, "S0"), _dev(out, "out"), _dev(S_final, "S_final"),
        _dev(cu_seqlens, "cu_seqlens"), N if cu_seqlens is not None else 0, B, T, H_qk, H_v,
        dk, dv, _dtype_code(q), float(scale), int(flags), _dev(workspace, "workspace"),
        workspace.numel(), _stream(stream))
    _check(st, "gdn_prefill")
    return out, S_final


def gdn_prefill_static_scratch(q, k, v, g, beta, S0=None, cu_seqlens=None, *, out, S_final,
                               scale: float = 1.0, flags: int = 0, stream=None):
    """gdn_prefill through the entry point that takes no workspace and allocates nothing.

    For callers that cannot allocate device memory: the library supplies its own
    static scratch.  ``out`` and ``S_final`` must be given (this call allocates nothing);
    S_final may be None to skip the final state.  Shapes as for gdn_prefill.
    """
    _check_dtypes(q, (("k", k), ("v", v), ("out", out)),
                  (("g", g), ("beta", beta), ("S0", S0), ("S_final", S_final)))
    if out is None:
        raise ValueError("out must be given: this entry point allocates nothing")
    B, T, N, H_qk, H_v, dk, dv = _prefill_shapes(q, k, v, g, beta, S0, cu_seqlens, out, S_final)
    st = lib().gdn_prefill_static_scratch(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
        _dev(S0, "S0"), _dev(out, "out"), _dev(S_final, "S_final"),
        _dev(cu_seqlens, "cu_seqlens"), N if cu_seqlens is not None else 0, B, T, H_qk, H_v,
        dk, dv, _dtype_code(q), float(scale), int(flags), _stream(stream))
    _check(st, "gdn_prefill_static_scratch")
    return out, S_final


def gdn_decode_step(q, k, v, g, beta, S_inout, *, out=None, scale: float = 1.0, flags: int = 0,
                    stream=None):
    """One decode step in place on S_inout [N, H_v, dk, dv]; q,k [N, H_qk, dk]; v [N, H_v, dv]."""
    _check_dtypes(q, (("k", k), ("v", v), ("out", out)),
                  (("g", g), ("beta", beta), ("S_inout", S_inout)))
    N, H_qk, dk = q.shape
    H_v, dv = v.shape[-2:]
    if out is None:
        out = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    st = lib().gdn_decode_step(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
        _dev(S_inout, "S_inout"), _dev(out, "out"), N, H_qk, H_v, dk, dv, _dtype_code(q),
        float(scale), int(flags), _stream(stream))
    _check(st, "gdn_decode_step")
    return out


def gdn_decode_multi(q, k, v, g, beta, S_inout, *, n_commit=None, out=None, scale: float = 1.0,
                     flags: int = 0, stream=None):
    """T consecutive tokens per (sequence, head) in one call: q,k [N, T, H_qk, dk];
    v [N, T, H_v, dv]; g, beta [N, T, H_v].  S_inout [N, H_v, dk, dv] becomes the state
    after n_commit[n] tokens (int32 [N] on the device; None = all T).  Returns out."""
    _check_dtypes(q, (("k", k), ("v", v), ("out", out)),
                  (("g", g), ("beta", beta), ("S_inout", S_inout)))
    N, T, H_qk, dk = q.shape
    H_v, dv = v.shape[-2:]
    if out is None:
        out = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    if n_commit is not None and n_commit.dtype != torch.int32:
        raise ValueError("n_commit must be int32")
    st = lib().gdn_decode_multi(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
        _dev(S_inout, "S_inout"), _dev(out, "out"), _dev(n_commit, "n_commit"), N, T, H_qk, H_v,
        dk, dv, _dtype_code(q), float(scale), int(flags), _stream(stream))
    _check(st, "gdn_decode_multi")
    return out


def gdn_backward(q, k, v, g, beta, d_out, S0=None, dS_final=None, cu_seqlens=None, *,
                 scale: float = 1.0, flags: int = 0, want_dS0: bool = True, workspace=None,
                 stream=None):
    """Gradients of a loss with respect to q, k, v, g, beta (and S0), given d_out (like out)
    and dS_final (fp32 [N, H_v, dk, dv] or None).  Shapes and varlen form as gdn_prefill.

    Returns a dict of fp32 tensors dq, dk (like q), dv (like v), dg, dbeta (like g) and
    dS0 ([N, H_v, dk, dv], None when want_dS0 is False).
    """
    _check_dtypes(q, (("k", k), ("v", v), ("d_out", d_out)),
                  (("g", g), ("beta", beta), ("S0", S0), ("dS_final", dS_final)))
    if cu_seqlens is not None:
        T_total, H_qk, dk = q.shape[-3:]
        B, T, N = 1, T_total, cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
    else:
        if q.dim() == 4:
            B, T, H_qk, dk = q.shape
        else:
            B, (T, H_qk, dk) = 1, q.shape
        T_total, N = B * T, B
    H_v, dv = v.shape[-2:]
    f32 = dict(dtype=torch.float32, device=v.device)
    grads = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32),
             "dv": torch.empty(v.shape, **f32), "dg": torch.empty(g.shape, **f32),
             "dbeta": torch.empty(beta.shape, **f32),
             "dS0": torch.empty(N, H_v, dk, dv, **f32) if want_dS0 else None}
    if workspace is None:
        n = int(lib().gdn_backward_workspace_size(N, T_total, H_v, dk, dv))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=v.device)
    st = lib().gdn_backward(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(g, "g"), _dev(beta, "beta"),
        _dev(S0, "S0"), _dev(d_out, "d_out"), _dev(dS_final, "dS_final"),
        _dev(grads["dq"], "dq"), _dev(grads["dk"], "dk"), _dev(grads["dv"], "dv"),
        _dev(grads["dg"], "dg"), _dev(grads["dbeta"], "dbeta"), _dev(grads["dS0"], "dS0"),
        _dev(cu_seqlens, "cu_seqlens"), N if cu_seqlens is not None else 0, B, T, H_qk, H_v,
        dk, dv, _dtype_code(q), float(scale), int(flags), _dev(workspace, "workspace"),
        workspace.numel(), _stream(stream))
    _check(st, "gdn_backward")
    return grads


def gdn_get_device_error(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream; return (and clear) the device error status in the workspace."""
    return int(lib().gdn_get_device_error(_dev(workspace, "workspace"), _stream(stream)))


# ------------------------------------------------------------------ QSA indexer
def _need(t, name, dtype, shape):
    """Raise before anything reaches the library if a QSA argument has the wrong type or
    shape (None in `shape` matches any size)."""
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != len(shape) or any(s is not None and s != d for s, d in zip(shape, t.shape)):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def gdn_qsa_compress(k, cu_seqlens, cu_blocks, *, k_hat, pos0=None, rope_base: float = 10000.0,
                     stream=None):
    """Block cache from indexer keys: k [T_total, 128] bf16 -> k_hat [total_blocks, 128] bf16
    (written in place and returned); cu_seqlens, cu_blocks int32 [N + 1], pos0 int32 [N]."""
    N = cu_seqlens.numel() - 1
    _need(k, "k", torch.bfloat16, (None, GDN_QSA_DIM))
    _need(k_hat, "k_hat", torch.bfloat16, (None, GDN_QSA_DIM))
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,))
    _need(cu_blocks, "cu_blocks", torch.int32, (N + 1,))
    if pos0 is not None:
        _need(pos0, "pos0", torch.int32, (N,))
    st = lib().gdn_qsa_compress(
        _dev(k, "k"), _dev(cu_seqlens, "cu_seqlens"), _dev(cu_blocks, "cu_blocks"),
        _dev(pos0, "pos0"), _dev(k_hat, "k_hat"), N, k_hat.shape[0], float(rope_base),
        _stream(stream))
    _check(st, "gdn_qsa_compress")
    return k_hat


def gdn_qsa_index_workspace_size(num_seqs: int, total_blocks: int) -> int:
    return int(lib().gdn_qsa_index_workspace_size(num_seqs, total_blocks))


def qsa_index_workspace(num_seqs: int, total_blocks: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size gdn_qsa_index_decode needs."""
    n = gdn_qsa_index_workspace_size(num_seqs, total_blocks)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def gdn_qsa_index_decode(q, q_pos, k_hat, cu_blocks, budget_blocks: int = 512, *,
                         rope_base: float = 10000.0, workspace=None, block_idx=None,
                         block_score=None, token_idx=None, want_scores: bool = True,
                         want_tokens: bool = True, stream=None):
    """Indexer for one new token per sequence: q [N, 4, 128] bf16, q_pos int32 [N],
    k_hat [total_blocks, 128] bf16, cu_blocks int32 [N + 1].  Returns (block_idx [N, budget],
    block_score [N, budget] or None, token_idx [N, 4 budget] or None)."""
    N = q.shape[0]
    _need(q, "q", torch.bfloat16, (N, GDN_QSA_HEADS, GDN_QSA_DIM))
    _need(q_pos, "q_pos", torch.int32, (N,))
    _need(k_hat, "k_hat", torch.bfloat16, (None, GDN_QSA_DIM))
    _need(cu_blocks, "cu_blocks", torch.int32, (N + 1,))
    dev = q.device
    if workspace is None:
        workspace = qsa_index_workspace(N, k_hat.shape[0], dev)
    if block_idx is None:
        block_idx = torch.empty(N, budget_blocks, dtype=torch.int32, device=dev)
    if block_score is None and want_scores:
        block_score = torch.empty(N, budget_blocks, dtype=torch.float32, device=dev)
    if token_idx is None and want_tokens:
        token_idx = torch.empty(N, GDN_QSA_R * budget_blocks, dtype=torch.int32, device=dev)
    st = lib().gdn_qsa_index_decode(
        _dev(q, "q"), _dev(q_pos, "q_pos"), _dev(k_hat, "k_hat"), _dev(cu_blocks, "cu_blocks"),
        N, k_hat.shape[0], int(budget_blocks), float(rope_base), _dev(block_idx, "block_idx"),
        _dev(block_score, "block_score"), _dev(token_idx, "token_idx"),
        _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "gdn_qsa_index_decode")
    return block_idx, block_score, token_idx


def gdn_qsa_index_multi_workspace_size(num_seqs: int, total_blocks: int, n_queries: int) -> int:
    return int(lib().gdn_qsa_index_multi_workspace_size(num_seqs, total_blocks, n_queries))


def qsa_index_multi_workspace(num_seqs: int, total_blocks: int, n_queries: int,
                              device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size gdn_qsa_index_multi needs."""
    n = gdn_qsa_index_multi_workspace_size(num_seqs, total_blocks, n_queries)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def gdn_qsa_index_multi(q, q_pos, k_hat, cu_blocks, budget_blocks: int = 512, *,
                        rope_base: float = 10000.0, workspace=None, block_idx=None,
                        block_score=None, token_idx=None, want_scores: bool = True,
                        want_tokens: bool = True, stream=None):
    """Indexer for T consecutive tokens per sequence: q [N, T, 4, 128] bf16 (query j of
    sequence n at position q_pos[n] + j), q_pos int32 [N], k_hat [total_blocks, 128] bf16,
    cu_blocks int32 [N + 1].  Returns (block_idx [N, T, budget], block_score or None,
    token_idx [N, T, 4 budget] or None)."""
    N, T = q.shape[0], q.shape[1]
    _need(q, "q", torch.bfloat16, (N, T, GDN_QSA_HEADS, GDN_QSA_DIM))
    _need(q_pos, "q_pos", torch.int32, (N,))
    _need(k_hat, "k_hat", torch.bfloat16, (None, GDN_QSA_DIM))
    _need(cu_blocks, "cu_blocks", torch.int32, (N + 1,))
    dev = q.device
    if workspace is None:
        workspace = qsa_index_multi_workspace(N, k_hat.shape[0], T, dev)
    if block_idx is None:
        block_idx = torch.empty(N, T, budget_blocks, dtype=torch.int32, device=dev)
    if block_score is None and want_scores:
        block_score = torch.empty(N, T, budget_blocks, dtype=torch.float32, device=dev)
    if token_idx is None and want_tokens:
        token_idx = torch.empty(N, T, GDN_QSA_R * budget_blocks, dtype=torch.int32, device=dev)
    st = lib().gdn_qsa_index_multi(
        _dev(q, "q"), _dev(q_pos, "q_pos"), _dev(k_hat, "k_hat"), _dev(cu_blocks, "cu_blocks"),
        N, k_hat.shape[0], T, int(budget_blocks), float(rope_base), _dev(block_idx, "block_idx"),
        _dev(block_score, "block_score"), _dev(token_idx, "token_idx"),
        _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "gdn_qsa_index_multi")
    return block_idx, block_score, token_idx
