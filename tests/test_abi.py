"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/*.h declares, and rejects bad arguments before launching."""
from __future__ import annotations

import ctypes
import glob
import os
import re

import pytest

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import build as gdn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


@pytest.fixture(scope="module")
def L():
    gdn_build.build()          # nvcc cross-compiles without a GPU
    return gdn.lib()


def declared_functions():
    text = "".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_]+)\s*\(", text)))


def test_header_declares_the_abi():
    assert declared_functions() == sorted(gdn.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    # nothing else with the gdn_ prefix leaks out of the library
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", gdn._binding.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = sorted(set(re.findall(r"\b(gdn_[a-z_]+)$", out, flags=re.M)))
    assert exported == declared_functions()


def test_status_strings(L):
    for s in range(5):
        assert gdn.gdn_status_string(s).startswith("GDN_")
    assert "unknown" in gdn.gdn_status_string(99)


def test_workspace_size(L):
    assert gdn.gdn_prefill_workspace_size(8, 135000, 16, 128, 128) >= 256


# fake, 256-byte aligned device-looking addresses: never dereferenced because every
# call below fails validation on the host before any CUDA call
A = 0x7f0000000000
P = ctypes.c_void_p


def _prefill(L, **over):
    args = dict(q=A, k=A + 0x1000, v=A + 0x2000, g=A + 0x3000, beta=A + 0x4000, S0=None,
                out=A + 0x5000, S_final=None, cu=None, num_seqs=0, B=1, T=64, H_qk=2, H_v=4,
                dk=128, dv=128, dtype=1, scale=1.0, flags=0, ws=A + 0x6000, ws_bytes=256)
    args.update(over)
    a = args
    return L.gdn_prefill(P(a["q"]), P(a["k"]), P(a["v"]), P(a["g"]), P(a["beta"]), P(a["S0"]),
                         P(a["out"]), P(a["S_final"]), P(a["cu"]), a["num_seqs"], a["B"], a["T"],
                         a["H_qk"], a["H_v"], a["dk"], a["dv"], a["dtype"], a["scale"],
                         a["flags"], P(a["ws"]), a["ws_bytes"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(beta=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(out=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(H_v=3), gdn.GDN_ERR_INVALID_ARG),             # H_v % H_qk != 0
    (dict(H_qk=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dv=32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dtype=7), gdn.GDN_ERR_INVALID_ARG),
    (dict(flags=64), gdn.GDN_ERR_INVALID_ARG),
    (dict(v=A + 0x2008), gdn.GDN_ERR_INVALID_ARG),      # 8-byte aligned only
    (dict(g=A + 0x3002), gdn.GDN_ERR_INVALID_ARG),
    (dict(S0=A + 0x7004), gdn.GDN_ERR_INVALID_ARG),
    (dict(ws=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(ws_bytes=16), gdn.GDN_ERR_INVALID_ARG),
    (dict(cu=A + 0x8000, B=2, num_seqs=2), gdn.GDN_ERR_INVALID_ARG),   # varlen needs B == 1
    (dict(cu=A + 0x8000, num_seqs=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(T=-5), gdn.GDN_ERR_INVALID_ARG),
])
def test_prefill_rejects_on_host(L, over, expect):
    assert _prefill(L, **over) == expect


def _decode(L, **over):
    a = dict(q=A, k=A + 0x1000, v=A + 0x2000, g=A + 0x3000, beta=A + 0x4000, S=A + 0x5000,
             out=A + 0x6000, N=4, H_qk=2, H_v=4, dk=128, dv=128, dtype=1, scale=1.0, flags=0)
    a.update(over)
    return L.gdn_decode_step(P(a["q"]), P(a["k"]), P(a["v"]), P(a["g"]), P(a["beta"]), P(a["S"]),
                             P(a["out"]), a["N"], a["H_qk"], a["H_v"], a["dk"], a["dv"],
                             a["dtype"], a["scale"], a["flags"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(S=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(S=A + 0x5004), gdn.GDN_ERR_INVALID_ARG),
    (dict(k=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(H_v=6, H_qk=4), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=256), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dtype=3), gdn.GDN_ERR_INVALID_ARG),
])
def test_decode_rejects_on_host(L, over, expect):
    assert _decode(L, **over) == expect


def test_decode_with_no_sequences_is_a_no_op(L):
    assert _decode(L, N=0) == gdn.GDN_OK


def _decode_multi(L, **over):
    a = dict(q=A, k=A + 0x1000, v=A + 0x2000, g=A + 0x3000, beta=A + 0x4000, S=A + 0x5000,
             out=A + 0x6000, commit=None, N=4, T=4, H_qk=2, H_v=4, dk=128, dv=128, dtype=1,
             scale=1.0, flags=0)
    a.update(over)
    return L.gdn_decode_multi(P(a["q"]), P(a["k"]), P(a["v"]), P(a["g"]), P(a["beta"]),
                              P(a["S"]), P(a["out"]), P(a["commit"]), a["N"], a["T"], a["H_qk"],
                              a["H_v"], a["dk"], a["dv"], a["dtype"], a["scale"], a["flags"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(T=0), gdn.GDN_ERR_UNSUPPORTED),
    (dict(T=9), gdn.GDN_ERR_UNSUPPORTED),
    (dict(S=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(commit=A + 0x7002), gdn.GDN_ERR_INVALID_ARG),     # int32 array, 2-byte aligned
    (dict(v=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=-2), gdn.GDN_ERR_INVALID_ARG),
    (dict(H_v=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(dv=96), gdn.GDN_ERR_UNSUPPORTED),
])
def test_decode_multi_rejects_on_host(L, over, expect):
    assert _decode_multi(L, **over) == expect


def test_decode_multi_with_no_sequences_is_a_no_op(L):
    assert _decode_multi(L, N=0) == gdn.GDN_OK


def _backward(L, **over):
    a = dict(q=A, k=A + 0x1000, v=A + 0x2000, g=A + 0x3000, beta=A + 0x4000, S0=None,
             d_out=A + 0x5000, dSf=None, dq=A + 0x6000, dk=A + 0x7000, dv=A + 0x8000,
             dg=A + 0x9000, db=A + 0xa000, dS0=None, cu=None, num_seqs=0, B=1, T=64, H_qk=2,
             H_v=4, dk_dim=128, dv_dim=128, dtype=1, scale=1.0, flags=0, ws=A + 0xb000,
             ws_bytes=1 << 40)
    a.update(over)
    return L.gdn_backward(P(a["q"]), P(a["k"]), P(a["v"]), P(a["g"]), P(a["beta"]), P(a["S0"]),
                          P(a["d_out"]), P(a["dSf"]), P(a["dq"]), P(a["dk"]), P(a["dv"]),
                          P(a["dg"]), P(a["db"]), P(a["dS0"]), P(a["cu"]), a["num_seqs"], a["B"],
                          a["T"], a["H_qk"], a["H_v"], a["dk_dim"], a["dv_dim"], a["dtype"],
                          a["scale"], a["flags"], P(a["ws"]), a["ws_bytes"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(flags=gdn.GDN_FLAG_QK_L2NORM), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dq=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(db=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(d_out=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(ws_bytes=1024), gdn.GDN_ERR_INVALID_ARG),
    (dict(ws=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dv=A + 0x8004), gdn.GDN_ERR_INVALID_ARG),
    (dict(dS0=A + 0xc008), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk_dim=96), gdn.GDN_ERR_UNSUPPORTED),
])
def test_backward_rejects_on_host(L, over, expect):
    assert _backward(L, **over) == expect


def test_backward_workspace_size(L):
    # checkpoints every 64 tokens plus one recomputed chunk, per (sequence, head, 16 columns)
    n = gdn._binding.lib().gdn_backward_workspace_size(2, 8192, 16, 128, 128)
    assert n == 2 * 16 * 8 * (8192 // 64 + 1 + 65) * 128 * 16 * 4


def test_get_device_error_rejects_null(L):
    assert L.gdn_get_device_error(None, None) == gdn.GDN_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros(4, 2, 128)
    with pytest.raises(ValueError):
        gdn.gdn_decode_step(x, x, x, torch.zeros(4, 2), torch.zeros(4, 2),
                            torch.zeros(4, 2, 128, 128))


# ------------------------------------------------------------------ QSA indexer
def _qsa_compress(L, **over):
    a = dict(k=A, cu=A + 0x1000, cub=A + 0x2000, pos0=None, k_hat=A + 0x3000, N=2, nb=64,
             base=10000.0)
    a.update(over)
    return L.gdn_qsa_compress(P(a["k"]), P(a["cu"]), P(a["cub"]), P(a["pos0"]), P(a["k_hat"]),
                              a["N"], a["nb"], a["base"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(k=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(cub=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(k_hat=A + 0x3008), gdn.GDN_ERR_INVALID_ARG),      # bf16 rows need 16-byte alignment
    (dict(pos0=A + 0x4002), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=0), gdn.GDN_ERR_INVALID_ARG),                   # blocks but no sequence
    (dict(nb=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(nb=1 << 31), gdn.GDN_ERR_INVALID_ARG),
    (dict(base=0.0), gdn.GDN_ERR_INVALID_ARG),
    (dict(base=float("inf")), gdn.GDN_ERR_INVALID_ARG),
])
def test_qsa_compress_rejects_on_host(L, over, expect):
    assert _qsa_compress(L, **over) == expect


def test_qsa_compress_without_blocks_is_a_no_op(L):
    assert _qsa_compress(L, nb=0, k=None, k_hat=None) == gdn.GDN_OK


def _qsa_index(L, **over):
    a = dict(q=A, qpos=A + 0x1000, k_hat=A + 0x2000, cub=A + 0x3000, N=2, nb=64, budget=512,
             base=10000.0, bi=A + 0x4000, bs=None, ti=None, ws=A + 0x5000, ws_bytes=1 << 40)
    a.update(over)
    return L.gdn_qsa_index_decode(P(a["q"]), P(a["qpos"]), P(a["k_hat"]), P(a["cub"]), a["N"],
                                  a["nb"], a["budget"], a["base"], P(a["bi"]), P(a["bs"]),
                                  P(a["ti"]), P(a["ws"]), a["ws_bytes"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(qpos=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(bi=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(ws=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(k_hat=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(q=A + 8), gdn.GDN_ERR_INVALID_ARG),
    (dict(ti=A + 0x6002), gdn.GDN_ERR_INVALID_ARG),
    (dict(budget=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(budget=4097), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=4097), gdn.GDN_ERR_UNSUPPORTED),
    (dict(ws_bytes=1024), gdn.GDN_ERR_INVALID_ARG),
    (dict(base=-1.0), gdn.GDN_ERR_INVALID_ARG),
])
def test_qsa_index_rejects_on_host(L, over, expect):
    assert _qsa_index(L, **over) == expect


def test_qsa_index_with_no_sequences_is_a_no_op(L):
    assert _qsa_index(L, N=0, q=None, qpos=None, bi=None, ws=None) == gdn.GDN_OK


def test_qsa_workspace_size(L):
    # per sequence: 4096-bin histogram, two counters, threshold and rank, the finished-item
    # counter (padded to 16 bytes), 4096 kept and 8192 candidate (key, block) pairs; then
    # one fp32 score per cached block (256-byte rounded)
    rec = 4096 * 4 + 4 * 4 + 4 * 4 + 4096 * 8 + 8192 * 8
    assert L.gdn_qsa_index_workspace_size(3, 1000) == 3 * rec + 4096
    assert L.gdn_qsa_index_workspace_size(-1, 10) == 0


def test_qsa_constants_match_the_header():
    text = open(os.path.join(ROOT, "include", "qsa.h")).read()
    vals = dict(re.findall(r"#define (GDN_QSA_[A-Z_]+) (\d+)", text))
    b = gdn._binding
    assert int(vals["GDN_QSA_R"]) == b.GDN_QSA_R == 4
    assert int(vals["GDN_QSA_DIM"]) == b.GDN_QSA_DIM == 128
    assert int(vals["GDN_QSA_ROPE_DIMS"]) == b.GDN_QSA_ROPE_DIMS == 64
    assert int(vals["GDN_QSA_HEADS"]) == b.GDN_QSA_HEADS == 4
    assert int(vals["GDN_QSA_MAX_BUDGET"]) == b.GDN_QSA_MAX_BUDGET
    assert int(vals["GDN_QSA_MAX_SEQS"]) == b.GDN_QSA_MAX_SEQS
    assert int(vals["GDN_QSA_MAX_QUERIES"]) == b.GDN_QSA_MAX_QUERIES == 4


def _qsa_multi(L, **over):
    a = dict(q=A, qpos=A + 0x1000, k_hat=A + 0x2000, cub=A + 0x3000, N=2, nb=64, T=4,
             budget=512, base=10000.0, bi=A + 0x4000, bs=None, ti=None, ws=A + 0x5000,
             ws_bytes=1 << 40)
    a.update(over)
    return L.gdn_qsa_index_multi(P(a["q"]), P(a["qpos"]), P(a["k_hat"]), P(a["cub"]), a["N"],
                                 a["nb"], a["T"], a["budget"], a["base"], P(a["bi"]), P(a["bs"]),
                                 P(a["ti"]), P(a["ws"]), a["ws_bytes"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(T=0), gdn.GDN_ERR_UNSUPPORTED),
    (dict(T=5), gdn.GDN_ERR_UNSUPPORTED),
    (dict(N=1025), gdn.GDN_ERR_UNSUPPORTED),                 # 1025 x 4 query units > 4096
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(budget=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(ws_bytes=4096), gdn.GDN_ERR_INVALID_ARG),
    (dict(bs=A + 0x6002), gdn.GDN_ERR_INVALID_ARG),
])
def test_qsa_multi_rejects_on_host(L, over, expect):
    assert _qsa_multi(L, **over) == expect


def test_qsa_multi_with_no_sequences_is_a_no_op(L):
    assert _qsa_multi(L, N=0, q=None, qpos=None, bi=None, ws=None) == gdn.GDN_OK


def test_qsa_multi_workspace_size(L):
    rec = 4096 * 4 + 4 * 4 + 4 * 4 + 4096 * 8 + 8192 * 8
    # one record per (sequence, query), one fp32 score per (cached block, query)
    assert L.gdn_qsa_index_multi_workspace_size(3, 1000, 4) == 12 * rec + 16128
    assert L.gdn_qsa_index_multi_workspace_size(3, 1000, 1) == L.gdn_qsa_index_workspace_size(3, 1000)
    assert L.gdn_qsa_index_multi_workspace_size(3, 1000, 5) == 0


def test_qsa_binding_checks_types_and_shapes(L):
    """Wrong dtypes or shapes raise in the binding before anything reaches the library
    (these run on CPU tensors: the checks come before the device-pointer checks)."""
    import torch
    N = 2
    q = torch.zeros(N, 4, 128, dtype=torch.bfloat16)
    pos = torch.zeros(N, dtype=torch.int32)
    kh = torch.zeros(10, 128, dtype=torch.bfloat16)
    cub = torch.zeros(N + 1, dtype=torch.int32)
    with pytest.raises(TypeError, match="k_hat"):
        gdn.gdn_qsa_index_decode(q, pos, kh.float(), cub)
    with pytest.raises(TypeError, match="q_pos"):
        gdn.gdn_qsa_index_decode(q, pos.long(), kh, cub)
    with pytest.raises(ValueError, match="q must have shape"):
        gdn.gdn_qsa_index_decode(q[:, :3], pos, kh, cub)
    with pytest.raises(ValueError, match="cu_blocks"):
        gdn.gdn_qsa_index_decode(q, pos, kh, cub[:2])
    with pytest.raises(ValueError, match="q must have shape"):
        gdn.gdn_qsa_index_multi(q, pos, kh, cub)                  # needs [N, T, 4, 128]
    with pytest.raises(TypeError, match="k must be"):
        gdn.gdn_qsa_compress(torch.zeros(40, 128), cub, cub, k_hat=kh)
    with pytest.raises(ValueError, match="pos0"):
        gdn.gdn_qsa_compress(torch.zeros(40, 128, dtype=torch.bfloat16), cub, cub, k_hat=kh,
                             pos0=torch.zeros(5, dtype=torch.int32))
    # well-formed CPU tensors get as far as the device check
    with pytest.raises(ValueError, match="CUDA tensor"):
        gdn.gdn_qsa_index_decode(q, pos, kh, cub)


def test_gdn_bindings_check_dtypes(L):
    """A tensor whose dtype differs from q's (or a non-float32 gate or state) raises in the
    binding instead of being read as the wrong type (CPU tensors: the checks come first)."""
    import torch
    bf, f32 = torch.bfloat16, torch.float32
    q = torch.zeros(4, 2, 128, dtype=bf)
    v = torch.zeros(4, 2, 128, dtype=bf)
    g = torch.zeros(4, 2)
    S = torch.zeros(4, 2, 128, 128)
    with pytest.raises(TypeError, match="k must have"):
        gdn.gdn_decode_step(q, q.float(), v, g, g, S)
    with pytest.raises(TypeError, match="g must be float32"):
        gdn.gdn_decode_step(q, q, v, g.to(bf), g, S)
    with pytest.raises(TypeError, match="S_inout must be float32"):
        gdn.gdn_decode_step(q, q, v, g, g, S.to(bf))
    with pytest.raises(TypeError, match="v must have"):
        gdn.gdn_prefill(q, q, v.float(), g, g)
    with pytest.raises(TypeError, match="d_out must have"):
        gdn.gdn_backward(q, q, v, g, g, v.float())
    with pytest.raises(TypeError, match="S_inout must be float32"):
        gdn.gdn_decode_multi(q[:, None], q[:, None], v[:, None], g[:, None], g[:, None], S.double())
    with pytest.raises(ValueError, match="CUDA tensor"):      # consistent dtypes pass on
        gdn.gdn_decode_step(q, q, v, g, g, S)
