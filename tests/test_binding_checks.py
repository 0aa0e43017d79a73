"""The Python binding refuses prefill operands whose shapes, offset type or device do not
match: the library reads and writes the extents the sizes imply, so each of these would
otherwise be an out-of-bounds device access.  Runs on CPU: every check fires before a
pointer is taken."""
from __future__ import annotations

import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs


def _varlen(lens=(5, 3)):
    x = inputs.draw(sum(lens), 2, 4, 64, 64, torch.bfloat16, 3, "cpu")
    x["cu"] = inputs.cu_seqlens_of(list(lens))
    x["out"] = torch.empty_like(x["v"])
    x["S"] = torch.empty(len(lens), 4, 64, 64)
    return x


def _call(fn, x, **over):
    a = dict(q=x["q"], k=x["k"], v=x["v"], g=x["g"], beta=x["beta"], S0=None,
             cu_seqlens=x["cu"], out=x["out"], S_final=x["S"])
    a.update(over)
    return fn(a.pop("q"), a.pop("k"), a.pop("v"), a.pop("g"), a.pop("beta"), a.pop("S0"),
              a.pop("cu_seqlens"), **a)


FNS = [gdn.gdn_prefill, gdn.gdn_prefill_static_scratch]


@pytest.mark.parametrize("fn", FNS)
def test_int64_offsets_refused(fn):
    x = _varlen()
    with pytest.raises(TypeError, match="int32"):
        _call(fn, x, cu_seqlens=x["cu"].long())


@pytest.mark.parametrize("fn", FNS)
@pytest.mark.parametrize("name,shape", [("out", (7, 4, 64)), ("S_final", (2, 4, 64, 32)),
                                        ("S_final", (3, 4, 64, 64)), ("S0", (1, 4, 64, 64)),
                                        ("k", (8, 2, 32)), ("g", (8, 2)), ("beta", (7, 4))])
def test_wrong_shape_refused(fn, name, shape):
    x = _varlen()
    dt = torch.float32 if name in ("S_final", "S0", "g", "beta") else torch.bfloat16
    with pytest.raises(ValueError, match=name):
        _call(fn, x, **{name: torch.empty(shape, dtype=dt)})


@pytest.mark.parametrize("fn", FNS)
def test_dense_out_shape_refused(fn):
    x = inputs.draw(16, 2, 2, 64, 64, torch.bfloat16, 4, "cpu")
    x = {k: t.view(2, 8, *t.shape[1:]) for k, t in x.items()}
    with pytest.raises(ValueError, match="out"):
        fn(x["q"], x["k"], x["v"], x["g"], x["beta"], None, None,
           out=torch.empty(16, 2, 64, dtype=torch.bfloat16), S_final=torch.empty(2, 2, 64, 64))


def test_static_scratch_needs_out():
    x = _varlen()
    with pytest.raises(ValueError, match="allocates nothing"):
        _call(gdn.gdn_prefill_static_scratch, x, out=None)


@pytest.mark.parametrize("fn", FNS)
def test_other_device_refused(fn):
    x = _varlen()
    meta = torch.empty(x["S"].shape, device="meta")
    with pytest.raises(ValueError, match="S_final is on meta"):
        _call(fn, x, S_final=meta)
