"""Failure handling without a GPU fault: the tensor-core prefill's bounded waits are
made to give up at once (GDN_TEST_WAIT_BUDGET=0, a test hook read per call), the
kernel records GDN_ERR_TIMEOUT in the workspace, lets its own copies land, frees its
TMEM and exits; the context stays usable and the next call is correct."""
from __future__ import annotations

import os

import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs
from parity import TOL, err, oracle_prefill

pytestmark = pytest.mark.gpu


def _case():
    lens = [100, 37]
    x = inputs.draw(sum(lens), 2, 2, 128, 128, torch.bfloat16, 99, "cuda")
    x["S0"] = None
    x["cu_seqlens"] = inputs.cu_seqlens_of(lens).cuda()
    return x


def test_timeout_is_reported_and_recoverable():
    x = _case()
    ws = gdn.prefill_workspace(2, 137, 2, 128, 128)
    os.environ["GDN_TEST_WAIT_BUDGET"] = "0"
    try:
        gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"],
                        workspace=ws)
        status = gdn.gdn_get_device_error(ws)
    finally:
        del os.environ["GDN_TEST_WAIT_BUDGET"]
    assert status == gdn.GDN_ERR_TIMEOUT
    assert gdn.gdn_get_device_error(ws) == gdn.GDN_OK          # read clears it
    o, S = gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"],
                           workspace=ws)
    assert gdn.gdn_get_device_error(ws) == gdn.GDN_OK
    o_ref, S_ref = oracle_prefill(x)
    assert err(o, o_ref) < TOL[torch.bfloat16] and err(S, S_ref) < TOL[torch.bfloat16]


def test_error_word_stays_clear_on_success():
    x = _case()
    ws = gdn.prefill_workspace(2, 137, 2, 128, 128)
    for _ in range(3):
        gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"],
                        workspace=ws)
    assert gdn.gdn_get_device_error(ws) == gdn.GDN_OK
