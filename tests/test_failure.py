"""Failure handling without a GPU fault: the tensor-core prefill's bounded waits are
made to give up at once (gdn_set_wait_budget(0)), the kernel records GDN_ERR_TIMEOUT in
the workspace, lets its own copies and MMAs finish, frees its TMEM and exits; the
context stays usable and the next call is correct.  Every schedule is covered: the
single-CTA kernel with one unit per sequence and with segments (transfer pass, scan,
output pass), and the four-CTA cluster kernel."""
from __future__ import annotations

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


@pytest.mark.parametrize("segment", [-1, 64, -2])
def test_timeout_is_reported_and_recoverable(segment):
    x = _case()
    gdn.gdn_set_prefill_segment_tokens(segment)
    try:
        ws = gdn.prefill_workspace(2, 137, 2, 128, 128)
        old = gdn.gdn_set_wait_budget(0)
        try:
            gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"],
                            workspace=ws)
            status = gdn.gdn_get_device_error(ws)
        finally:
            gdn.gdn_set_wait_budget(old)
        assert status == gdn.GDN_ERR_TIMEOUT
        assert gdn.gdn_get_device_error(ws) == gdn.GDN_OK          # read clears it
        o, S = gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"],
                               workspace=ws)
        assert gdn.gdn_get_device_error(ws) == gdn.GDN_OK
    finally:
        gdn.gdn_set_prefill_segment_tokens(0)
    o_ref, S_ref = oracle_prefill(x)
    assert err(o, o_ref) < TOL[torch.bfloat16] and err(S, S_ref) < TOL[torch.bfloat16]


def test_error_word_stays_clear_on_success():
    x = _case()
    ws = gdn.prefill_workspace(2, 137, 2, 128, 128)
    for _ in range(3):
        gdn.gdn_prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"],
                        workspace=ws)
    assert gdn.gdn_get_device_error(ws) == gdn.GDN_OK
