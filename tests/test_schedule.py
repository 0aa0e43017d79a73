"""The prefill dispatcher (gdn_prefill_schedule): which kernel and segment length a call
gets, how the override and the workspace size steer it, and that the workspace a
segmented call asks for holds its intermediates.  Runs on CPU: with no device the
library plans for a 148-SM B200."""
from __future__ import annotations

import pytest
import torch

import linear_attention_token_b200 as gdn


@pytest.fixture(autouse=True)
def _automatic():
    gdn.gdn_set_prefill_segment_tokens(0)
    yield
    gdn.gdn_set_prefill_segment_tokens(0)


def test_workload_schedules():
    # long context, 16 heads: segments (local + transfer chains, scan, correction)
    long = gdn.gdn_prefill_schedule(1, 262144, 16, 128, 128)
    assert long["kernel"] == "chain" and long["segment_tokens"] > 0
    assert long["segment_tokens"] % 64 == 0 and long["launches"] == 3
    # varlen adds the device-side unit table
    assert gdn.gdn_prefill_schedule(1, 262144, 16, 128, 128, varlen=True)["launches"] == 4
    # many heads over short sequences: the four-CTA cluster kernel
    assert gdn.gdn_prefill_schedule(2, 8192, 16, 128, 128)["kernel"] == "cluster"
    # 8 sequences x 16 heads fill the GPU: one unit per sequence, no segments
    assert gdn.gdn_prefill_schedule(8, 122112, 16, 128, 128, varlen=True) == \
        {"kernel": "chain", "segment_tokens": 0, "launches": 1}


def test_segments_grow_with_the_sequence():
    s1 = gdn.gdn_prefill_schedule(1, 262144, 16, 128, 128)["segment_tokens"]
    s2 = gdn.gdn_prefill_schedule(1, 1048576, 16, 128, 128)["segment_tokens"]
    assert 0 < s1 < s2


@pytest.mark.parametrize("dk,dv,dtype", [(64, 128, torch.bfloat16), (128, 64, torch.bfloat16),
                                         (128, 128, torch.float32)])
def test_cuda_core_shapes(dk, dv, dtype):
    """fp32 and 64-wide heads run on the CUDA-core kernel."""
    assert gdn.gdn_prefill_schedule(2, 8192, 16, dk, dv, dtype=dtype)["kernel"] == "cuda_core"


def test_nothing_to_do():
    assert gdn.gdn_prefill_schedule(0, 0, 16, 128, 128)["launches"] == 0


def test_overrides():
    gdn.gdn_set_prefill_segment_tokens(-1)
    assert gdn.gdn_prefill_schedule(1, 262144, 16, 128, 128) == \
        {"kernel": "chain", "segment_tokens": 0, "launches": 1}
    gdn.gdn_set_prefill_segment_tokens(-2)
    assert gdn.gdn_prefill_schedule(1, 262144, 16, 128, 128)["kernel"] == "cluster"
    gdn.gdn_set_prefill_segment_tokens(128)
    assert gdn.gdn_prefill_schedule(1, 262144, 16, 128, 128)["segment_tokens"] == 128
    with pytest.raises(gdn.GdnError):
        gdn.gdn_set_prefill_segment_tokens(100)            # not a multiple of 64


def test_small_workspace_falls_back_to_one_unit():
    """A workspace too small for the segment intermediates: one unit per sequence."""
    s = gdn.gdn_prefill_schedule(1, 262144, 16, 128, 128, workspace_bytes=256)
    assert s == {"kernel": "chain", "segment_tokens": 0, "launches": 1}


def test_segmented_workspace_holds_its_intermediates():
    T, H = 262144, 16
    seg = gdn.gdn_prefill_schedule(1, T, H, 128, 128)["segment_tokens"]
    units = -(-T // seg)
    need = T * H * 128 * 2 + 3 * units * H * 128 * 128 * 4     # Psi, and M, B, S_in per unit
    assert gdn.gdn_prefill_workspace_size(1, T, H, 128, 128) >= need
    assert gdn.gdn_prefill_workspace_size(2, 8192, 16, 128, 128) == 256   # no segments
