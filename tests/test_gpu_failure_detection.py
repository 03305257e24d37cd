"""Failure detection on the GPU without faulting it: a bounded wait that runs out.

A self-test kernel waits on a barrier nothing arrives on; after its short limit it gives up
and sets the per-device status word, the host reads TARA_ERR_DEVICE_TIMEOUT once, the word is
cleared, and the context stays usable for the attention kernels.
"""
import pytest
import torch

import workloads as W
from video_diffusion_attention_b200 import _binding as B

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_then_cleared():
    assert B.device_status() == 0
    B.selftest_wait(20_000, arrive=False)        # 20 ms limit, nothing arrives
    assert B.device_status() == -10               # TARA_ERR_DEVICE_TIMEOUT
    assert B.device_status() == 0                 # read once, then cleared


def test_wait_that_completes_sets_nothing():
    B.selftest_wait(20_000, arrive=True)
    assert B.device_status() == 0


def test_attention_runs_normally_after_a_reported_timeout():
    B.selftest_wait(5_000, arrive=False)
    assert B.device_status() == -10
    w = W.custom("after", B=1, H=1, D=128, dtype="bf16", segments=[
        W.Segment(W.TEXT, 1, 50), W.Segment(W.TARGET, 3, 40, frame_dt_s=4 / 24),
        W.Segment(W.GUIDE, 3, 40, frame_dt_s=4 / 24)], seed_index=500)
    q, k, v = W.make_qkv(w, "cuda")
    meta = B.DeviceMeta(B.pack_token_meta(w.segments), q.device)
    O, L = B.attn_forward(q, k, v, meta, B.params_from(w.params))
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert torch.isfinite(O.float()).all() and torch.isfinite(L).all()
    # same inputs through plain attention where no bias applies: the text rows
    s = (q.float()[0, 0, :50] @ k.float()[0, 0].T) / 128 ** 0.5
    ref = torch.softmax(s, dim=-1) @ v.float()[0, 0]
    assert (O.float()[0, 0, :50] - ref).abs().max().item() < 1.5e-2


def test_rejects_limits_out_of_range():
    with pytest.raises(B.TaraError):
        B.selftest_wait(0, arrive=False)
