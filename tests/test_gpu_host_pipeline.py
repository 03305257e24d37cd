"""tara_attn_forward_host: the forward on host buffers (needs a B200).

Every (branch, head) plane is computed by the same kernels as tara_attn_forward on device
buffers, so the chunked three-stream pipeline must reproduce the device-buffer result bit for
bit, across chunk boundaries (a 1, 2, 4, ... ramp at both ends, kernels of consecutive chunks
on alternating streams), branch cuts of per-branch metadata, extra bindings and the INT8 QK^T
variant.
"""
import numpy as np
import pytest
import torch

import video_diffusion_attention_b200 as T
import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _both(w, per_branch_meta=False, m_extra=None, qk_int8=0):
    q, k, v = (t.to(DEV) for t in W.make_qkv(w, DEV))
    meta = T.pack_token_meta(w.segments)
    N = len(meta["seg"])
    stride = 0
    if per_branch_meta:
        meta = {key: np.concatenate([val] * w.B) for key, val in meta.items()}
        stride = N
    if m_extra is not None:
        meta["m_extra"] = np.concatenate([np.asarray(m_extra, np.float32)] * (w.B if per_branch_meta else 1), axis=1)
    params = T.params_from(w.params, qk_int8)
    O_d, L_d = T.attn_forward(q, k, v, T.DeviceMeta(meta, DEV, batch_stride=stride, N=N), params)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    del q, k, v
    O_h, L_h = T.attn_forward_host(hq, hk, hv, T.HostMeta(meta, batch_stride=stride, N=N), params)
    torch.cuda.synchronize()
    assert T.device_status() == 0
    assert torch.equal(O_h, O_d.cpu())
    assert torch.equal(L_h, L_d.cpu())


def test_single_chunk_fp32():
    _both(W.get("tiny"))


def test_single_chunk_bf16_int8():
    _both(W.get("medium"), qk_int8=1)


def test_full_shot_ramped_chunks():
    # 56 heads of 27.4 MB planes: chunks of 1, 2, 4, 8, 9, 9, 8, 8, 4, 2, 1 planes
    _both(W.get("full"))


def test_ramp_cut_at_branches_int8():
    # 2 branches x 5 heads with per-branch metadata: the ramp 1, 2, 4, 2, 1 is cut at the
    # branch boundary (planes 3-6 become 3-4 and 5-6); INT8 quantisation per chunk
    w = W.custom("hramp", B=2, H=5, D=128, dtype="bf16", segments=[
        W.Segment(W.TEXT, 1, 70), W.Segment(W.PICTURE, 1, 200, pic=1),
        W.Segment(W.TARGET, 4, 120, frame_dt_s=4 / 24, mask=W.uniform_mask(5, 120)),
        W.Segment(W.GUIDE, 4, 97, frame_dt_s=4 / 24), W.Segment(W.AUDIO, 1, 33)],
        params=W.Params(gain=(1.4,) + (1.0,) * 8), seed_index=910)
    _both(w, per_branch_meta=True, qk_int8=1)


def test_per_branch_metadata_chunks_cut_at_branches():
    # 2 branches x 56 heads with per-branch metadata: chunks stay inside a branch
    _both(W.get("ragged"), per_branch_meta=True)


def test_chained_bindings_through_host_buffers():
    w = W.custom("hch", B=2, H=3, D=128, dtype="bf16", segments=[
        W.Segment(W.TEXT, 1, 40), W.Segment(W.PICTURE, 1, 300, pic=1),
        W.Segment(W.PICTURE, 1, 90, pic=2),
        W.Segment(W.TARGET, 5, 64, frame_dt_s=4 / 24, mask=W.uniform_mask(3, 64)),
        W.Segment(W.GUIDE, 5, 64, frame_dt_s=4 / 24)],
        params=W.Params(gain=(1.3, 0.8) + (1.0,) * 7, extra_gain=((0.7, 1.6) + (1.0,) * 7,)),
        seed_index=900)
    _both(w, per_branch_meta=True, m_extra=W.chained_masks(w, 1))


def test_ordering_on_a_side_stream():
    # work queued on a user stream: the call returns at once and the stream carries the result
    w = W.get("medium")
    q, k, v = (t.to(DEV) for t in W.make_qkv(w, DEV))
    meta = T.pack_token_meta(w.segments)
    params = T.params_from(w.params)
    O_d, L_d = T.attn_forward(q, k, v, T.DeviceMeta(meta, DEV), params)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    s = torch.cuda.Stream()
    out = torch.zeros_like(hq).pin_memory()
    lse = torch.zeros((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    for _ in range(2):   # a second call reuses the pipeline's buffers after the first
        T.attn_forward_host(hq, hk, hv, T.HostMeta(meta), params, out, lse, stream=s)
    s.synchronize()
    assert torch.equal(out, O_d.cpu()) and torch.equal(lse, L_d.cpu())
