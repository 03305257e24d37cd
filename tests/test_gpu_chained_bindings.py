"""Chained bindings on the CUDA path vs the fp64 oracle (needs a B200).

Two subjects bound to two Pictures are two chained binding nodes; where their masks overlap,
a target query adds the log gains of both ("BFS H3 Reference Attention Binding
(Experimental)", section "Common issues").  Every call here carries one to three bindings
beyond the first, with overlapping masks, through the C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import compare, rows_from_sample, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _check(w, n_extra, per_branch_meta=False, rows=None):
    q, k, v = (t.to(DEV) for t in W.make_qkv(w, DEV))
    mx = W.chained_masks(w, n_extra)
    O, L = run_gpu(w, q, k, v, per_branch_meta=per_branch_meta, m_extra=mx)
    if rows is None:
        rows = oracle.all_rows(w.B, w.H, w.N)
    Oref, Lref = run_oracle(w, q, k, v, rows, m_extra=mx)
    return compare(w, O, L, rows, Oref, Lref, w.dtype)


def _layout(tpf=64, frames=6):
    # a long single-picture run (constant-picture tiles), a short picture sharing tiles with
    # text (per-edge tiles), target and guide videos, and a picture only the extra bindings
    # weight (its first-binding gain is 1)
    return [
        W.Segment(W.TEXT, 1, 40),
        W.Segment(W.PICTURE, 1, 300, pic=1),
        W.Segment(W.PICTURE, 1, 70, pic=2),
        W.Segment(W.PICTURE, 1, 90, pic=3),
        W.Segment(W.TARGET, frames, tpf, frame_dt_s=4 / 24, mask=W.uniform_mask(21, tpf)),
        W.Segment(W.GUIDE, frames, tpf, frame_dt_s=4 / 24),
        W.Segment(W.AUDIO, 1, 33),
    ]


def _params(n_extra):
    extra = [(0.6, 1.8) + (1.0,) * 7,            # binding 2: Picture 2 up, Picture 1 down
             (1.0, 1.0, 2.5) + (1.0,) * 6,       # binding 3: Picture 3 only
             (1.3,) * 9][:n_extra]               # binding 4: every Picture
    return W.Params(gain=(1.6, 0.8) + (1.0,) * 7, extra_gain=tuple(extra))


def _small(name, dtype, D, n_extra, H=2, B=1, seed=700):
    return W.custom(name, B=B, H=H, D=D, dtype=dtype, segments=_layout(),
                    params=_params(n_extra), seed_index=seed)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("n_extra", [1, 3])
def test_chained_tensor_core(dtype, D, n_extra):
    _check(_small("ch", dtype, D, n_extra, seed=700 + n_extra), n_extra)


@pytest.mark.parametrize("n_extra", [1, 2, 3])
def test_chained_fp32(n_extra):
    w = W.custom("chf", B=1, H=2, D=64, dtype="fp32", segments=_layout(tpf=24, frames=5),
                 params=_params(n_extra), seed_index=720 + n_extra)
    _check(w, n_extra)


def test_chained_batch_strided_meta():
    w = _small("chb", "bf16", 128, 2, H=2, B=2, seed=730)
    _check(w, 2, per_branch_meta=True)


def test_chained_full_shot_sampled_rows():
    # the full-size shot with two extra subjects whose masks overlap the first binding's
    base = W.get("full")
    segs = base.segments
    gains = (1.5,) + (1.0,) * 8
    w = W.custom("chfull", B=base.B, H=base.H, D=base.D, dtype=base.dtype, segments=segs,
                 params=W.Params(gain=gains, extra_gain=((0.7, 1.3) + (1.0,) * 7,
                                                         (1.4,) + (1.0,) * 8)),
                 qk_scale=base.qk_scale, seed_index=base.index)
    _check(w, 2, rows=rows_from_sample(W.sample_rows(w, per_head=256)))


def test_neutral_extra_bindings_are_bit_identical():
    # extra bindings whose gains are all 1 add ln(1) = 0 to every edge
    import video_diffusion_attention_b200 as T
    w = _small("chn", "bf16", 128, 0, seed=740)
    q, k, v = (t.to(DEV) for t in W.make_qkv(w, DEV))
    O0, L0 = run_gpu(w, q, k, v)
    w.params = W.Params(gain=w.params.gain, extra_gain=((1.0,) * 9, (1.0,) * 9))
    O1, L1 = run_gpu(w, q, k, v, m_extra=W.chained_masks(w, 2))
    assert torch.equal(O0, O1) and torch.equal(L0, L1)
    assert T.device_status() == 0
