"""INT8 Q K^T variant on the CUDA path vs the INT8-QK^T oracle (needs a B200).

"TARA: Native Temporal Alignment for MiniMax H3 References", section "Three backends": the
one-pass kernels run the rule on dense INT8 attention.  The codes and scales are integer /
exactly-specified float32 decisions and must match the oracle bit for bit; the attention
output is compared with the oracle evaluated on the same codes, within the 16-bit bar.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import int8_qk
import workloads as W
from parity_util import compare, rows_from_sample, run_gpu, run_oracle_int8

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _codes_match(q, k, heads=None):
    import video_diffusion_attention_b200 as T
    qc, qs, kc, ks = T.quantize_qk_int8(q, k)
    torch.cuda.synchronize()
    dtype = oracle.torch_to_numpy_raw(q[:, :1])[1]
    heads = range(q.shape[1]) if heads is None else heads
    for h in heads:
        qf = int8_qk._widen_f32(oracle.torch_to_numpy_raw(q[:, h:h + 1])[0], dtype)
        kf = int8_qk._widen_f32(oracle.torch_to_numpy_raw(k[:, h:h + 1])[0], dtype)
        cq, sq = int8_qk.quantise_q(qf)
        ck, sk = int8_qk.quantise_k(kf)
        np.testing.assert_array_equal(qc[:, h:h + 1].cpu().numpy(), cq)
        np.testing.assert_array_equal(kc[:, h:h + 1].cpu().numpy(), ck)
        np.testing.assert_array_equal(qs[:, h:h + 1].cpu().numpy().view(np.uint32), sq.view(np.uint32))
        np.testing.assert_array_equal(ks[:, h:h + 1].cpu().numpy().view(np.uint32), sk.view(np.uint32))


def _check(w, rows=None, m_extra=None, qkv=None):
    q, k, v = qkv if qkv is not None else (t.to(DEV) for t in W.make_qkv(w, DEV))
    O, L = run_gpu(w, q, k, v, m_extra=m_extra, qk_int8=1)
    if rows is None:
        rows = oracle.all_rows(w.B, w.H, w.N)
    Oref, Lref = run_oracle_int8(w, q, k, v, rows, m_extra=m_extra)
    return compare(w, O, L, rows, Oref, Lref, w.dtype)


def _layout(tpf=64, frames=6):
    return [
        W.Segment(W.TEXT, 1, 37),
        W.Segment(W.PICTURE, 1, 300, pic=1),
        W.Segment(W.TARGET, frames, tpf, frame_dt_s=4 / 24, mask=W.uniform_mask(31, tpf)),
        W.Segment(W.GUIDE, frames, tpf, frame_dt_s=4 / 24),
        W.Segment(W.AUDIO, 1, 29),
    ]


GAINS = W.Params(gain=(1.4, 0.7) + (1.0,) * 7)


# ---------------------------------------------------------------------------------------
# the codes, bit for bit
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("N", [1, 127, 300])
def test_codes_bit_exact(dtype, D, N):
    w = W.custom("qc", B=2, H=3, D=D, dtype=dtype, segments=[W.Segment(W.TEXT, 1, N)],
                 qk_scale=2.0, seed_index=800 + N)
    q, k, _ = (t.to(DEV) for t in W.make_qkv(w, DEV))
    _codes_match(q, k)


def test_codes_bit_exact_zero_and_tiny_groups():
    w = W.custom("qz", B=1, H=2, D=128, dtype="bf16", segments=[W.Segment(W.TEXT, 1, 260)],
                 seed_index=810)
    q, k, _ = (t.to(DEV) for t in W.make_qkv(w, DEV))
    q[0, 0, 5] = 0.0                   # an all-zero Q row
    q[0, 1, 7] = 1e-32                 # a row below the amax floor (bf16 keeps it nonzero)
    k[0, 0, 128:256] = 0.0             # an all-zero K block
    _codes_match(q, k)


def test_codes_bit_exact_full_shot_heads():
    w = W.get("full")
    q, k, _ = (t.to(DEV) for t in W.make_qkv(w, DEV))
    _codes_match(q, k, heads=[0, 17, 55])


# ---------------------------------------------------------------------------------------
# the forward pass
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_forward_small(dtype):
    w = W.custom("q8", B=1, H=3, D=128, dtype=dtype, segments=_layout(), params=GAINS,
                 qk_scale=1.5, seed_index=820)
    _check(w)


def test_forward_medium_all_rows():
    _check(W.get("medium"))


@pytest.mark.parametrize("N", [1, 2, 127, 129, 383])
def test_forward_ragged_lengths(N):
    nt, ng = N // 3, N // 3
    segs = [W.Segment(W.TEXT, 1, N - nt - ng)] if N - nt - ng > 0 else []
    if nt:
        segs.append(W.Segment(W.TARGET, 1, nt, frame_dt_s=4 / 24))
    if ng:
        segs.append(W.Segment(W.GUIDE, 1, ng, t0_s=0.5))
    _check(W.custom("q8len", B=1, H=2, D=128, dtype="bf16", segments=segs, seed_index=830 + N))


def test_forward_zero_rows_and_blocks():
    # an all-zero Q row (scale 0) and an all-zero K tile (scale 0), past the ragged tail
    w = W.custom("q8z", B=1, H=2, D=128, dtype="bf16", segments=_layout(tpf=50, frames=5),
                 params=GAINS, seed_index=840)
    q, k, v = (t.to(DEV) for t in W.make_qkv(w, DEV))
    q[0, 0, 3] = 0.0
    q[0, 1, 200:260] = 0.0
    k[0, 1, 128:256] = 0.0
    _check(w, qkv=(q, k, v))


def test_forward_every_tile_class_and_chained_bindings():
    segs = [
        W.Segment(W.TEXT, 1, 64),
        W.Segment(W.PICTURE, 1, 384, pic=1),
        W.Segment(W.PICTURE, 1, 256, pic=2),
        W.Segment(W.TARGET, 10, 128, frame_dt_s=4 / 24, mask=W.uniform_mask(9, 128)),
        W.Segment(W.GUIDE, 10, 128, frame_dt_s=4 / 24),
        W.Segment(W.AUDIO, 1, 100),
    ]
    p = W.Params(gain=(1.25, 0.75) + (1.0,) * 7, extra_gain=((0.8, 1.5) + (1.0,) * 7,))
    w = W.custom("q8cls", B=1, H=2, D=128, dtype="bf16", segments=segs, params=p, qk_scale=1.5,
                 seed_index=850)
    _check(w, m_extra=W.chained_masks(w, 1))


def test_forward_full_shot_sampled_rows():
    w = W.get("full")
    sample = {key: val for key, val in W.sample_rows(w, per_head=256).items()
              if key[1] in (0, 29, 55)}
    _check(w, rows=rows_from_sample(sample))


def test_int8_stays_near_the_16bit_path():
    # the quantised logits move by a few hundredths at most on these inputs: O stays close to
    # the 16-bit result (a sanity check of the scales, not a parity bar)
    w = W.get("medium")
    q, k, v = (t.to(DEV) for t in W.make_qkv(w, DEV))
    O8, L8 = run_gpu(w, q, k, v, qk_int8=1)
    O16, L16 = run_gpu(w, q, k, v)
    assert (L8 - L16).abs().max().item() < 0.05
    assert (O8.float() - O16.float()).abs().mean().item() < 0.01


def test_forward_per_branch_metadata():
    # two branches with their own metadata (batch-strided) through the 8-bit path
    import video_diffusion_attention_b200 as T
    w = W.custom("q8pb", B=2, H=2, D=128, dtype="bf16", segments=_layout(tpf=40, frames=4),
                 params=GAINS, seed_index=860)
    q, k, v = (t.to(DEV) for t in W.make_qkv(w, DEV))
    meta = T.pack_token_meta(w.segments)
    N = len(meta["seg"])
    stacked = {key: np.concatenate([val] * w.B) for key, val in meta.items()}
    O, L = T.attn_forward(q, k, v, T.DeviceMeta(stacked, DEV, batch_stride=N, N=N),
                          T.params_from(w.params, 1))
    torch.cuda.synchronize()
    assert T.device_status() == 0
    rows = oracle.all_rows(w.B, w.H, w.N)
    from parity_util import run_oracle_int8
    Oref, Lref = run_oracle_int8(w, q, k, v, rows)
    compare(w, O, L, rows, Oref, Lref, w.dtype)
