"""CUDA path vs the fp64 oracle, element by element, through the C ABI (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import TOL, compare, rows_from_sample, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _check(w, rows=None, per_branch_meta=False, seed_device=DEV):
    q, k, v = W.make_qkv(w, seed_device)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    O, L = run_gpu(w, q, k, v, per_branch_meta=per_branch_meta)
    if rows is None:
        rows = oracle.all_rows(w.B, w.H, w.N)
    Oref, Lref = run_oracle(w, q, k, v, rows)
    return compare(w, O, L, rows, Oref, Lref, w.dtype)


# ---------------------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------------------
def test_tiny_fp32_all_rows():
    _check(W.get("tiny"))


def test_medium_bf16_all_rows():
    _check(W.get("medium"))


@pytest.mark.parametrize("name", ["micro", "full", "ragged"])
def test_large_sampled_rows(name):
    w = W.get(name)
    _check(w, rows_from_sample(W.sample_rows(w, per_head=256)))


def test_ragged_per_branch_metadata():
    # the same packing supplied once per CFG branch (batch-strided metadata)
    w = W.get("ragged")
    rows = rows_from_sample({k: v[:64] for k, v in W.sample_rows(w, per_head=64).items()
                             if k[1] < 4})
    _check(w, rows, per_branch_meta=True)


# ---------------------------------------------------------------------------------------
# dtypes and head dims
# ---------------------------------------------------------------------------------------
def _small(name, dtype, D, segs, params=None, H=2, B=1, qk=1.0, seed=200):
    return W.custom(name, B=B, H=H, D=D, dtype=dtype, segments=segs, params=params,
                    qk_scale=qk, seed_index=seed)


def _layout(tpf=40, frames=5, guide_t0=0.0, picture=(96, 1)):
    return [
        W.Segment(W.TEXT, 1, 37),
        W.Segment(W.PICTURE, 1, picture[0], pic=picture[1]),
        W.Segment(W.TARGET, frames, tpf, frame_dt_s=4 / 24,
                  mask=W.uniform_mask(7, tpf)),
        W.Segment(W.GUIDE, frames, tpf, t0_s=guide_t0, frame_dt_s=4 / 24),
        W.Segment(W.AUDIO, 1, 21),
    ]


GAINS = W.Params(gain=(1.25, 0.75) + (1.0,) * 7)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("D", [64, 128])
def test_dtype_headdim(dtype, D):
    w = _small("dt", dtype, D, _layout(tpf=64, frames=7), GAINS, H=3)
    _check(w)


def test_fp32_head_dim_128_and_odd():
    _check(_small("f32a", "fp32", 128, _layout(tpf=24, frames=6), GAINS))
    _check(_small("f32b", "fp32", 72, _layout(tpf=10, frames=6), GAINS))


# ---------------------------------------------------------------------------------------
# edge cases: sizes, tails, roles, parameters
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("N", [1, 2, 31, 127, 128, 129, 255, 257, 383])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_ragged_lengths(N, dtype):
    # one target frame block and one guide block split around the middle; plain text pads
    nt = N // 3
    ng = N // 3
    segs = [W.Segment(W.TEXT, 1, N - nt - ng)] if N - nt - ng > 0 else []
    if nt:
        segs.append(W.Segment(W.TARGET, 1, nt, frame_dt_s=4 / 24))
    if ng:
        segs.append(W.Segment(W.GUIDE, 1, ng, t0_s=0.5))
    D = 128 if dtype == "bf16" else 64
    _check(_small("len%d" % N, dtype, D, segs, W.Params(), H=2, seed=300 + N))


def test_no_target_rows_is_plain_attention():
    segs = [W.Segment(W.TEXT, 1, 200), W.Segment(W.GUIDE, 3, 50, frame_dt_s=0.2),
            W.Segment(W.PICTURE, 1, 60, pic=1)]
    _check(_small("notgt", "bf16", 128, segs, GAINS))


def test_every_tile_class():
    # constant-cap tiles (distant frames), constant-picture tiles (a long single picture),
    # zero tiles (near frames, no gain) and per-edge tiles (boundaries) in one call
    segs = [
        W.Segment(W.TEXT, 1, 64),
        W.Segment(W.PICTURE, 1, 384, pic=1),
        W.Segment(W.PICTURE, 1, 256, pic=2),
        W.Segment(W.TARGET, 10, 128, frame_dt_s=4 / 24, mask=W.uniform_mask(9, 128)),
        W.Segment(W.GUIDE, 10, 128, frame_dt_s=4 / 24),
        W.Segment(W.AUDIO, 1, 100),
    ]
    _check(_small("cls", "bf16", 128, segs, GAINS, H=2, qk=1.5))


@pytest.mark.parametrize("p", [
    W.Params(strength=0.0),
    W.Params(cap=0.0),
    W.Params(window=0.0, falloff=0.05, strength=5.0, cap=12.0),
    W.Params(window=1.0),
    W.Params(gain=(3.0,) + (0.2,) * 8),
    W.Params(softmax_scale=0.05),
])
def test_parameter_corners(p):
    _check(_small("par", "bf16", 128, _layout(tpf=50, frames=8), p, H=2))


@pytest.mark.parametrize("p", [
    W.Params(),
    W.Params(window=0.0, falloff=0.05, strength=5.0, cap=12.0),
    W.Params(window=0.3, falloff=1.0, strength=0.5, cap=2.0, gain=(1.5,) + (1.0,) * 8),
])
def test_single_frame_guide_tiles(p):
    # guide frames of exactly one 128-token tile: every near-diagonal guide key tile holds one
    # time, so the per-row guide class carries the temporal bias; the offset target start puts
    # query tiles across two target frames
    segs = [
        W.Segment(W.TEXT, 1, 128),
        W.Segment(W.PICTURE, 1, 128, pic=1),
        W.Segment(W.GUIDE, 9, 128, frame_dt_s=4 / 24),
        W.Segment(W.TARGET, 9, 128, t0_s=1 / 24, frame_dt_s=4 / 24, mask=W.uniform_mask(5, 128)),
        W.Segment(W.AUDIO, 1, 77),
    ]
    _check(_small("sfg", "bf16", 128, segs, p, H=2, qk=1.5, seed=410))


def test_unsorted_roles_and_other_video():
    # roles interleaved out of the usual order, plus a non-selected video reference
    segs = [
        W.Segment(W.GUIDE, 2, 70, t0_s=0.3, frame_dt_s=4 / 24),
        W.Segment(W.TARGET, 3, 45, frame_dt_s=4 / 24),
        W.Segment(W.PICTURE, 1, 33, pic=3),
        W.Segment(W.OTHER_VIDEO, 2, 40, frame_dt_s=4 / 24),
        W.Segment(W.TARGET, 2, 45, t0_s=0.5, frame_dt_s=4 / 24),
        W.Segment(W.TEXT, 1, 9),
    ]
    _check(_small("mix", "bf16", 128, segs, W.Params(gain=(1.0, 1.0, 2.0) + (1.0,) * 6)))


def test_batch_of_branches_shared_and_strided_meta():
    w = _small("br", "bf16", 128, _layout(tpf=40, frames=4), GAINS, H=2, B=3)
    _check(w)
    _check(w, per_branch_meta=True)


def test_calls_on_two_streams_do_not_share_summaries_concurrently():
    # two shots of the same length with different role layouts, launched back to back on two
    # streams: the library orders them on the shared workspace, so each matches its own
    # single-stream result bit for bit
    import video_diffusion_attention_b200 as T
    segs_a = _layout(tpf=64, frames=6)
    segs_b = [W.Segment(W.TEXT, 1, 37), W.Segment(W.PICTURE, 1, 96, pic=2),
              W.Segment(W.GUIDE, 6, 64, t0_s=0.3, frame_dt_s=4 / 24),
              W.Segment(W.TARGET, 6, 64, frame_dt_s=4 / 24), W.Segment(W.AUDIO, 1, 21)]
    wa = _small("sa", "bf16", 128, segs_a, GAINS, H=8, seed=600)
    wb = _small("sb", "bf16", 128, segs_b, GAINS, H=8, seed=601)
    assert wa.N == wb.N
    ins = [tuple(t.to(DEV) for t in W.make_qkv(w, DEV)) for w in (wa, wb)]
    metas = [T.DeviceMeta(T.pack_token_meta(w.segments), DEV) for w in (wa, wb)]
    params = [T.params_from(w.params) for w in (wa, wb)]
    ref = [T.attn_forward(*ins[i], metas[i], params[i]) for i in range(2)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for _ in range(3):
        for i in range(2):
            outs.append((i, T.attn_forward(*ins[i], metas[i], params[i], stream=streams[i])))
    torch.cuda.synchronize()
    assert T.device_status() == 0
    for i, (O, L) in outs:
        assert torch.equal(O, ref[i][0]) and torch.equal(L, ref[i][1])


@pytest.mark.parametrize("dtype,D", [("fp16", 128), ("bf16", 64)])
def test_full_length_shot_other_dtype_and_head_dim(dtype, D):
    # the 107,126-token layout at 8 heads in fp16, and with 64-wide heads, on sampled rows
    base = W.get("micro")
    w = W.custom("mic_%s_%d" % (dtype, D), B=1, H=4, D=D, dtype=dtype, segments=base.segments,
                 params=W.Params(gain=(1.25, 0.75) + (1.0,) * 7), seed_index=950 + D)
    _check(w, rows_from_sample(W.sample_rows(w, per_head=256)))


def test_many_branch_head_planes():
    # 3 x 700 (branch, head) planes: grid y/z well past one wave of CTAs per plane
    segs = [W.Segment(W.TEXT, 1, 20), W.Segment(W.PICTURE, 1, 60, pic=1),
            W.Segment(W.TARGET, 3, 50, frame_dt_s=4 / 24), W.Segment(W.GUIDE, 3, 50,
                                                                      frame_dt_s=4 / 24)]
    w = _small("bh", "bf16", 128, segs, GAINS, H=700, B=3, seed=960)
    rng = np.random.Generator(np.random.PCG64(3))
    b = rng.integers(0, 3, 600)
    h = rng.integers(0, 700, 600)
    i = rng.integers(0, w.N, 600)
    _check(w, np.stack([b, h, i], axis=1).astype(np.int64))
