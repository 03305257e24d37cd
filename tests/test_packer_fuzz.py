"""Property test of the host token packer (C ABI) against the oracle's own packer (no GPU).

Random segment lists (every role, frame counts, tokens per frame, Picture indices, start times,
frame spacings, static and per-frame masks) must pack to bit-identical arrays.
"""
import numpy as np
from hypothesis import HealthCheck, given, settings, strategies as st

import oracle
import workloads as W
from video_diffusion_attention_b200 import _binding as B


@st.composite
def segment(draw):
    kind = draw(st.sampled_from([W.TEXT, W.PICTURE, W.TARGET, W.GUIDE, W.AUDIO, W.OTHER_VIDEO]))
    frames = draw(st.integers(1, 4))
    tpf = draw(st.integers(1, 40))
    pic = draw(st.integers(1, 9)) if kind == W.PICTURE else 0
    t0 = draw(st.floats(-2.0, 5.0, allow_nan=False, width=32))
    dt = draw(st.floats(0.0, 0.5, allow_nan=False, width=32))
    mask = None
    if kind == W.TARGET and draw(st.booleans()):
        n = tpf if draw(st.booleans()) else frames * tpf
        seed = draw(st.integers(0, 2**31 - 1))
        mask = np.random.Generator(np.random.PCG64(seed)).uniform(0, 1, n).astype(np.float32)
    return W.Segment(kind, frames, tpf, pic=pic, t0_s=float(t0), frame_dt_s=float(dt), mask=mask)


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(st.lists(segment(), min_size=1, max_size=8))
def test_packer_matches_oracle_on_random_layouts(segs):
    B.load_library()
    a = B.pack_token_meta(segs)
    b = oracle.pack_token_meta(segs)
    assert B.packed_length(segs) == len(b["seg"])
    for key in ("seg", "time_s", "pic", "m"):
        np.testing.assert_array_equal(a[key].view(np.uint8), b[key].view(np.uint8))
