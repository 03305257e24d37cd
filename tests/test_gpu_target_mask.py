"""Target-mask preparation on the device vs the fp64 oracle, and fed into the forward pass."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import compare, run_oracle
from video_diffusion_attention_b200 import _binding as B

pytestmark = pytest.mark.gpu

CASES = [
    # (F_in, Hp, Wp, shot_len, tau, F_lat, Hq, Wq)
    (1, 80, 100, 107, 4, 26, 40, 50),        # static mask, integer ratio
    (107, 80, 100, 107, 4, 26, 40, 50),      # one mask per frame of a 107-frame shot
    (22, 45, 61, 22, 4, 6, 9, 13),           # fractional ratios, short last span
    (5, 7, 10, 5, 1, 5, 3, 4),               # tiny, one pixel frame per latent frame
    (39, 20, 24, 39, 4, 10, 40, 50),         # upsampling (patch grid finer than the mask)
    (107, 720, 1280, 107, 4, 27, 40, 50),    # pixel-resolution mask of the full shot
    (107, 544, 928, 107, 4, 27, 40, 50),     # the pages' user-run resolution (narrow rows)
    (22, 33, 1024, 22, 4, 6, 7, 50),         # widest narrow-row case
    (22, 33, 516, 22, 4, 6, 7, 50),          # narrow rows: only thread 0 has a second column group
    (1, 17, 508, 107, 4, 26, 5, 9),          # static narrow mask, no second column group
    (22, 33, 1028, 22, 4, 6, 7, 50),         # just past it: the general kernel
]


@pytest.mark.parametrize("case", CASES)
def test_mask_prep_matches_oracle(case):
    F_in, Hp, Wp, L, tau, F_lat, Hq, Wq = case
    m = W.pixel_ellipse_mask(77 + F_in, F_in, Hp, Wp)
    out = B.prepare_target_mask(torch.from_numpy(m).cuda(), L, tau, F_lat, Hq, Wq)
    torch.cuda.synchronize()
    ref = oracle.prepare_target_mask(m, L, F_lat, tau, Hq, Wq)
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref).max()
    assert err <= 1e-5, err


def test_mask_prep_rejects_lengths_on_device():
    m = torch.zeros((360, 8, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(B.TaraError) as e:
        B.prepare_target_mask(m, 107, 4, 26, 4, 4)      # whole-clip mask into a 107-frame shot
    assert e.value.code == -12


def test_prepared_mask_drives_the_binding_gain():
    # mask (pixels, per frame) -> m on the device -> token metadata -> forward, against the
    # oracle fed with its own preparation of the same mask
    L, tau, F, Hq, Wq = 22, 4, 6, 8, 10
    segs = [W.Segment(W.TEXT, 1, 40), W.Segment(W.PICTURE, 1, 150, pic=1),
            W.Segment(W.TARGET, F, Hq * Wq, frame_dt_s=4 / 24),
            W.Segment(W.GUIDE, F, Hq * Wq, frame_dt_s=4 / 24), W.Segment(W.AUDIO, 1, 30)]
    w = W.custom("maskfwd", B=1, H=2, D=128, dtype="bf16", segments=segs,
                 params=W.Params(gain=(1.8,) + (1.0,) * 8), qk_scale=1.5, seed_index=600)
    px = W.pixel_ellipse_mask(5, L, 64, 80)
    m_dev = B.prepare_target_mask(torch.from_numpy(px).cuda(), L, tau, F, Hq, Wq)
    meta = B.pack_token_meta(segs)
    dmeta = B.DeviceMeta(meta, "cuda")
    start = 40 + 150
    dmeta.m[start:start + F * Hq * Wq].copy_(m_dev.reshape(-1))
    q, k, v = W.make_qkv(w, "cuda")
    O, Lse = B.attn_forward(q, k, v, dmeta, B.params_from(w.params))
    torch.cuda.synchronize()
    m_ref = oracle.prepare_target_mask(px, L, F, tau, Hq, Wq).astype(np.float32)
    segs_ref = list(segs)
    segs_ref[2] = W.Segment(W.TARGET, F, Hq * Wq, frame_dt_s=4 / 24, mask=m_ref.reshape(-1))
    w_ref = W.custom("maskfwd", B=1, H=2, D=128, dtype="bf16", segments=segs_ref,
                     params=w.params, qk_scale=1.5, seed_index=600)
    rows = oracle.all_rows(w.B, w.H, w.N)
    Oref, Lref = run_oracle(w_ref, q, k, v, rows)
    compare(w_ref, O, Lse, rows, Oref, Lref, "bf16")
