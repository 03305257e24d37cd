"""tara_attn_forward_noalloc: the forward pass for callers that cannot allocate device memory.

Such callers (frameworks that own all device memory through their own pool, serving loops
that must not enter the allocator) get the same result as tara_attn_forward, with the
scratch taken from a fixed array inside the library instead of a cudaMalloc'd workspace.
The size checks of this entry point run on the CPU in test_abi_host.py.  This file is
collected last on purpose.
"""

import pytest
import torch

import workloads as W
from parity_util import TOL
from video_diffusion_attention_b200 import _binding as B


def _shot():
    return W.custom("noalloc", B=2, H=3, D=128, dtype="bf16", segments=[
        W.Segment(W.TEXT, 1, 70),
        W.Segment(W.PICTURE, 1, 200, pic=1),
        W.Segment(W.PICTURE, 1, 130, pic=2),
        W.Segment(W.TARGET, 9, 96, frame_dt_s=4 / 24, mask=W.uniform_mask(21, 96)),
        W.Segment(W.GUIDE, 9, 75, t0_s=1 / 24, frame_dt_s=4 / 24),
        W.Segment(W.AUDIO, 1, 45),
    ], params=W.Params(gain=(1.25, 0.75) + (1.0,) * 7), qk_scale=1.5, seed_index=400)


@pytest.mark.gpu
def test_noalloc_matches_forward_twice():
    w = _shot()
    dev = torch.device("cuda:0")
    q, k, v = W.make_qkv(w, dev)
    meta = B.DeviceMeta(B.pack_token_meta(w.segments), dev)
    params = B.params_from(w.params)
    O_ref, L_ref = B.attn_forward(q, k, v, meta, params)
    torch.cuda.synchronize()
    tol = TOL["bf16"]
    for call in range(2):   # two calls in a row share the same scratch array
        O = torch.full_like(q, float("nan"))
        L = torch.full((w.B, w.H, w.N), float("nan"), dtype=torch.float32, device=dev)
        B.attn_forward_noalloc(q, k, v, meta, params, O, L)
        torch.cuda.synchronize()
        assert B.device_status() == 0
        d_o = (O.float() - O_ref.float()).abs()
        d_l = (L - L_ref).abs()
        assert torch.isfinite(O.float()).all() and torch.isfinite(L).all()
        assert d_o.max().item() <= tol["o_max"], call
        assert d_o.mean().item() <= tol["o_mean"], call
        assert d_l.max().item() <= tol["lse_max"], call
        # the same kernels on the same inputs: the results are identical bit for bit
        assert torch.equal(O, O_ref) and torch.equal(L, L_ref), call
