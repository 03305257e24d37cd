"""The debug build (libtara_attn_debug.so, compiled with -DTARA_DEBUG=1): its kernels check on
the device what the host cannot see and record a failed check in the status word instead of
trapping.  On valid inputs it reports nothing and matches the oracle like the release build;
on a target token whose clock is not a number it reports TARA_ERR_DEBUG_CHECK, where the
release build, which has no such checks, reports nothing.  No case faults or traps."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_util import TOL
from video_diffusion_attention_b200 import _binding as B
from video_diffusion_attention_b200 import build as libbuild


@pytest.fixture(scope="module")
def dlib():
    libbuild.build(debug=True)
    lib = B.load_library(libbuild.LIB_DEBUG)
    assert lib.tara_debug_build() == 1
    return lib


def _forward(lib, w, q, k, v, meta):
    dev = q.device
    O = torch.empty_like(q)
    L = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    cq, ck, cv, co = (B.tensor_struct(t) for t in (q, k, v, O))
    cm = meta.c_struct()
    p = B.params_from(w.params)
    stream = torch.cuda.current_stream(dev)
    rc = lib.tara_attn_forward(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv),
                               ctypes.byref(cm), ctypes.byref(p), ctypes.byref(co),
                               ctypes.c_void_p(L.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
    assert rc == 0, rc
    status = lib.tara_device_status(ctypes.c_void_p(stream.cuda_stream))
    return O, L, status


def _ragged(N, D, dtype):
    tgt = (N - 40) // 2
    return W.custom("dbg%d" % N, B=1, H=2, D=D, dtype=dtype, segments=[
        W.Segment(W.TEXT, 1, 9), W.Segment(W.PICTURE, 1, 13, pic=1),
        W.Segment(W.TARGET, 1, tgt, frame_dt_s=4 / 24, mask=W.uniform_mask(5, tgt)),
        W.Segment(W.GUIDE, 1, N - 40 - tgt, frame_dt_s=4 / 24), W.Segment(W.AUDIO, 1, 18),
    ], params=W.Params(gain=(1.25,) + (1.0,) * 8), seed_index=77)


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["tiny", "ragged129_d128", "ragged129_d64"])
def test_debug_build_reports_nothing_and_matches_the_oracle(dlib, case):
    dev = torch.device("cuda:0")
    if case == "tiny":
        w = W.get("tiny")
    else:
        w = _ragged(129, 128 if case.endswith("128") else 64, "bf16")
    q, k, v = W.make_qkv(w, dev)
    meta = B.DeviceMeta(B.pack_token_meta(w.segments), dev)
    O, L, status = _forward(dlib, w, q, k, v, meta)
    assert status == 0
    raw = [oracle.torch_to_numpy_raw(t) for t in (q, k, v)]
    Oref, Lref = oracle.attention_rows(raw[0][0], raw[1][0], raw[2][0], raw[0][1],
                                       oracle.pack_token_meta(w.segments), w.params,
                                       oracle.all_rows(w.B, w.H, w.N))
    tol = TOL[w.dtype]
    d_o = np.abs(O.float().cpu().numpy().reshape(-1, w.D) - Oref)
    d_l = np.abs(L.cpu().numpy().reshape(-1) - Lref)
    assert d_o.max() <= tol["o_max"] and d_o.mean() <= tol["o_mean"] and d_l.max() <= tol["lse_max"]


@pytest.mark.gpu
@pytest.mark.parametrize("D", [128, 64])
def test_debug_build_flags_a_target_clock_that_is_not_a_number(dlib, D):
    dev = torch.device("cuda:0")
    w = _ragged(129, D, "bf16")
    q, k, v = W.make_qkv(w, dev)
    packed = B.pack_token_meta(w.segments)
    first_target = int(np.nonzero(packed["seg"] == W.TARGET)[0][0])
    packed["time_s"] = packed["time_s"].copy()
    packed["time_s"][first_target] = np.float32("nan")
    meta = B.DeviceMeta(packed, dev)
    _, _, status = _forward(dlib, w, q, k, v, meta)
    assert status == {v: k for k, v in B.STATUS.items()}["TARA_ERR_DEBUG_CHECK"]
    # the word was cleared: a valid call afterwards reports nothing
    ok_meta = B.DeviceMeta(B.pack_token_meta(w.segments), dev)
    assert _forward(dlib, w, q, k, v, ok_meta)[2] == 0
    # the release build has no device-side checks
    rel = B.load_library()
    assert rel.tara_debug_build() == 0
    assert _forward(rel, w, q, k, v, meta)[2] == 0
