"""The C ABI on the host (no GPU): exports, argument checks, and the token packer.

Every call to tara_attn_forward here fails its argument checks before anything touches a
device, so the fake pointers below are never dereferenced.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import workloads as W
from video_diffusion_attention_b200 import _binding as B
from video_diffusion_attention_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return B.load_library()


def declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names.update(re.findall(r"\b(tara_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_function(lib):
    names = declared_functions()
    assert {"tara_attn_forward", "tara_pack_token_meta", "tara_default_params"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert set(B.EXPORTS) <= names


def test_debug_build_flag(lib):
    # the release library has no device-side checks; its debug twin compiles them in
    assert lib.tara_debug_build() == 0
    dbg = B.load_library(libbuild.build(debug=True))
    assert dbg.tara_debug_build() == 1
    assert b"debug" in lib.tara_status_string(-13)


def test_status_strings(lib):
    for code in list(B.STATUS) + [-99]:
        assert lib.tara_status_string(code)


def test_default_params_are_the_pages_defaults(lib, golden_rule):
    p = B.default_params()
    for key in ("window", "falloff", "strength", "cap"):
        assert getattr(p, key) == pytest.approx(golden_rule[key][0], rel=1e-7)
    assert list(p.gain) == [1.0] * 9 and p.softmax_scale == 0.0


# ---------------------------------------------------------------------------------------
# argument checks (fake, never-dereferenced pointers)
# ---------------------------------------------------------------------------------------
FAKE = 0x7f0000001000


def _t(ptr=FAKE, dtype=B.TARA_BF16, shape=(1, 2, 300, 128)):
    t = B.TaraTensor()
    t.ptr, t.dtype = ptr, dtype
    t.B, t.H, t.N, t.D = shape
    return t


def _meta(N=300, stride=0, ptr=FAKE, extra=None, extra_stride=0):
    m = B.TaraTokenMeta()
    m.seg = m.pic = ptr
    m.time_s = m.m = ptr
    m.N, m.batch_stride = N, stride
    m.extra_m, m.extra_m_stride = extra, extra_stride
    return m


def _call(lib, Q=None, K=None, V=None, meta=None, p=None, O=None, lse=FAKE):
    Q, K, V, O = (x if x is not None else _t() for x in (Q, K, V, O))
    meta = meta if meta is not None else _meta()
    p = p if p is not None else B.make_params()
    return lib.tara_attn_forward(ctypes.byref(Q), ctypes.byref(K), ctypes.byref(V),
                                 ctypes.byref(meta), ctypes.byref(p), ctypes.byref(O),
                                 ctypes.c_void_p(lse), None)


def _call_noalloc(lib, Q, meta, p=None):
    p = p if p is not None else B.make_params()
    return lib.tara_attn_forward_noalloc(ctypes.byref(Q), ctypes.byref(Q), ctypes.byref(Q),
                                         ctypes.byref(meta), ctypes.byref(p), ctypes.byref(Q),
                                         ctypes.c_void_p(FAKE), None)


def _noalloc_scratch(nsets, N):
    """Bytes of scratch the allocation-free entry point needs: per metadata set and 128-token
    tile, in ascending and in descending tile order, a 32-byte tile record and 128 16-byte key
    records; each of the two arrays rounded to 256 bytes."""
    up = lambda x: (x + 255) // 256 * 256
    ntiles = (N + 127) // 128
    return up(2 * nsets * ntiles * 32) + up(2 * nsets * ntiles * 128 * 16)


def _noalloc_max_tokens(nsets):
    cap = B.TARA_NOALLOC_SCRATCH_BYTES
    N = cap // (32 * nsets) + 128
    while _noalloc_scratch(nsets, N) > cap:
        N -= 1
    return N


@pytest.mark.parametrize("nsets", [1, 3])
def test_noalloc_rejects_sizes_above_its_scratch(lib, nsets):
    # one token more than the fixed array holds is refused before any CUDA call
    header = open(os.path.join(ROOT, "include", "tara_attn.h")).read()
    assert "#define TARA_NOALLOC_SCRATCH_BYTES (8u << 20)" in header
    assert B.TARA_NOALLOC_SCRATCH_BYTES == 8 << 20
    n_fit = _noalloc_max_tokens(nsets)
    n = n_fit + 1
    assert _noalloc_scratch(nsets, n) > B.TARA_NOALLOC_SCRATCH_BYTES
    Q = _t(shape=(nsets, 2, n, 128))
    m = _meta(N=n, stride=0 if nsets == 1 else n)
    assert _call_noalloc(lib, Q, m) == -11   # TARA_ERR_TOO_LARGE
    # its other refusals: fp32 inputs (no scratch needed) and 8-bit Q/K
    assert _call_noalloc(lib, _t(dtype=B.TARA_FP32), _meta()) == -3
    p = B.make_params()
    p.qk_int8 = 1
    assert _call_noalloc(lib, _t(), _meta(), p) == -5


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="a size that fits would launch on the fake pointers")
@pytest.mark.parametrize("nsets", [1, 3])
def test_noalloc_accepts_the_largest_size_that_fits(lib, nsets):
    # the largest size passes the size check and stops at the first CUDA call (no device
    # here), so the fake pointers are never used
    n_fit = _noalloc_max_tokens(nsets)
    Q = _t(shape=(nsets, 2, n_fit, 128))
    m = _meta(N=n_fit, stride=0 if nsets == 1 else n_fit)
    assert _call_noalloc(lib, Q, m) == -9   # TARA_ERR_CUDA


def test_rejects_null(lib):
    assert lib.tara_attn_forward(None, None, None, None, None, None, None, None) == -1
    assert _call(lib, Q=_t(ptr=0)) == -1
    assert _call(lib, lse=0) == -1
    assert _call(lib, meta=_meta(ptr=0)) == -1


def test_rejects_dtype(lib):
    assert _call(lib, K=_t(dtype=B.TARA_FP16)) == -3
    assert _call(lib, O=_t(dtype=B.TARA_FP32)) == -3
    assert _call(lib, Q=_t(dtype=7), K=_t(dtype=7), V=_t(dtype=7), O=_t(dtype=7)) == -3


def test_rejects_shape(lib):
    assert _call(lib, K=_t(shape=(1, 2, 299, 128))) == -2
    assert _call(lib, V=_t(shape=(1, 3, 300, 128))) == -2
    assert _call(lib, O=_t(shape=(2, 2, 300, 128))) == -2
    assert _call(lib, meta=_meta(N=301)) == -2
    assert _call(lib, meta=_meta(stride=10)) == -2
    assert _call(lib, meta=_meta(stride=-1)) == -2
    z = (1, 2, 0, 128)
    assert _call(lib, Q=_t(shape=z), K=_t(shape=z), V=_t(shape=z), O=_t(shape=z),
                 meta=_meta(N=0)) == -2


def test_rejects_more_work_items_than_an_int_holds(lib):
    # 46,340 x 46,340 planes fit the plane count, but with 1,024 tokens each (eight 128-token
    # query tiles, two work items of four) the 4.3e9 work items do not fit an int
    Q = _t(shape=(46340, 46340, 1024, 128))
    assert _call(lib, Q=Q, K=Q, V=Q, O=Q, meta=_meta(N=1024)) == -11


def test_rejects_head_dim(lib):
    for d in (32, 96, 256):
        s = (1, 2, 300, d)
        assert _call(lib, Q=_t(shape=s), K=_t(shape=s), V=_t(shape=s), O=_t(shape=s)) == -4
    s = (1, 2, 300, 257)
    f = B.TARA_FP32
    assert _call(lib, Q=_t(dtype=f, shape=s), K=_t(dtype=f, shape=s), V=_t(dtype=f, shape=s),
                 O=_t(dtype=f, shape=s)) == -4


def test_rejects_misalignment(lib):
    assert _call(lib, V=_t(ptr=FAKE + 8)) == -6
    assert _call(lib, lse=FAKE + 2) == -6


@pytest.mark.parametrize("kw", [
    dict(falloff=0.0), dict(falloff=-1.0), dict(window=-0.1), dict(strength=-2.0),
    dict(cap=-1.0), dict(cap=float("inf")), dict(window=float("nan")),
    dict(gain=(0.0,) + (1.0,) * 8), dict(gain=(1.0,) * 8 + (-1.0,)),
    dict(gain=(float("inf"),) + (1.0,) * 8), dict(softmax_scale=-1.0),
])
def test_rejects_parameters(lib, kw):
    assert _call(lib, p=B.make_params(**kw)) == -5


def test_default_params_have_no_extra_bindings(lib):
    p = B.default_params()
    assert p.n_extra_bindings == 0
    assert all(p.extra_gain[k][i] == 1.0 for k in range(B.MAX_EXTRA_BINDINGS) for i in range(9))


def _extra_params(n, bad=None):
    p = B.make_params()
    p.n_extra_bindings = n
    for k in range(B.MAX_EXTRA_BINDINGS):
        for i in range(9):
            p.extra_gain[k][i] = 1.0
    if bad is not None:
        p.extra_gain[min(n, B.MAX_EXTRA_BINDINGS) - 1][4] = bad
    return p


def test_extra_binding_checks(lib):
    ok_meta = _meta(extra=FAKE, extra_stride=300)
    for n in (-1, 4, 1000):
        assert _call(lib, meta=ok_meta, p=_extra_params(n)) == -5
    for bad in (0.0, -2.0, float("inf"), float("nan")):
        assert _call(lib, meta=ok_meta, p=_extra_params(2, bad)) == -5
    assert _call(lib, meta=_meta(extra=None, extra_stride=300), p=_extra_params(1)) == -1
    assert _call(lib, meta=_meta(extra=FAKE, extra_stride=299), p=_extra_params(1)) == -2
    # batch-strided metadata: each mask spans (B-1)*stride + N entries
    s2 = (2, 2, 300, 128)
    t2 = dict(Q=_t(shape=s2), K=_t(shape=s2), V=_t(shape=s2), O=_t(shape=s2))
    assert _call(lib, meta=_meta(stride=320, extra=FAKE, extra_stride=619),
                 p=_extra_params(1), **t2) == -2
    assert _call(lib, meta=_meta(extra=FAKE + 2, extra_stride=300), p=_extra_params(1)) == -6
    # gains of unused binding slots are not read
    p = _extra_params(1)
    p.extra_gain[2][0] = -1.0
    assert _call(lib, meta=_meta(extra=FAKE, extra_stride=300, ptr=0), p=p) == -1
    with pytest.raises(ValueError):
        B.make_params(extra_gain=((1.0,) * 9,) * 4)
    with pytest.raises(ValueError):
        B.make_params(extra_gain=((1.0,) * 8,))


def test_int8_qk_checks(lib):
    assert B.default_params().qk_int8 == 0
    for bad in (2, -1):
        assert _call(lib, p=B.make_params(qk_int8=bad)) == -5
    f, s64 = B.TARA_FP32, (1, 2, 300, 64)
    assert _call(lib, Q=_t(dtype=f), K=_t(dtype=f), V=_t(dtype=f), O=_t(dtype=f),
                 p=B.make_params(qk_int8=1)) == -3
    assert _call(lib, Q=_t(shape=s64), K=_t(shape=s64), V=_t(shape=s64), O=_t(shape=s64),
                 p=B.make_params(qk_int8=1)) == -4
    p = B.make_params(qk_int8=1)
    rc = lib.tara_attn_forward_noalloc(ctypes.byref(_t()), ctypes.byref(_t()), ctypes.byref(_t()),
                                       ctypes.byref(_meta()), ctypes.byref(p), ctypes.byref(_t()),
                                       ctypes.c_void_p(FAKE), None)
    assert rc == -5


def _quant_call(lib, Q=None, K=None, qc=FAKE, qs=FAKE, kc=FAKE, ks=FAKE):
    Q = Q if Q is not None else _t()
    K = K if K is not None else _t()
    return lib.tara_quantize_qk_int8(ctypes.byref(Q), ctypes.byref(K), ctypes.c_void_p(qc),
                                     ctypes.c_void_p(qs), ctypes.c_void_p(kc),
                                     ctypes.c_void_p(ks), None)


def test_quantize_argument_checks(lib):
    assert _quant_call(lib, qc=0) == -1
    assert _quant_call(lib, ks=0) == -1
    assert _quant_call(lib, Q=_t(ptr=0)) == -1
    assert _quant_call(lib, Q=_t(dtype=B.TARA_FP32), K=_t(dtype=B.TARA_FP32)) == -3
    assert _quant_call(lib, K=_t(dtype=B.TARA_FP16)) == -3
    assert _quant_call(lib, K=_t(shape=(1, 2, 301, 128))) == -2
    assert _quant_call(lib, Q=_t(shape=(1, 2, 0, 128)), K=_t(shape=(1, 2, 0, 128))) == -2
    s96 = (1, 2, 300, 96)
    assert _quant_call(lib, Q=_t(shape=s96), K=_t(shape=s96)) == -4
    big = (300, 300, 4, 128)
    assert _quant_call(lib, Q=_t(shape=big), K=_t(shape=big)) == -11
    assert _quant_call(lib, kc=FAKE + 8) == -6
    assert _quant_call(lib, qs=FAKE + 2) == -6
    assert _quant_call(lib, K=_t(ptr=FAKE + 4)) == -6


def test_host_forward_argument_checks(lib):
    def call(Q=None, K=None, V=None, meta=None, p=None, O=None, lse=FAKE):
        Q, K, V, O = (x if x is not None else _t() for x in (Q, K, V, O))
        meta = meta if meta is not None else _meta()
        p = p if p is not None else B.make_params()
        return lib.tara_attn_forward_host(ctypes.byref(Q), ctypes.byref(K), ctypes.byref(V),
                                          ctypes.byref(meta), ctypes.byref(p), ctypes.byref(O),
                                          ctypes.c_void_p(lse), None)
    assert lib.tara_attn_forward_host(None, None, None, None, None, None, None, None) == -1
    assert call(lse=0) == -1
    assert call(meta=_meta(ptr=0)) == -1
    assert call(K=_t(dtype=B.TARA_FP16)) == -3
    assert call(V=_t(shape=(1, 2, 301, 128))) == -2
    assert call(meta=_meta(N=301)) == -2
    s96 = (1, 2, 300, 96)
    assert call(Q=_t(shape=s96), K=_t(shape=s96), V=_t(shape=s96), O=_t(shape=s96)) == -4
    assert call(p=B.make_params(falloff=0.0)) == -5
    assert call(p=B.make_params(qk_int8=3)) == -5
    f = B.TARA_FP32
    assert call(Q=_t(dtype=f), K=_t(dtype=f), V=_t(dtype=f), O=_t(dtype=f),
                p=B.make_params(qk_int8=1)) == -3
    p1 = B.make_params(extra_gain=((1.5,) * 9,))
    assert call(p=p1, meta=_meta(extra=None, extra_stride=300)) == -1
    assert call(p=p1, meta=_meta(extra=FAKE, extra_stride=10)) == -2


# ---------------------------------------------------------------------------------------
# the packer against the oracle's packer (bit-exact) and its error handling
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("name", W.ORDER)
def test_packer_matches_oracle_bit_exact(lib, name):
    segs = W.get(name).segments
    a = B.pack_token_meta(segs)
    b = oracle.pack_token_meta(segs)
    assert B.packed_length(segs) == len(b["seg"])
    for key in ("seg", "time_s", "pic", "m"):
        np.testing.assert_array_equal(a[key].view(np.uint8), b[key].view(np.uint8))


def test_packer_mask_modes_and_offsets(lib):
    rng = np.random.Generator(np.random.PCG64(5))
    segs = [
        W.Segment(W.TARGET, 3, 7, t0_s=0.25, frame_dt_s=1 / 24, mask=rng.uniform(0, 1, 7).astype(np.float32)),
        W.Segment(W.TARGET, 3, 7, t0_s=-1.0, frame_dt_s=4 / 24, mask=rng.uniform(0, 1, 21).astype(np.float32)),
        W.Segment(W.TARGET, 2, 5),
        W.Segment(W.GUIDE, 4, 3, t0_s=1 / 24, frame_dt_s=4 / 24),
        W.Segment(W.PICTURE, 1, 4, pic=9),
        W.Segment(W.OTHER_VIDEO, 2, 2, frame_dt_s=0.5),
    ]
    a = B.pack_token_meta(segs)
    b = oracle.pack_token_meta(segs)
    for key in ("seg", "time_s", "pic", "m"):
        np.testing.assert_array_equal(a[key].view(np.uint8), b[key].view(np.uint8))


@pytest.mark.parametrize("bad", [
    W.Segment(9, 1, 4),
    W.Segment(W.TEXT, 0, 4),
    W.Segment(W.TEXT, 1, 0),
    W.Segment(W.PICTURE, 1, 4, pic=0),
    W.Segment(W.PICTURE, 1, 4, pic=10),
    W.Segment(W.TARGET, 2, 4, mask=np.ones(5, np.float32)),
    W.Segment(W.GUIDE, 2, 4, mask=np.ones(4, np.float32)),
    W.Segment(W.TARGET, 2, 4, t0_s=float("nan")),
])
def test_packer_rejects_bad_segments(lib, bad):
    with pytest.raises(B.TaraError) as e:
        B.pack_token_meta([W.Segment(W.TEXT, 1, 3), bad])
    assert e.value.code == -7


def test_packer_capacity_mismatch(lib):
    arr, keep = B._segments_to_c([W.Segment(W.TEXT, 1, 10)])
    buf = np.zeros(64, np.uint8)
    fb = np.zeros(64, np.float32)
    rc = lib.tara_pack_token_meta(arr, 1, buf.ctypes.data, fb.ctypes.data, buf.ctypes.data,
                                  fb.ctypes.data, 11)
    assert rc == -8
    assert lib.tara_pack_token_meta(arr, 1, None, None, None, None, 10) == -1


# ---------------------------------------------------------------------------------------
# target-mask preparation: argument checks (fake pointers, rejected before any launch)
# ---------------------------------------------------------------------------------------
def _mask_call(lib, F_in=107, Hp=8, Wp=8, L=107, tau=4, F_lat=26, Hq=4, Wq=4, ptr=FAKE, out=FAKE):
    return lib.tara_prepare_target_mask(ctypes.c_void_p(ptr), F_in, Hp, Wp, L, tau, F_lat, Hq,
                                        Wq, ctypes.c_void_p(out), None)


def test_mask_prep_argument_checks(lib):
    assert _mask_call(lib, ptr=0) == -1
    assert _mask_call(lib, out=0) == -1
    assert _mask_call(lib, Hp=0) == -2
    assert _mask_call(lib, tau=0) == -2
    assert _mask_call(lib, F_in=360) == -12          # whole-clip mask into a 107-frame shot
    assert _mask_call(lib, F_in=106) == -12
    assert _mask_call(lib, L=108, F_in=108) == -12   # not a 17n+5 shot
    assert _mask_call(lib, L=4, F_in=1) == -12
    assert _mask_call(lib, F_lat=28) == -2           # latent frame 27 starts past the shot
    assert _mask_call(lib, F_in=1, F_lat=70000) == -11
    assert _mask_call(lib, Wq=20000) == -11
    assert _mask_call(lib, ptr=FAKE + 2) == -6
