"""ctypes binding of libtara_attn.so (argument marshalling only).

Every step of the attention runs in the library's kernels; this module only turns torch
tensors and Python segment lists into the C structs of include/tara_attn.h.  There is no
fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libtara_attn.so")

TARA_BF16, TARA_FP16, TARA_FP32 = 0, 1, 2
# size of the fixed scratch array of tara_attn_forward_noalloc (the header's define)
TARA_NOALLOC_SCRATCH_BYTES = 8 << 20
SEG_TEXT, SEG_PICTURE, SEG_TARGET, SEG_GUIDE, SEG_AUDIO, SEG_OTHER_VIDEO = range(6)

STATUS = {
    0: "TARA_OK", -1: "TARA_ERR_NULL", -2: "TARA_ERR_SHAPE", -3: "TARA_ERR_DTYPE",
    -4: "TARA_ERR_HEAD_DIM", -5: "TARA_ERR_PARAM", -6: "TARA_ERR_ALIGN",
    -7: "TARA_ERR_SEGMENT", -8: "TARA_ERR_CAPACITY", -9: "TARA_ERR_CUDA",
    -10: "TARA_ERR_DEVICE_TIMEOUT", -11: "TARA_ERR_TOO_LARGE", -12: "TARA_ERR_MASK_LENGTH",
    -13: "TARA_ERR_DEBUG_CHECK",
}
EXPORTS = ("tara_default_params", "tara_status_string", "tara_attn_forward",
           "tara_device_status", "tara_packed_length", "tara_pack_token_meta",
           "tara_set_kernel_events", "tara_selftest_wait", "tara_attn_forward_noalloc",
           "tara_prepare_target_mask", "tara_quantize_qk_int8", "tara_attn_forward_host",
           "tara_debug_build")


class TaraError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s (%d)" % (what, STATUS.get(code, "?"), code))
        self.code = code


class TaraTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("dtype", ctypes.c_int), ("B", ctypes.c_int32),
                ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("D", ctypes.c_int32)]


MAX_EXTRA_BINDINGS = 3   # TARA_MAX_EXTRA_BINDINGS


class TaraTokenMeta(ctypes.Structure):
    _fields_ = [("seg", ctypes.c_void_p), ("time_s", ctypes.c_void_p),
                ("pic", ctypes.c_void_p), ("m", ctypes.c_void_p), ("N", ctypes.c_int32),
                ("batch_stride", ctypes.c_int64), ("extra_m", ctypes.c_void_p),
                ("extra_m_stride", ctypes.c_int64)]


class TaraParams(ctypes.Structure):
    _fields_ = [("window", ctypes.c_float), ("falloff", ctypes.c_float),
                ("strength", ctypes.c_float), ("cap", ctypes.c_float),
                ("gain", ctypes.c_float * 9), ("softmax_scale", ctypes.c_float),
                ("n_extra_bindings", ctypes.c_int32),
                ("extra_gain", (ctypes.c_float * 9) * MAX_EXTRA_BINDINGS),
                ("qk_int8", ctypes.c_int32)]


class TaraSegment(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("frames", ctypes.c_int32),
                ("tokens_per_frame", ctypes.c_int32), ("pic", ctypes.c_int32),
                ("t0_s", ctypes.c_double), ("frame_dt_s", ctypes.c_double),
                ("mask", ctypes.c_void_p), ("mask_len", ctypes.c_int64)]


_lib = None


def load_library(path: Optional[str] = None):
    """Load the library (once).  Raises OSError when it is missing: there is no fallback."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise OSError("libtara_attn.so not built (%s); run "
                      "`python -m video_diffusion_attention_b200.build`" % p)
    lib = ctypes.CDLL(p)
    lib.tara_default_params.restype = None
    lib.tara_default_params.argtypes = [ctypes.POINTER(TaraParams)]
    lib.tara_status_string.restype = ctypes.c_char_p
    lib.tara_status_string.argtypes = [ctypes.c_int]
    lib.tara_attn_forward.restype = ctypes.c_int
    lib.tara_attn_forward.argtypes = [ctypes.POINTER(TaraTensor)] * 3 + [
        ctypes.POINTER(TaraTokenMeta), ctypes.POINTER(TaraParams), ctypes.POINTER(TaraTensor),
        ctypes.c_void_p, ctypes.c_void_p]
    lib.tara_attn_forward_noalloc.restype = ctypes.c_int
    lib.tara_attn_forward_noalloc.argtypes = lib.tara_attn_forward.argtypes
    lib.tara_attn_forward_host.restype = ctypes.c_int
    lib.tara_attn_forward_host.argtypes = lib.tara_attn_forward.argtypes
    lib.tara_quantize_qk_int8.restype = ctypes.c_int
    lib.tara_quantize_qk_int8.argtypes = [ctypes.POINTER(TaraTensor)] * 2 + [ctypes.c_void_p] * 5
    lib.tara_set_kernel_events.restype = ctypes.c_int
    lib.tara_set_kernel_events.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.tara_prepare_target_mask.restype = ctypes.c_int
    lib.tara_prepare_target_mask.argtypes = [ctypes.c_void_p] + [ctypes.c_int32] * 8 + [
        ctypes.c_void_p, ctypes.c_void_p]
    lib.tara_selftest_wait.restype = ctypes.c_int
    lib.tara_selftest_wait.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    lib.tara_device_status.restype = ctypes.c_int
    lib.tara_device_status.argtypes = [ctypes.c_void_p]
    lib.tara_debug_build.restype = ctypes.c_int
    lib.tara_debug_build.argtypes = []
    lib.tara_packed_length.restype = ctypes.c_int64
    lib.tara_packed_length.argtypes = [ctypes.POINTER(TaraSegment), ctypes.c_int32]
    lib.tara_pack_token_meta.restype = ctypes.c_int
    lib.tara_pack_token_meta.argtypes = [ctypes.POINTER(TaraSegment), ctypes.c_int32] + [
        ctypes.c_void_p] * 4 + [ctypes.c_int32]
    if path is None:
        _lib = lib
    return lib


# ---------------------------------------------------------------------------------------
# parameters and packing
# ---------------------------------------------------------------------------------------
def make_params(window=0.20, falloff=0.25, strength=2.0, cap=6.0, gain=(1.0,) * 9,
                softmax_scale=0.0, extra_gain=(), qk_int8=0) -> TaraParams:
    """TaraParams; extra_gain lists the 9 gains of each chained binding beyond the first;
    qk_int8=1 selects 8-bit Q K^T."""
    p = TaraParams()
    p.window, p.falloff, p.strength, p.cap = window, falloff, strength, cap
    g = list(gain)
    if len(g) != 9:
        raise ValueError("gain needs 9 entries (Pictures 1..9)")
    for i in range(9):
        p.gain[i] = g[i]
    p.softmax_scale = softmax_scale
    extra = [list(row) for row in extra_gain]
    if len(extra) > MAX_EXTRA_BINDINGS or any(len(row) != 9 for row in extra):
        raise ValueError("extra_gain: at most %d bindings of 9 gains" % MAX_EXTRA_BINDINGS)
    p.n_extra_bindings = len(extra)
    for k in range(MAX_EXTRA_BINDINGS):
        for i in range(9):
            p.extra_gain[k][i] = extra[k][i] if k < len(extra) else 1.0
    p.qk_int8 = int(qk_int8)
    return p


def params_from(obj, qk_int8: int = 0) -> TaraParams:
    """TaraParams from any object with window, falloff, strength, cap, gain, softmax_scale
    (and optionally extra_gain)."""
    return make_params(obj.window, obj.falloff, obj.strength, obj.cap, obj.gain,
                       getattr(obj, "softmax_scale", 0.0), getattr(obj, "extra_gain", ()),
                       qk_int8)


def default_params() -> TaraParams:
    p = TaraParams()
    load_library().tara_default_params(ctypes.byref(p))
    return p


def _segments_to_c(segments):
    arr = (TaraSegment * max(1, len(segments)))()
    keep = []
    for i, s in enumerate(segments):
        c = arr[i]
        c.kind, c.frames, c.tokens_per_frame = int(s.kind), int(s.frames), int(s.tokens_per_frame)
        c.pic = int(getattr(s, "pic", 0))
        c.t0_s, c.frame_dt_s = float(getattr(s, "t0_s", 0.0)), float(getattr(s, "frame_dt_s", 0.0))
        mask = getattr(s, "mask", None)
        if mask is not None and len(mask) > 0:
            mk = np.ascontiguousarray(mask, dtype=np.float32)
            keep.append(mk)
            c.mask, c.mask_len = mk.ctypes.data, mk.size
        else:
            c.mask, c.mask_len = None, 0
    return arr, keep


def packed_length(segments) -> int:
    arr, _keep = _segments_to_c(segments)
    n = load_library().tara_packed_length(arr, len(segments))
    if n < 0:
        raise TaraError(int(n), "tara_packed_length")
    return int(n)


def pack_token_meta(segments):
    """Host packer: dict of numpy arrays seg (u8), time_s (f32), pic (u8), m (f32)."""
    lib = load_library()
    arr, _keep = _segments_to_c(segments)
    n = lib.tara_packed_length(arr, len(segments))
    if n < 0:
        raise TaraError(int(n), "tara_packed_length")
    out = {"seg": np.empty(n, np.uint8), "time_s": np.empty(n, np.float32),
           "pic": np.empty(n, np.uint8), "m": np.empty(n, np.float32)}
    rc = lib.tara_pack_token_meta(arr, len(segments), out["seg"].ctypes.data,
                                  out["time_s"].ctypes.data, out["pic"].ctypes.data,
                                  out["m"].ctypes.data, int(n))
    if rc != 0:
        raise TaraError(rc, "tara_pack_token_meta")
    return out


# ---------------------------------------------------------------------------------------
# device calls (torch tensors in, torch tensors out)
# ---------------------------------------------------------------------------------------
class DeviceMeta:
    """Per-token metadata resident on a device (the arrays of tara_token_meta).

    meta["m_extra"], when present, holds the masks of the extra chained bindings, one row of
    len(m) weights per binding."""

    def __init__(self, meta: dict, device, batch_stride: int = 0, N: Optional[int] = None):
        import torch
        self.seg = torch.as_tensor(np.ascontiguousarray(meta["seg"]), dtype=torch.uint8).to(device)
        self.time_s = torch.as_tensor(np.ascontiguousarray(meta["time_s"]),
                                      dtype=torch.float32).to(device)
        self.pic = torch.as_tensor(np.ascontiguousarray(meta["pic"]), dtype=torch.uint8).to(device)
        self.m = torch.as_tensor(np.ascontiguousarray(meta["m"]), dtype=torch.float32).to(device)
        self.extra_m = None
        if meta.get("m_extra") is not None and len(meta["m_extra"]) > 0:
            mx = np.ascontiguousarray(meta["m_extra"], dtype=np.float32).reshape(-1, self.m.numel())
            self.extra_m = torch.as_tensor(mx).to(device)
        self.batch_stride = int(batch_stride)
        self.N = int(self.seg.numel()) if N is None else int(N)

    def c_struct(self, N: Optional[int] = None) -> TaraTokenMeta:
        c = TaraTokenMeta()
        c.seg, c.time_s = self.seg.data_ptr(), self.time_s.data_ptr()
        c.pic, c.m = self.pic.data_ptr(), self.m.data_ptr()
        c.N = self.N if N is None else N
        c.batch_stride = self.batch_stride
        if self.extra_m is not None:
            c.extra_m, c.extra_m_stride = self.extra_m.data_ptr(), self.extra_m.shape[1]
        else:
            c.extra_m, c.extra_m_stride = None, 0
        return c


class HostMeta(DeviceMeta):
    """Per-token metadata in (pinned) host memory, for attn_forward_host."""

    def __init__(self, meta: dict, batch_stride: int = 0, N: Optional[int] = None,
                 pin: bool = True):
        import torch
        def host(a, dt):
            t = torch.as_tensor(np.ascontiguousarray(a), dtype=dt).contiguous()
            return t.pin_memory() if pin else t
        self.seg = host(meta["seg"], torch.uint8)
        self.time_s = host(meta["time_s"], torch.float32)
        self.pic = host(meta["pic"], torch.uint8)
        self.m = host(meta["m"], torch.float32)
        self.extra_m = None
        if meta.get("m_extra") is not None and len(meta["m_extra"]) > 0:
            self.extra_m = host(np.asarray(meta["m_extra"], np.float32).reshape(
                -1, self.m.numel()), torch.float32)
        self.batch_stride = int(batch_stride)
        self.N = int(self.seg.numel()) if N is None else int(N)


def _dtype_code(t) -> int:
    import torch
    return {torch.bfloat16: TARA_BF16, torch.float16: TARA_FP16, torch.float32: TARA_FP32}[t.dtype]


def tensor_struct(t) -> TaraTensor:
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError("tensors must be contiguous [B][H][N][D]")
    c = TaraTensor()
    c.ptr = t.data_ptr()
    c.dtype = _dtype_code(t)
    c.B, c.H, c.N, c.D = (int(x) for x in t.shape)
    return c


def attn_forward(q, k, v, meta: DeviceMeta, params: TaraParams, out=None, lse=None,
                 stream=None):
    """O, LSE = the TARA-biased attention forward of q, k, v ([B][H][N][D] CUDA tensors)."""
    import torch
    lib = load_library()
    B, H, N, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    cq, ck, cv, co = tensor_struct(q), tensor_struct(k), tensor_struct(v), tensor_struct(out)
    cm = meta.c_struct()
    rc = lib.tara_attn_forward(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv),
                               ctypes.byref(cm), ctypes.byref(params), ctypes.byref(co),
                               ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise TaraError(rc, "tara_attn_forward")
    return out, lse


def attn_forward_host(q, k, v, meta: "HostMeta", params: TaraParams, out=None, lse=None,
                      stream=None):
    """The forward on host tensors ([B][H][N][D] CPU tensors, pinned for overlap): copies,
    kernels and copies back run as a chunked three-stream pipeline inside the library.

    Asynchronous on `stream` (default: the current CUDA stream); synchronise it before reading
    `out` / `lse` or touching the inputs."""
    import torch
    lib = load_library()
    B, H, N, D = q.shape
    if out is None:
        out = torch.empty_like(q, pin_memory=True)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, pin_memory=True)
    if stream is None:
        stream = torch.cuda.current_stream()
    for t in (q, k, v, out, lse):
        if t.is_cuda:
            raise ValueError("attn_forward_host takes host tensors")
    cq, ck, cv, co = tensor_struct(q), tensor_struct(k), tensor_struct(v), tensor_struct(out)
    cm = meta.c_struct()
    rc = lib.tara_attn_forward_host(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv),
                                    ctypes.byref(cm), ctypes.byref(params), ctypes.byref(co),
                                    ctypes.c_void_p(lse.data_ptr()),
                                    ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise TaraError(rc, "tara_attn_forward_host")
    return out, lse


def set_kernel_events(start, stop) -> None:
    """Record torch.cuda.Event `start`/`stop` around the attention kernel of the next call.

    torch creates an event's handle on its first record(), so record both once beforehand."""
    if start is not None and (start.cuda_event == 0 or stop.cuda_event == 0):
        raise ValueError("record both events once before handing them to the library")
    rc = load_library().tara_set_kernel_events(
        ctypes.c_void_p(start.cuda_event if start is not None else 0),
        ctypes.c_void_p(stop.cuda_event if stop is not None else 0))
    if rc != 0:
        raise TaraError(rc, "tara_set_kernel_events")


def attn_forward_noalloc(q, k, v, meta: DeviceMeta, params: TaraParams, out, lse, stream=None):
    """The same forward through tara_attn_forward_noalloc: the library allocates nothing.

    `out` and `lse` must be provided by the caller (16-bit inputs only)."""
    import torch
    lib = load_library()
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    cq, ck, cv, co = tensor_struct(q), tensor_struct(k), tensor_struct(v), tensor_struct(out)
    cm = meta.c_struct()
    rc = lib.tara_attn_forward_noalloc(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv),
                                       ctypes.byref(cm), ctypes.byref(params), ctypes.byref(co),
                                       ctypes.c_void_p(lse.data_ptr()),
                                       ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise TaraError(rc, "tara_attn_forward_noalloc")
    return out, lse


def quantize_qk_int8(q, k, stream=None):
    """8-bit codes and scales of Q (per token) and K (per 128-token block), on the device:
    (q_codes int8 [B][H][N][D], q_scale f32 [B][H][N], k_codes int8 [B][H][N][D],
    k_scale f32 [B][H][ceil(N/128)])."""
    import torch
    B, H, N, D = q.shape
    qc = torch.empty((B, H, N, D), dtype=torch.int8, device=q.device)
    kc = torch.empty((B, H, N, D), dtype=torch.int8, device=q.device)
    qs = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    ks = torch.empty((B, H, (N + 127) // 128), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    cq, ck = tensor_struct(q), tensor_struct(k)
    rc = load_library().tara_quantize_qk_int8(
        ctypes.byref(cq), ctypes.byref(ck), ctypes.c_void_p(qc.data_ptr()),
        ctypes.c_void_p(qs.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
        ctypes.c_void_p(ks.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise TaraError(rc, "tara_quantize_qk_int8")
    return qc, qs, kc, ks


def prepare_target_mask(mask, shot_len: int, frames_per_latent: int, F_lat: int, Hq: int,
                        Wq: int, out=None, stream=None):
    """Per-target-token mask weights [F_lat][Hq][Wq] from a device pixel mask [F_in][Hp][Wp]
    (float32, contiguous), on the device (see include/tara_attn.h)."""
    import torch
    if mask.dim() != 3 or mask.dtype != torch.float32 or not mask.is_contiguous():
        raise ValueError("mask must be a contiguous float32 [F][H][W] tensor")
    F_in, Hp, Wp = (int(x) for x in mask.shape)
    if out is None:
        out = torch.empty((F_lat, Hq, Wq), dtype=torch.float32, device=mask.device)
    if stream is None:
        stream = torch.cuda.current_stream(mask.device)
    rc = load_library().tara_prepare_target_mask(
        ctypes.c_void_p(mask.data_ptr()), F_in, Hp, Wp, int(shot_len), int(frames_per_latent),
        int(F_lat), int(Hq), int(Wq), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise TaraError(rc, "tara_prepare_target_mask")
    return out


def selftest_wait(limit_us: int, arrive: bool, stream=None) -> None:
    """Launch the bounded-wait self-test kernel (see include/tara_attn.h)."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    rc = load_library().tara_selftest_wait(int(limit_us), 1 if arrive else 0,
                                          ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise TaraError(rc, "tara_selftest_wait")


def device_status(stream=None) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(load_library().tara_device_status(ctypes.c_void_p(stream.cuda_stream)))
