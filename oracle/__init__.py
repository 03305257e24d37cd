"""fp64 CPU oracle of the TARA-biased joint attention forward pass.

TEST INFRASTRUCTURE.  Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline legs of
`bench.py` may import this package.  It shares no code with the CUDA path: its own token
packer, its own bias rule, its own attention (plain C in `tara_oracle.c`, fp64, one dense
logit row at a time, OpenMP over rows).

Sources, by page and section:
  - "TARA: Native Temporal Alignment for MiniMax H3 References", "The temporal rule":
    dt = |output time - guide time|, penalty = min(strength*(max(dt-window,0)/falloff)^2, cap),
    score = q.k/sqrt(head_dim) - penalty, for output-video queries x selected motion-video keys
    only; defaults window 0.20 s, falloff 0.25 s, strength 2.0, cap 6.0.
  - "BFS H3 Reference Attention Binding (Experimental)", "The exact rule": a target-video
    query with mask weight m and a key of Picture i gain m*log(gain_i) on the logit.
  - "BFS H3 Reference Attention Binding", "Common issues": chained bindings (one per subject)
    combine their log gains: binding k adds m_k * log(gain_k,i) for its own mask m_k.
  - "TARA: ...", "Three backends": the output is attention with its log-sum-exp.

Readings taken where the pages are silent:
  - per-token time is seconds on the shared, RoPE-aligned clock; a latent frame's tokens share
    one time; the time of frame f of a segment is t0 + f*frame_dt;
  - LSE is the natural-log log-sum-exp of the scaled, biased logits;
  - the bias is added after the 1/sqrt(d) scaling, never scaled itself;
  - a Picture index outside 1..9 is neutral; the mask weight of non-target tokens is unused
    and packed as 1.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Dict, Iterable, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tara_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")

TEXT, PICTURE, TARGET, GUIDE, AUDIO, OTHER_VIDEO = 0, 1, 2, 3, 4, 5
_DTYPE_CODE = {"bf16": 0, "fp16": 1, "fp32": 2, "fp64": 3}


def build(force: bool = False) -> str:
    """Compile tara_oracle.c into _build/liboracle.so with gcc (plain -O2, OpenMP)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _bind(lib):
    """Declare the C signatures on a loaded oracle library (the built one, or a test's copy)."""
    lib.oracle_attention_rows.restype = ctypes.c_int
    lib.oracle_attention_rows.argtypes = (
        [ctypes.c_void_p] * 3 + [ctypes.c_int] + [ctypes.c_int64] * 4 +
        [ctypes.c_void_p] * 4 + [ctypes.c_int64] + [ctypes.c_double] * 4 +
        [ctypes.c_void_p, ctypes.c_double, ctypes.c_void_p, ctypes.c_int64,
         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
         ctypes.c_void_p, ctypes.c_int64])
    lib.oracle_penalty.restype = ctypes.c_double
    lib.oracle_penalty.argtypes = [ctypes.c_double] * 5
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_logit_row.restype = ctypes.c_int
    lib.oracle_logit_row.argtypes = (
        [ctypes.c_void_p] * 2 + [ctypes.c_int] + [ctypes.c_int64] * 4 +
        [ctypes.c_void_p] * 4 + [ctypes.c_int64] + [ctypes.c_double] * 4 +
        [ctypes.c_void_p, ctypes.c_double] + [ctypes.c_int64] * 3 + [ctypes.c_void_p] +
        [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64])
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


# ---------------------------------------------------------------------------------------
# token packing (own implementation of the packed-sequence convention)
# ---------------------------------------------------------------------------------------
def pack_token_meta(segments) -> Dict[str, np.ndarray]:
    """Per-token role, time (s), Picture index and mask weight of a packed sequence.

    `segments` are objects with kind, frames, tokens_per_frame, pic, t0_s, frame_dt_s, mask.
    Token (f, p) of a segment: time = float32(t0 + f*frame_dt) evaluated in double; mask weight
    of a TARGET token = 1 without a mask, mask[p] for one static mask, mask[f*tpf+p] for one
    mask per frame ("BFS H3 Reference Attention Binding", "Inputs you'll set"); every other
    token packs m = 1.
    """
    seg, time_s, pic, m = [], [], [], []
    for s in segments:
        F, T = int(s.frames), int(s.tokens_per_frame)
        mask = None if s.mask is None else np.asarray(s.mask, dtype=np.float32).reshape(-1)
        for f in range(F):
            t = np.float32(float(s.t0_s) + f * float(s.frame_dt_s))
            for p in range(T):
                seg.append(s.kind)
                time_s.append(t)
                pic.append(s.pic if s.kind == PICTURE else 0)
                if s.kind == TARGET and mask is not None and len(mask) > 0:
                    m.append(mask[p] if len(mask) == T else mask[f * T + p])
                else:
                    m.append(np.float32(1.0))
    return {"seg": np.array(seg, dtype=np.uint8), "time_s": np.array(time_s, dtype=np.float32),
            "pic": np.array(pic, dtype=np.uint8), "m": np.array(m, dtype=np.float32)}


# ---------------------------------------------------------------------------------------
# the rule
# ---------------------------------------------------------------------------------------
def penalty(dt, window=0.20, falloff=0.25, strength=2.0, cap=6.0):
    """Temporal penalty, fp64 (C implementation, called element by element)."""
    lib = _load()
    arr = np.asarray(dt, dtype=np.float64)
    out = np.array([lib.oracle_penalty(float(x), window, falloff, strength, cap)
                    for x in arr.reshape(-1)], dtype=np.float64)
    return out.reshape(arr.shape) if arr.shape else float(out[0])


def _as_float32(x) -> float:
    return float(np.float32(x))


def _extra(meta: Dict, params, cv):
    """(n, gains [n*9] float64, masks [n][m_len] float32, m_len) of the extra bindings."""
    gains = list(getattr(params, "extra_gain", ()) or ())
    n = len(gains)
    if n == 0:
        return 0, None, None, 0
    g = np.ascontiguousarray([[cv(x) for x in row] for row in gains], dtype=np.float64)
    assert g.shape == (n, 9)
    mm = np.ascontiguousarray(meta["m_extra"], dtype=np.float32).reshape(n, -1)
    return n, g, mm, mm.shape[1]


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, dtype: str, meta: Dict,
                   params, rows: np.ndarray, meta_batch_stride: int = 0,
                   n_threads: int = 0, params_as_float32: bool = True):
    """O and LSE (fp64) of the requested query rows.

    q, k, v : contiguous numpy arrays [B][H][N][D]; for bf16/fp16 pass the raw 16-bit patterns
              as uint16 (`dtype` says how to widen them), else float32 / float64.
    meta    : dict with seg, time_s, pic, m (length N, or B*stride when batch-strided).
    params  : object with window, falloff, strength, cap, gain (9), softmax_scale.
    rows    : int64 array [n][3] of (b, h, i).
    params_as_float32: widen the parameters from their float32 values, as the GPU sees them.
    Returns (O [n][D] float64, LSE [n] float64).
    """
    lib = _load()
    B, H, N, D = q.shape
    for t in (q, k, v):
        assert t.shape == (B, H, N, D) and t.flags["C_CONTIGUOUS"]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    seg = np.ascontiguousarray(meta["seg"], dtype=np.uint8)
    ts = np.ascontiguousarray(meta["time_s"], dtype=np.float32)
    pic = np.ascontiguousarray(meta["pic"], dtype=np.uint8)
    m = np.ascontiguousarray(meta["m"], dtype=np.float32)
    cv = _as_float32 if params_as_float32 else float
    gain = np.ascontiguousarray([cv(g) for g in params.gain], dtype=np.float64)
    assert gain.shape == (9,)
    scale = cv(params.softmax_scale) if params.softmax_scale else 0.0
    O = np.empty((n, D), dtype=np.float64)
    L = np.empty((n,), dtype=np.float64)
    ne, eg, em, mlen = _extra(meta, params, cv)
    rc = lib.oracle_attention_rows(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, _DTYPE_CODE[dtype], B, H, N, D,
        seg.ctypes.data, ts.ctypes.data, pic.ctypes.data, m.ctypes.data, int(meta_batch_stride),
        cv(params.window), cv(params.falloff), cv(params.strength), cv(params.cap),
        gain.ctypes.data, scale, rows.ctypes.data, n, O.ctypes.data, L.ctypes.data,
        int(n_threads), ne, None if eg is None else eg.ctypes.data,
        None if em is None else em.ctypes.data, mlen)
    if rc != 0:
        raise RuntimeError("oracle_attention_rows failed")
    return O, L


def logit_row(q, k, dtype: str, meta: Dict, params, b: int, h: int, i: int,
              meta_batch_stride: int = 0, params_as_float32: bool = True) -> np.ndarray:
    """The dense scaled, biased logit row of query (b, h, i): N float64 values."""
    lib = _load()
    B, H, N, D = q.shape
    cv = _as_float32 if params_as_float32 else float
    gain = np.ascontiguousarray([cv(g) for g in params.gain], dtype=np.float64)
    seg = np.ascontiguousarray(meta["seg"], dtype=np.uint8)
    ts = np.ascontiguousarray(meta["time_s"], dtype=np.float32)
    pic = np.ascontiguousarray(meta["pic"], dtype=np.uint8)
    m = np.ascontiguousarray(meta["m"], dtype=np.float32)
    out = np.empty((N,), dtype=np.float64)
    scale = cv(params.softmax_scale) if params.softmax_scale else 0.0
    ne, eg, em, mlen = _extra(meta, params, cv)
    rc = lib.oracle_logit_row(q.ctypes.data, k.ctypes.data, _DTYPE_CODE[dtype], B, H, N, D,
                              seg.ctypes.data, ts.ctypes.data, pic.ctypes.data, m.ctypes.data,
                              int(meta_batch_stride), cv(params.window), cv(params.falloff),
                              cv(params.strength), cv(params.cap), gain.ctypes.data, scale,
                              b, h, i, out.ctypes.data, ne, None if eg is None else eg.ctypes.data,
                              None if em is None else em.ctypes.data, mlen)
    if rc != 0:
        raise RuntimeError("oracle_logit_row failed")
    return out


from .target_mask import (  # noqa: E402,F401
    area_weights, mask_length_ok, prepare_target_mask, shot_length_ok)


def all_rows(B: int, H: int, N: int) -> np.ndarray:
    b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(N), indexing="ij")
    return np.stack([b.reshape(-1), h.reshape(-1), i.reshape(-1)], axis=1).astype(np.int64)


def torch_to_numpy_raw(t):
    """Host copy of a torch tensor in the layout `attention_rows` takes (16-bit as uint16)."""
    import torch
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16), (
            "bf16" if t.dtype == torch.bfloat16 else "fp16")
    if t.dtype == torch.float32:
        return t.numpy(), "fp32"
    if t.dtype == torch.float64:
        return t.numpy(), "fp64"
    raise TypeError(t.dtype)
