"""Oracle of the INT8 QK^T variant: symmetric 8-bit quantisation of Q and K, then the exact rule.

TEST INFRASTRUCTURE (same restrictions as the rest of `oracle/`).

"TARA: Native Temporal Alignment for MiniMax H3 References", section "Three backends": the
one-pass kernels fuse the rule into dense INT8 attention.  The page does not give the scaling
scheme; the reading taken here:

  - Q is quantised per token: each row of D values gets its own scale;
  - K is quantised per block of 128 consecutive tokens of one (branch, head): the block's
    128 x D values share one scale (the last block of a ragged sequence covers only its valid
    tokens);
  - symmetric, 8-bit signed codes in [-127, 127]:  amax = max |x| over the group,
        inv   = float32(127 / amax)          (IEEE float32 division)
        code  = rint(float32(x * inv))       (float32 product, ties to even)
        scale = float32(amax / 127)          (IEEE float32 division)
    a group with amax <= 1e-30 (all zeros, or values too small to matter) gets codes 0 and
    scale 0;
  - the quantised operand is code * scale; the logit is (Q_deq . K_deq) * softmax scale plus
    the rule's bias, and V stays in its 16-bit type (only QK^T is quantised);
  - every decision that yields an integer code is taken in float32, the precision the CUDA
    kernel takes it in, so the codes are comparable bit for bit.

The attention itself is the fp64 oracle (`oracle.attention_rows`) on the dequantised
operands, which are exact in fp64 (an 8-bit code times a float32 scale).
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

QMAX = np.float32(127.0)
KBLOCK = 128
AMAX_FLOOR = np.float32(1e-30)


def _widen_f32(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float32 values of raw bf16 (uint16 bit patterns), fp16 (uint16) or fp32 data."""
    if dtype == "bf16":
        return (raw.astype(np.uint32) << np.uint32(16)).view(np.float32)
    if dtype == "fp16":
        return raw.view(np.float16).astype(np.float32)
    if dtype == "fp32":
        return np.asarray(raw, dtype=np.float32)
    raise ValueError(dtype)


def _quantise_groups(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Symmetric int8 quantisation of each row of x ([G][n] float32): (codes [G][n], scales [G])."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], np.float32)
    live = amax > AMAX_FLOOR
    safe = np.where(live, amax, np.float32(1.0)).astype(np.float32)
    inv = (QMAX / safe).astype(np.float32)
    prod = (x * inv[:, None]).astype(np.float32)
    codes = np.rint(prod)
    codes = np.where(live[:, None], codes, np.float32(0.0))
    assert np.all(np.abs(codes) <= 127.0)
    scales = np.where(live, (amax / QMAX).astype(np.float32), np.float32(0.0)).astype(np.float32)
    return codes.astype(np.int8), scales


def quantise_q(q: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-token quantisation of Q [B][H][N][D] (float32): codes int8 [B][H][N][D], scales [B][H][N]."""
    B, H, N, D = q.shape
    codes, scales = _quantise_groups(q.reshape(B * H * N, D))
    return codes.reshape(B, H, N, D), scales.reshape(B, H, N)


def quantise_k(k: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-128-token-block quantisation of K [B][H][N][D]: codes int8 [B][H][N][D], scales
    [B][H][ceil(N/128)]."""
    B, H, N, D = k.shape
    nb = (N + KBLOCK - 1) // KBLOCK
    codes = np.empty((B, H, N, D), np.int8)
    scales = np.empty((B, H, nb), np.float32)
    for j in range(nb):
        lo, hi = j * KBLOCK, min(N, (j + 1) * KBLOCK)
        blk = k[:, :, lo:hi, :].reshape(B * H, (hi - lo) * D)
        c, s = _quantise_groups(blk)
        codes[:, :, lo:hi, :] = c.reshape(B, H, hi - lo, D)
        scales[:, :, j] = s.reshape(B, H)
    return codes, scales


def dequantise_q(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """code * scale per token, fp64 (exact)."""
    return codes.astype(np.float64) * scales.astype(np.float64)[..., None]


def dequantise_k(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """code * scale of each token's block, fp64 (exact)."""
    N = codes.shape[2]
    per_tok = np.repeat(scales.astype(np.float64), KBLOCK, axis=2)[:, :, :N]
    return codes.astype(np.float64) * per_tok[..., None]


def quantised_operands(q_raw, k_raw, v_raw, dtype: str):
    """Q_deq, K_deq (fp64, through the 8-bit codes) and V (fp64, exact) from raw inputs."""
    qf, kf = _widen_f32(q_raw, dtype), _widen_f32(k_raw, dtype)
    qd = dequantise_q(*quantise_q(qf))
    kd = dequantise_k(*quantise_k(kf))
    vd = _widen_f32(v_raw, dtype).astype(np.float64)
    return (np.ascontiguousarray(qd), np.ascontiguousarray(kd), np.ascontiguousarray(vd))


def attention_rows_int8qk(q_raw, k_raw, v_raw, dtype: str, meta, params, rows,
                          meta_batch_stride: int = 0, n_threads: int = 0):
    """O, LSE (fp64) of the INT8-QK^T variant for the requested rows (b, h, i)."""
    from . import attention_rows
    qd, kd, vd = quantised_operands(q_raw, k_raw, v_raw, dtype)
    return attention_rows(qd, kd, vd, "fp64", meta, params, rows,
                          meta_batch_stride=meta_batch_stride, n_threads=n_threads)
