"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on one input."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as W

# Tolerances (max abs on O and LSE; mean abs on O for 16-bit inputs), measured against the
# oracle on the same 16-bit-rounded inputs.
TOL = {
    "fp32": dict(o_max=1e-5, o_mean=1e-5, lse_max=1e-5),
    "bf16": dict(o_max=1.5e-2, o_mean=2e-3, lse_max=5e-3),
    "fp16": dict(o_max=1.5e-2, o_mean=2e-3, lse_max=5e-3),
}


def _with_extra(meta: dict, m_extra, copies: int = 1) -> dict:
    if m_extra is not None:
        meta["m_extra"] = np.concatenate([np.asarray(m_extra, np.float32)] * copies, axis=1)
    return meta


def run_gpu(w: W.Workload, q, k, v, per_branch_meta: bool = False, m_extra=None,
            qk_int8: int = 0):
    """O, LSE from the CUDA path (through the C ABI) for workload w on cuda tensors q, k, v.

    m_extra: [n][N] masks of the chained bindings named by w.params.extra_gain (or None);
    qk_int8: 1 runs Q K^T on 8-bit codes."""
    import video_diffusion_attention_b200 as T
    meta = T.pack_token_meta(w.segments)
    if per_branch_meta:
        N = len(meta["seg"])
        stacked = {key: np.concatenate([val] * w.B) for key, val in meta.items()}
        dmeta = T.DeviceMeta(_with_extra(stacked, m_extra, w.B), q.device, batch_stride=N, N=N)
    else:
        dmeta = T.DeviceMeta(_with_extra(meta, m_extra), q.device)
    O, L = T.attn_forward(q, k, v, dmeta, T.params_from(w.params, qk_int8))
    torch.cuda.synchronize()
    assert T.device_status() == 0
    return O, L


def run_oracle(w: W.Workload, q, k, v, rows: np.ndarray, m_extra=None):
    """O, LSE (fp64) of the oracle on host copies of the same tensors, for rows (b, h, i)."""
    meta = _with_extra(oracle.pack_token_meta(w.segments), m_extra)
    raw = [oracle.torch_to_numpy_raw(t) for t in (q, k, v)]
    return oracle.attention_rows(raw[0][0], raw[1][0], raw[2][0], raw[0][1], meta, w.params,
                                 rows)


def run_oracle_int8(w: W.Workload, q, k, v, rows: np.ndarray, m_extra=None):
    """O, LSE (fp64) of the INT8-QK^T oracle for rows (b, h, i), one head at a time (the
    quantisation groups never span heads), in the order of `rows`."""
    from oracle import int8_qk
    meta = _with_extra(oracle.pack_token_meta(w.segments), m_extra)
    raw = [oracle.torch_to_numpy_raw(t) for t in (q, k, v)]
    dtype = raw[0][1]
    O = np.empty((rows.shape[0], w.D))
    L = np.empty((rows.shape[0],))
    for h in np.unique(rows[:, 1]):
        sel = np.where(rows[:, 1] == h)[0]
        sub = [np.ascontiguousarray(r[0][:, h:h + 1]) for r in raw]
        local = rows[sel].copy()
        local[:, 1] = 0
        O[sel], L[sel] = int8_qk.attention_rows_int8qk(sub[0], sub[1], sub[2], dtype, meta,
                                                       w.params, local)
    return O, L


def rows_from_sample(sample: dict) -> np.ndarray:
    out = []
    for (b, h), idx in sorted(sample.items()):
        out.append(np.stack([np.full_like(idx, b), np.full_like(idx, h), idx], axis=1))
    return np.concatenate(out).astype(np.int64)


def compare(w: W.Workload, O_gpu, L_gpu, rows: np.ndarray, O_ref, L_ref, dtype: str):
    """Element-wise comparison of the sampled rows; returns a stats dict, asserts the bar."""
    b, h, i = (torch.from_numpy(rows[:, c]) for c in range(3))
    og = O_gpu.float().cpu()[b, h, i].double().numpy()
    lg = L_gpu.cpu()[b, h, i].double().numpy()
    assert np.all(np.isfinite(og)) and np.all(np.isfinite(lg))
    d_o = np.abs(og - O_ref)
    d_l = np.abs(lg - L_ref)
    stats = dict(o_max=float(d_o.max()), o_mean=float(d_o.mean()), lse_max=float(d_l.max()),
                 rows=int(rows.shape[0]))
    tol = TOL[dtype]
    assert stats["o_max"] <= tol["o_max"], stats
    assert stats["o_mean"] <= tol["o_mean"], stats
    assert stats["lse_max"] <= tol["lse_max"], stats
    return stats
