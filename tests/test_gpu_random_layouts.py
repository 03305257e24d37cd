"""Seeded random shots through the CUDA path vs the oracle (needs a B200).

Each seed draws a segment list (roles in any order, ragged frame sizes, static or per-frame
masks), rule parameters, gains, chained bindings, dtype, head dim, branch count, shared or
per-branch metadata and, for 16-bit D=128, the INT8 QK^T variant; every output row is compared
with the oracle at the dtype's bar.  Q and K are drawn with scales up to 1.5, the peakiest
softmax of the pages' workloads: the bf16 bar is stated for those (at a scale near 2 a single
dominant key can put the bf16 rounding of P at the 1.5e-2 edge of O).
"""
import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import compare, run_gpu, run_oracle, run_oracle_int8

pytestmark = pytest.mark.gpu

DEV = "cuda"
KINDS = [W.TEXT, W.PICTURE, W.TARGET, W.GUIDE, W.AUDIO, W.OTHER_VIDEO]


def _draw(seed):
    g = np.random.Generator(np.random.PCG64(1000 + seed))
    segs = []
    for _ in range(int(g.integers(3, 9))):
        kind = KINDS[int(g.integers(0, len(KINDS)))]
        frames, tpf = int(g.integers(1, 7)), int(g.integers(1, 90))
        mask = None
        if kind == W.TARGET and g.random() < 0.6:
            n = tpf if g.random() < 0.5 else frames * tpf
            mask = g.uniform(0, 1, n).astype(np.float32)
        segs.append(W.Segment(kind, frames, tpf, pic=int(g.integers(1, 10)) if kind == W.PICTURE else 0,
                              t0_s=float(g.uniform(0, 1.5)), frame_dt_s=float(g.choice([1 / 24, 4 / 24, 0.3])),
                              mask=mask))
    if not any(s.kind == W.TARGET for s in segs):
        segs.append(W.Segment(W.TARGET, 3, 40, frame_dt_s=4 / 24))
    if not any(s.kind == W.GUIDE for s in segs):
        segs.insert(0, W.Segment(W.GUIDE, 3, 40, frame_dt_s=4 / 24))
    n_extra = int(g.integers(0, 3))
    params = W.Params(window=float(g.uniform(0, 0.5)), falloff=float(g.uniform(0.05, 1.0)),
                      strength=float(g.uniform(0, 5)), cap=float(g.uniform(0, 10)),
                      gain=tuple(float(x) for x in g.uniform(0.3, 3.0, 9)),
                      extra_gain=tuple(tuple(float(x) for x in g.uniform(0.3, 3.0, 9))
                                       for _ in range(n_extra)))
    dtype = str(g.choice(["bf16", "fp16", "fp32"]))
    D = int(g.choice([64, 128])) if dtype != "fp32" else int(g.choice([32, 64, 96, 128]))
    B, H = int(g.integers(1, 3)), int(g.integers(1, 4))
    per_branch = B > 1 and g.random() < 0.5
    q8 = int(dtype != "fp32" and D == 128 and g.random() < 0.4)
    w = W.custom("rnd%d" % seed, B=B, H=H, D=D, dtype=dtype, segments=segs, params=params,
                 qk_scale=float(g.uniform(0.5, 1.5)), seed_index=1100 + seed)
    return w, n_extra, per_branch, q8


@pytest.mark.parametrize("seed", range(48))
def test_random_shot(seed):
    w, n_extra, per_branch, q8 = _draw(seed)
    q, k, v = (t.to(DEV) for t in W.make_qkv(w, DEV))
    mx = W.chained_masks(w, n_extra) if n_extra else None
    O, L = run_gpu(w, q, k, v, per_branch_meta=per_branch, m_extra=mx, qk_int8=q8)
    rows = oracle.all_rows(w.B, w.H, w.N)
    ref = run_oracle_int8 if q8 else run_oracle
    Oref, Lref = ref(w, q, k, v, rows, m_extra=mx)
    compare(w, O, L, rows, Oref, Lref, w.dtype)
