"""Seeded synthetic inputs shaped like the pages' workloads.

This module only describes and draws inputs: the packed shot layouts (which segments, how
many latent frames and patches, on which clock), the rule parameters each workload uses, the
random Q/K/V tensors and target masks, and the seeded row samples used for parity checks.  It
holds none of the attention or bias arithmetic; both the CUDA path and the oracle consume what
it returns, and neither is imported here.

Workloads (shapes from the pages' microbenchmark in "TARA: Native Temporal Alignment for
MiniMax H3 References", section "What the numbers say": 107,126 packed tokens, 8 heads, BF16;
H3's 56 heads; ragged guide and CFG branches as in the same section's RTX 5090 runs):

  tiny     B1 H2  D64  fp32  N=192      16 text | 32 Picture-1 | 4f x16 target | 4f x16 guide | 16 audio
  medium   B1 H8  D128 bf16  N=8,704    256 | 512 (Pic1) | 12f x320 | 12f x320 | 256
  micro    B1 H8  D128 bf16  N=107,126  512 | 2,048 (Pic1) | 26f x2,000 | 26f x2,000 | 566
  full     B1 H56 D128 bf16  N=107,126  512 | 1,024 (Pic1) | 1,024 (Pic2) | 26f x2,000 | 26f x2,000 | 566
  ragged   B2 H56 D128 bf16  N=67,112   512 | 2,048 (Pic1) | 26f x2,000 | 26f x461 (+1/24 s) | 566

Latent frame f of the target and guide videos sits at f*4/24 s on the shared 24 fps clock.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

# Token roles, as numbered in include/tara_attn.h (an interface both sides implement).
TEXT, PICTURE, TARGET, GUIDE, AUDIO, OTHER_VIDEO = 0, 1, 2, 3, 4, 5

LATENT_FRAME_DT = 4.0 / 24.0      # seconds per latent frame on the 24 fps clock
BASE_SEED = 20261023


@dataclasses.dataclass
class Segment:
    kind: int
    frames: int = 1
    tokens_per_frame: int = 1
    pic: int = 0
    t0_s: float = 0.0
    frame_dt_s: float = 0.0
    mask: Optional[np.ndarray] = None   # float32, length 0, tokens_per_frame or frames*tpf

    @property
    def length(self) -> int:
        return self.frames * self.tokens_per_frame


@dataclasses.dataclass
class Params:
    window: float = 0.20
    falloff: float = 0.25
    strength: float = 2.0
    cap: float = 6.0
    gain: tuple = (1.0,) * 9
    softmax_scale: float = 0.0          # 0: 1/sqrt(D)
    extra_gain: tuple = ()              # gains (9 each) of chained bindings beyond the first


@dataclasses.dataclass
class Workload:
    name: str
    index: int
    B: int
    H: int
    D: int
    dtype: str                          # "fp32" | "bf16" | "fp16"
    segments: List[Segment]
    params: Params
    qk_scale: float = 1.0               # Q and K drawn as qk_scale * N(0,1)
    branch_seeds: bool = False          # B branches drawn from independent seeds

    @property
    def N(self) -> int:
        return sum(s.length for s in self.segments)

    @property
    def flops(self) -> float:
        """Dense attention FLOPs of one forward call: 4*B*H*N*N*D."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.D

    def seed(self, stream: int, branch: int = 0) -> int:
        """Seed of one random stream (0 Q, 1 K, 2 V, 3 mask) of one branch."""
        return (BASE_SEED + self.index) * 16 + stream * 4 + (branch if self.branch_seeds else 0)


def _video(kind, frames, tpf, t0=0.0, mask=None) -> Segment:
    return Segment(kind=kind, frames=frames, tokens_per_frame=tpf, t0_s=t0,
                   frame_dt_s=LATENT_FRAME_DT, mask=mask)


def ellipse_mask(seed: int, rows: int = 40, cols: int = 50) -> np.ndarray:
    """Soft elliptic target mask on a rows x cols patch grid (row-major), values in (0,1).

    Centre uniform over the middle half of the grid, semi-axes U[8,16] x U[10,20] patches,
    a logistic edge of width 0.1 in normalised radius.  Drawn once; constant across frames.
    """
    g = np.random.Generator(np.random.PCG64(seed))
    cy = g.uniform(rows * 0.25, rows * 0.75)
    cx = g.uniform(cols * 0.25, cols * 0.75)
    ay = g.uniform(8.0, 16.0)
    ax = g.uniform(10.0, 20.0)
    y, x = np.meshgrid(np.arange(rows, dtype=np.float64), np.arange(cols, dtype=np.float64),
                       indexing="ij")
    r = np.sqrt(((y - cy) / ay) ** 2 + ((x - cx) / ax) ** 2)
    return (1.0 / (1.0 + np.exp((r - 1.0) / 0.1))).astype(np.float32).reshape(-1)


def pixel_ellipse_mask(seed: int, frames: int, height: int, width: int) -> np.ndarray:
    """Soft elliptic pixel mask [frames][height][width] (float32) whose centre drifts linearly
    across the frames (a tracked subject); same edge profile as `ellipse_mask`."""
    g = np.random.Generator(np.random.PCG64(seed))
    cy0, cy1 = g.uniform(height * 0.3, height * 0.7, size=2)
    cx0, cx1 = g.uniform(width * 0.3, width * 0.7, size=2)
    ay = g.uniform(0.2, 0.4) * height
    ax = g.uniform(0.2, 0.4) * width
    y = np.arange(height, dtype=np.float64)[:, None] + 0.5
    x = np.arange(width, dtype=np.float64)[None, :] + 0.5
    out = np.empty((frames, height, width), dtype=np.float32)
    for f in range(frames):
        a = f / max(1, frames - 1)
        cy, cx = cy0 + a * (cy1 - cy0), cx0 + a * (cx1 - cx0)
        r = np.sqrt(((y - cy) / ay) ** 2 + ((x - cx) / ax) ** 2)
        out[f] = (1.0 / (1.0 + np.exp((r - 1.0) / 0.1))).astype(np.float32)
    return out


def uniform_mask(seed: int, n: int) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(seed))
    return g.uniform(0.0, 1.0, size=n).astype(np.float32)


def _tiny() -> Workload:
    w = Workload("tiny", 0, B=1, H=2, D=64, dtype="fp32", segments=[], params=Params(
        gain=(1.25,) + (1.0,) * 8))
    w.segments = [
        Segment(TEXT, 1, 16),
        Segment(PICTURE, 1, 32, pic=1),
        _video(TARGET, 4, 16, mask=uniform_mask(w.seed(3), 64)),
        _video(GUIDE, 4, 16),
        Segment(AUDIO, 1, 16),
    ]
    return w


def _medium() -> Workload:
    return Workload("medium", 1, B=1, H=8, D=128, dtype="bf16", segments=[
        Segment(TEXT, 1, 256),
        Segment(PICTURE, 1, 512, pic=1),
        _video(TARGET, 12, 320),
        _video(GUIDE, 12, 320),
        Segment(AUDIO, 1, 256),
    ], params=Params())


def _micro() -> Workload:
    return Workload("micro", 2, B=1, H=8, D=128, dtype="bf16", segments=[
        Segment(TEXT, 1, 512),
        Segment(PICTURE, 1, 2048, pic=1),
        _video(TARGET, 26, 2000),
        _video(GUIDE, 26, 2000),
        Segment(AUDIO, 1, 566),
    ], params=Params())


def _full() -> Workload:
    w = Workload("full", 3, B=1, H=56, D=128, dtype="bf16", segments=[], params=Params(
        gain=(1.25,) + (0.75,) * 8), qk_scale=1.5)
    w.segments = [
        Segment(TEXT, 1, 512),
        Segment(PICTURE, 1, 1024, pic=1),
        Segment(PICTURE, 1, 1024, pic=2),
        _video(TARGET, 26, 2000, mask=ellipse_mask(w.seed(3))),
        _video(GUIDE, 26, 2000),
        Segment(AUDIO, 1, 566),
    ]
    return w


def _ragged() -> Workload:
    return Workload("ragged", 4, B=2, H=56, D=128, dtype="bf16", segments=[
        Segment(TEXT, 1, 512),
        Segment(PICTURE, 1, 2048, pic=1),
        _video(TARGET, 26, 2000),
        _video(GUIDE, 26, 461, t0=1.0 / 24.0),
        Segment(AUDIO, 1, 566),
    ], params=Params(window=0.10, falloff=0.40, strength=3.0, cap=8.0,
                     gain=(1.5,) + (1.0,) * 8), branch_seeds=True)


WORKLOADS = {f().name: f for f in (_tiny, _medium, _micro, _full, _ragged)}
ORDER = ["tiny", "medium", "micro", "full", "ragged"]


def get(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        name_or_index = ORDER[name_or_index]
    return WORKLOADS[name_or_index]()


def custom(name: str, B: int, H: int, D: int, dtype: str, segments: List[Segment],
           params: Optional[Params] = None, qk_scale: float = 1.0, seed_index: int = 100,
           branch_seeds: bool = False) -> Workload:
    """A workload outside the five named ones (edge cases, small shapes)."""
    return Workload(name, seed_index, B=B, H=H, D=D, dtype=dtype, segments=segments,
                    params=params or Params(), qk_scale=qk_scale, branch_seeds=branch_seeds)


def make_qkv(w: Workload, device="cpu"):
    """Draw Q, K, V as torch tensors [B][H][N][D] of the workload's dtype on `device`.

    Q and K ~ qk_scale * N(0,1), V ~ N(0,1), drawn in fp32 from one torch.Generator per
    stream (per branch when the workload draws branches independently), then rounded to the
    workload's dtype.  The same seed gives different numbers on CPU and CUDA generators, so
    callers that compare two implementations draw once and copy.
    """
    import torch
    tdt = {"fp32": torch.float32, "bf16": torch.bfloat16, "fp16": torch.float16}[w.dtype]
    out = []
    for stream in range(3):
        t = torch.empty((w.B, w.H, w.N, w.D), dtype=tdt, device=device)
        for b in range(w.B):
            g = torch.Generator(device=device)
            g.manual_seed(w.seed(stream, b) if w.branch_seeds else w.seed(stream) + 97 * b)
            for h in range(w.H):
                x = torch.randn((w.N, w.D), generator=g, dtype=torch.float32, device=device)
                if stream < 2 and w.qk_scale != 1.0:
                    x.mul_(w.qk_scale)
                t[b, h].copy_(x)
        out.append(t)
    return out


def chained_masks(w: Workload, n: int, seed: int = 11) -> np.ndarray:
    """[n][N] float32 masks of n extra chained bindings, in packing order.

    Each binding's mask is a soft ellipse over the target's patch grid (`ellipse_mask` when the
    frame is 40 x 50 patches, else uniform in [0,1]), the same on every frame; the bindings are
    drawn independently, so their masks overlap.  Tokens outside TARGET segments get uniform
    noise: the rule ignores them, and nonzero values there check that it does.
    """
    g = np.random.Generator(np.random.PCG64(w.seed(40 + seed)))
    out = np.empty((n, w.N), np.float32)
    for k in range(n):
        row, start = [], 0
        for s in w.segments:
            if s.kind == TARGET:
                if s.tokens_per_frame == 40 * 50:
                    frame = ellipse_mask(w.seed(50 + seed + k))
                else:
                    frame = uniform_mask(w.seed(60 + seed + k) + start, s.tokens_per_frame)
                row.append(np.tile(frame, s.frames))
            else:
                row.append(g.uniform(0.0, 1.0, size=s.length).astype(np.float32))
            start += s.length
        out[k] = np.concatenate(row)
    return out


def segment_bounds(w: Workload) -> List[tuple]:
    """(kind, start, end, frames, tokens_per_frame) of every segment, in packing order."""
    out, start = [], 0
    for s in w.segments:
        out.append((s.kind, start, start + s.length, s.frames, s.tokens_per_frame))
        start += s.length
    return out


def sample_rows(w: Workload, per_head: int = 256, seed_offset: int = 7) -> Dict[tuple, np.ndarray]:
    """Seeded, stratified query-row sample for every (b, h): at least `per_head` rows.

    Always includes the first and last row of every segment, the first and last row of every
    latent frame of the target video, and the final row; the rest is drawn uniformly without
    replacement, independently for every (b, h).
    """
    N = w.N
    fixed = {0, N - 1}
    for kind, a, e, frames, tpf in segment_bounds(w):
        fixed.update((a, e - 1))
        if kind == TARGET:
            for f in range(frames):
                fixed.update((a + f * tpf, a + (f + 1) * tpf - 1))
    fixed = np.array(sorted(fixed), dtype=np.int64)
    out = {}
    g = np.random.Generator(np.random.PCG64(w.seed(0) + seed_offset))
    for b in range(w.B):
        for h in range(w.H):
            need = max(0, per_head - len(fixed))
            if len(fixed) >= N:
                rows = np.arange(N, dtype=np.int64)
            else:
                pool = np.setdiff1d(np.arange(N, dtype=np.int64), fixed)
                extra = g.choice(pool, size=min(need, len(pool)), replace=False)
                rows = np.sort(np.concatenate([fixed, extra]))
            out[(b, h)] = rows
    return out
