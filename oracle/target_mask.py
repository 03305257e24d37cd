"""fp64 oracle of the target-mask preparation (TEST INFRASTRUCTURE, like the rest of oracle/).

"BFS H3 Reference Attention Binding (Experimental)":
  - "The exact rule": soft masks are area-downsampled to the target's patch resolution and
    averaged across the latent temporal spans;
  - "Inputs you'll set": no mask, one static mask, or one mask per prepared shot frame;
  - "Common issues": the mask must be one frame or exactly the prepared 17n+5 shot length
    (107 is such a length); any other length is an error.

Readings where the page is silent:
  - area downsampling is the exact area average: output cell (y, x) is the mean of the input
    over the rectangle [y*Hp/Hq, (y+1)*Hp/Hq) x [x*Wp/Wq, (x+1)*Wp/Wq) of the piecewise-
    constant input image (pixels straddling a cell boundary count by their overlap);
  - latent frame f spans the pixel frames [f*tau, min((f+1)*tau, L)) of the prepared shot of
    length L (tau = pixel frames per latent frame, 4 for a latent frame every 4/24 s); a one-
    frame mask applies unchanged to every latent frame.
"""
from __future__ import annotations

import numpy as np


def shot_length_ok(L: int) -> bool:
    """A prepared shot has 17n+5 frames, n >= 0."""
    return L >= 5 and (L - 5) % 17 == 0


def mask_length_ok(F_in: int, L: int) -> bool:
    return shot_length_ok(L) and (F_in == 1 or F_in == L)


def area_weights(n_in: int, n_out: int) -> np.ndarray:
    """[n_out][n_in] matrix: overlap of input cell [i, i+1) with output cell
    [o*n_in/n_out, (o+1)*n_in/n_out), divided by the output cell's length (rows sum to 1)."""
    W = np.zeros((n_out, n_in), dtype=np.float64)
    step = n_in / n_out
    for o in range(n_out):
        lo, hi = o * step, (o + 1) * step
        for i in range(int(np.floor(lo)), min(n_in, int(np.ceil(hi)))):
            ov = min(hi, i + 1) - max(lo, i)
            if ov > 0:
                W[o, i] = ov / step
    return W


def prepare_target_mask(mask: np.ndarray, L: int, F_lat: int, tau: int, Hq: int, Wq: int):
    """Per-target-token mask weights [F_lat][Hq][Wq] (fp64) from a pixel mask [F_in][Hp][Wp]."""
    mask = np.asarray(mask, dtype=np.float64)
    F_in, Hp, Wp = mask.shape
    if not mask_length_ok(F_in, L):
        raise ValueError("mask length %d does not match a %d-frame shot" % (F_in, L))
    if F_lat < 1 or tau < 1 or Hq < 1 or Wq < 1:
        raise ValueError("bad grid")
    if F_in > 1 and (F_lat - 1) * tau >= L:
        raise ValueError("latent frames exceed the shot")
    Wy = area_weights(Hp, Hq)
    Wx = area_weights(Wp, Wq)
    down = np.stack([Wy @ mask[t] @ Wx.T for t in range(F_in)])
    if F_in == 1:
        return np.repeat(down, F_lat, axis=0)
    out = np.empty((F_lat, Hq, Wq), dtype=np.float64)
    for f in range(F_lat):
        t0, t1 = f * tau, min((f + 1) * tau, L)
        out[f] = down[t0:t1].mean(axis=0)
    return out
