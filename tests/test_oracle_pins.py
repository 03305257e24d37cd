"""Pins of the fp64 oracle to what the pages and the mathematics fix (CPU only).

Each test names the passage it rests on.  None of them re-types the oracle's own formula:
they check printed values, library routines (torch SDPA in fp64), invariants the pages state,
and an independent brute force in high precision.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W


# ---------------------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------------------
def tiny_case(seed=0, frames=6, tpf=3, D=16, H=2, B=1, frame_dt=0.125, guide_t0=0.0,
              params=None, mask=True, extra_other=True):
    """A small joint sequence with every role: text, 2 pictures, target, guide, audio, other."""
    rng = np.random.Generator(np.random.PCG64(1234 + seed))
    segs = [
        W.Segment(W.TEXT, 1, 3),
        W.Segment(W.PICTURE, 1, 4, pic=1),
        W.Segment(W.PICTURE, 1, 2, pic=2),
        W.Segment(W.TARGET, frames, tpf, frame_dt_s=frame_dt,
                  mask=rng.uniform(0, 1, frames * tpf).astype(np.float32) if mask else None),
        W.Segment(W.GUIDE, frames, tpf, t0_s=guide_t0, frame_dt_s=frame_dt),
        W.Segment(W.AUDIO, 1, 2),
    ]
    if extra_other:
        segs.append(W.Segment(W.OTHER_VIDEO, 2, 2, frame_dt_s=frame_dt))
    meta = oracle.pack_token_meta(segs)
    N = len(meta["seg"])
    q = rng.standard_normal((B, H, N, D))
    k = rng.standard_normal((B, H, N, D))
    v = rng.standard_normal((B, H, N, D))
    p = params or W.Params(gain=(1.25, 0.75) + (1.0,) * 7)
    return q, k, v, meta, p


def run_all(q, k, v, meta, p, dtype="fp64", **kw):
    B, H, N, D = q.shape
    O, L = oracle.attention_rows(q, k, v, dtype, meta, p, oracle.all_rows(B, H, N), **kw)
    return O.reshape(B, H, N, D), L.reshape(B, H, N)


def sdpa64(q, k, v, bias=None):
    """torch scaled_dot_product_attention in fp64 on CPU, plus its log-sum-exp."""
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    b = None if bias is None else torch.from_numpy(bias)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=b)
    s = qt @ kt.transpose(-1, -2) / math.sqrt(q.shape[-1])
    if b is not None:
        s = s + b
    lse = torch.logsumexp(s, dim=-1)
    return o.numpy(), lse.numpy()


# ---------------------------------------------------------------------------------------
# P1: the printed defaults and the printed cap point
# ---------------------------------------------------------------------------------------
def test_penalty_zero_inside_free_window(golden_rule):
    # "Inside the free window there is no penalty at all." ("The temporal rule")
    w, f, s, c = (golden_rule[k][0] for k in ("window", "falloff", "strength", "cap"))
    dts = np.linspace(0.0, w, 2001)
    assert np.all(oracle.penalty(dts, w, f, s, c) == 0.0)
    assert oracle.penalty(np.nextafter(w, 1.0), w, f, s, c) > 0.0
    assert oracle.penalty(w + 1e-3, w, f, s, c) > 0.0


def test_penalty_reaches_cap_at_printed_delay(golden_rule):
    # "With the defaults the local correction goes to zero at about 0.633 s": the penalty
    # stops changing (sits at the cap) from that delay on.
    w, f, s, c = (golden_rule[k][0] for k in ("window", "falloff", "strength", "cap"))
    t_star, tol = golden_rule["cap_reached_at_s"]
    lo, hi = w, 10.0
    for _ in range(200):          # bisection for the first delay with penalty == cap
        mid = 0.5 * (lo + hi)
        if oracle.penalty(mid, w, f, s, c) >= c:
            hi = mid
        else:
            lo = mid
    assert abs(hi - t_star) <= tol
    assert oracle.penalty(t_star - tol - 1e-3, w, f, s, c) < c
    grid = np.linspace(t_star + tol, 60.0, 500)
    assert np.all(oracle.penalty(grid, w, f, s, c) == c)
    # the local derivative is zero past the cap point and positive before it
    e = 1e-4
    assert oracle.penalty(t_star + 0.01 + e, w, f, s, c) - oracle.penalty(t_star + 0.01, w, f, s, c) == 0
    assert oracle.penalty(t_star - 0.01 + e, w, f, s, c) - oracle.penalty(t_star - 0.01, w, f, s, c) > 0


def test_penalty_grows_quadratically_then_caps(golden_rule):
    # "Outside it the penalty grows quadratically until it reaches the cap, so distant guide
    # frames stay available at a small weight instead of being masked out."
    w, f, s, c = (golden_rule[k][0] for k in ("window", "falloff", "strength", "cap"))
    for x in (0.01, 0.03, 0.05, 0.1):
        p1 = oracle.penalty(w + x, w, f, s, c)
        p2 = oracle.penalty(w + 2 * x, w, f, s, c)
        p3 = oracle.penalty(w + 3 * x, w, f, s, c)
        assert p2 < c
        assert p2 / p1 == pytest.approx(4.0, rel=1e-12)
        if p3 < c:
            assert p3 / p1 == pytest.approx(9.0, rel=1e-12)
    dts = np.linspace(0, 5, 5001)
    pen = oracle.penalty(dts, w, f, s, c)
    assert np.all(np.diff(pen) >= 0.0)
    assert np.all(np.isfinite(pen)) and pen.max() == c
    # strength scales the quadratic part linearly; the cap bounds it
    assert oracle.penalty(w + 0.05, w, f, 2 * s, c) == pytest.approx(
        2 * oracle.penalty(w + 0.05, w, f, s, c), rel=1e-12)


def test_penalty_on_default_latent_grid(golden_rule):
    # P1: the rule at its printed defaults on the 4/24 s latent clock, against the exact
    # rational values derived by hand in the golden file ("The temporal rule")
    w, f, s, c = (golden_rule[k][0] for k in ("window", "falloff", "strength", "cap"))
    for d in range(5):
        val, tol = golden_rule["penalty_default_d%d" % d]
        assert abs(oracle.penalty(d / 6.0, w, f, s, c) - val) <= tol, d


def _ragged_rule(golden_rule):
    return tuple(golden_rule["ragged_" + k][0] for k in ("window", "falloff", "strength", "cap"))


def test_penalty_at_non_default_parameters(golden_rule):
    # P2: every parameter away from its default (the ragged workload's window 0.10, falloff
    # 0.40, strength 3.0, cap 8.0), with the guide clock offset by 1/24 s; exact values
    # derived by hand in the golden file.  A rule that ignores any one of the four
    # parameters in favour of its default misses several of them.
    w, f, s, c = _ragged_rule(golden_rule)
    for d in range(-4, 6):
        key = "penalty_ragged_d%s" % (("m%d" % -d) if d < 0 else str(d))
        val, tol = golden_rule[key]
        dt = abs(4 * d - 1) / 24.0
        assert abs(oracle.penalty(dt, w, f, s, c) - val) <= tol, d


def test_cap_point_at_non_default_parameters(golden_rule):
    # The first delay at which the penalty equals the cap: window + falloff*sqrt(cap/strength)
    # (inverting the quadratic branch of "The temporal rule").  Checked against the golden
    # value for the ragged parameters and, by bisection, for parameter sets where each of
    # the four moves on its own.
    w, f, s, c = _ragged_rule(golden_rule)
    sets = [(w, f, s, c, golden_rule["ragged_cap_reached_at_s"][0]),
            (0.05, 0.25, 2.0, 6.0, None), (0.20, 0.60, 2.0, 6.0, None),
            (0.20, 0.25, 5.0, 6.0, None), (0.20, 0.25, 2.0, 1.5, None)]
    for (ww, ff, ss, cc, printed) in sets:
        t_star = ww + ff * math.sqrt(cc / ss)
        if printed is not None:
            assert abs(t_star - printed) <= 1e-11
        lo, hi = ww, 100.0
        for _ in range(200):
            mid = 0.5 * (lo + hi)
            if oracle.penalty(mid, ww, ff, ss, cc) >= cc:
                hi = mid
            else:
                lo = mid
        assert abs(hi - t_star) <= 1e-12, (ww, ff, ss, cc)


def test_logit_row_at_non_default_parameters(golden_rule):
    # The oracle's dense logit row of one target query with Q = 0 (so every dot product is
    # 0): its guide entries are minus the ragged penalties above, its picture entries
    # m*ln(gain) ("BFS H3 Reference Attention Binding (Experimental)", "The exact rule") and
    # every other entry 0.  Times pass through the packer's float32 clock, which moves dt by
    # under 1e-7 s; the penalty's slope (< 30 per second here) bounds the effect.
    w, f, s, c = _ragged_rule(golden_rule)
    off = golden_rule["ragged_guide_offset_s"][0]
    segs = [W.Segment(W.TEXT, 1, 2), W.Segment(W.PICTURE, 1, 3, pic=1),
            W.Segment(W.TARGET, 10, 1, frame_dt_s=4 / 24,
                      mask=np.full(10, 0.625, dtype=np.float32)),
            W.Segment(W.GUIDE, 10, 1, t0_s=off, frame_dt_s=4 / 24), W.Segment(W.AUDIO, 1, 2)]
    meta = oracle.pack_token_meta(segs)
    N = len(meta["seg"])
    q = np.zeros((1, 1, N, 8))
    k = np.random.Generator(np.random.PCG64(5)).standard_normal((1, 1, N, 8))
    p = W.Params(window=w, falloff=f, strength=s, cap=c, gain=(1.5,) + (1.0,) * 8)
    t0 = 5                                  # the query: target frame 5
    row = oracle.logit_row(q, k, "fp64", meta, p, 0, 0, t0 + 5, params_as_float32=False)
    tgt = np.arange(5, 15)
    gde = np.arange(15, 25)
    for g, j in enumerate(gde):
        d = 5 - g
        key = "penalty_ragged_d%s" % (("m%d" % -d) if d < 0 else str(d))
        assert abs(row[j] + golden_rule[key][0]) <= 1e-6, d
    assert np.allclose(row[2:5], 0.625 * math.log(1.5), rtol=0, atol=1e-7)
    assert np.all(row[:2] == 0.0) and np.all(row[tgt] == 0.0) and np.all(row[25:] == 0.0)


# ---------------------------------------------------------------------------------------
# P3: strength 0 and neutral gains reduce to library attention (SDPA, fp64)
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("which", ["strength0", "cap0"])
def test_unbiased_equals_sdpa(which):
    # "setting strength to zero removes the bias" ("The temporal rule"); gain 1 is neutral
    # ("Inputs you'll set").  A zero cap removes the bias the same way.
    p = W.Params(strength=0.0) if which == "strength0" else W.Params(cap=0.0)
    q, k, v, meta, _ = tiny_case(seed=1, B=2)
    O, L = run_all(q, k, v, meta, p)
    Os, Ls = sdpa64(q, k, v)
    np.testing.assert_allclose(O, Os, atol=1e-12, rtol=0)
    np.testing.assert_allclose(L, Ls, atol=1e-12, rtol=0)


def test_softmax_scale_override_equals_sdpa():
    q, k, v, meta, _ = tiny_case(seed=2)
    p = W.Params(strength=0.0, softmax_scale=0.5)
    O, L = run_all(q, k, v, meta, p)
    D = q.shape[-1]
    Os, Ls = sdpa64(q * (0.5 * math.sqrt(D)), k, v)
    np.testing.assert_allclose(O, Os, atol=1e-12, rtol=0)
    np.testing.assert_allclose(L, Ls, atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------------------
# P4: the full biased case equals SDPA with the additive bias matrix
# ---------------------------------------------------------------------------------------
def test_biased_equals_sdpa_with_bias_matrix():
    # The bias matrix is assembled here from the scope rules of the two pages, with the
    # penalty values taken from the oracle's penalty routine (pinned above).
    q, k, v, meta, p = tiny_case(seed=3, frames=7, tpf=2, frame_dt=4 / 24)
    seg, t, pic, m = meta["seg"], meta["time_s"].astype(np.float64), meta["pic"], meta["m"]
    N = len(seg)
    bias = np.zeros((N, N))
    gains = [float(np.float32(g)) for g in p.gain]
    for i in range(N):
        if seg[i] != W.TARGET:
            continue
        for j in range(N):
            if seg[j] == W.GUIDE:
                bias[i, j] = -oracle.penalty(abs(t[i] - t[j]), float(np.float32(p.window)),
                                             float(np.float32(p.falloff)),
                                             float(np.float32(p.strength)),
                                             float(np.float32(p.cap)))
            elif seg[j] == W.PICTURE:
                bias[i, j] = float(m[i]) * math.log(gains[pic[j] - 1])
    assert (bias < -5.9).any() and (bias > 0).any() and (bias < 0).any()
    O, L = run_all(q, k, v, meta, p)
    Os, Ls = sdpa64(q, k, v, bias)
    np.testing.assert_allclose(O, Os, atol=1e-12, rtol=0)
    np.testing.assert_allclose(L, Ls, atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------------------
# P5 / scope: per-edge multipliers read through one-hot values
# ---------------------------------------------------------------------------------------
def _edge_weights(q, k, meta, p):
    """Unnormalised attention weights of every edge, read from the oracle with V = identity.

    With V[j] = e_j, O[i, j] is the softmax weight of edge (i, j); exp(LSE_i) * O[i, j] is the
    unnormalised weight exp(s_ij).
    """
    B, H, N, D = q.shape
    v = np.broadcast_to(np.eye(N), (B, H, N, N)).copy()
    qn = np.zeros((B, H, N, N)); qn[..., :D] = q
    kn = np.zeros((B, H, N, N)); kn[..., :D] = k
    p2 = W.Params(p.window, p.falloff, p.strength, p.cap, p.gain,
                  softmax_scale=1.0 / math.sqrt(D), extra_gain=p.extra_gain)
    O, L = run_all(qn, kn, v, meta, p2)
    return O * np.exp(L)[..., None]


def test_picture_edge_multiplied_by_gain_power_m():
    # "the unnormalized attention weight is multiplied by gain_i ** m, before the shared
    # softmax" ("The exact rule"); only target-video queries against image keys are touched.
    q, k, _, meta, p = tiny_case(seed=4)
    neutral = W.Params(p.window, p.falloff, p.strength, p.cap, (1.0,) * 9)
    Wg = _edge_weights(q, k, meta, p)
    W1 = _edge_weights(q, k, meta, neutral)
    ratio = Wg / W1
    seg, pic, m = meta["seg"], meta["pic"], meta["m"].astype(np.float64)
    gains = np.array([float(np.float32(g)) for g in p.gain])
    N = len(seg)
    for i in range(N):
        for j in range(N):
            if seg[i] == W.TARGET and seg[j] == W.PICTURE:
                expect = gains[pic[j] - 1] ** m[i]
            else:
                expect = 1.0
            assert ratio[0, 0, i, j] == pytest.approx(expect, rel=1e-12, abs=0), (i, j)


def test_temporal_edges_scope_and_sign(golden_rule):
    # Only edges from output-video queries to the selected motion video's keys change, and the
    # penalty is subtracted ("The temporal rule"); text, audio, other videos, pictures without
    # a gain and target self-attention keep their rule.
    q, k, _, meta, _ = tiny_case(seed=5, frames=7, tpf=2, frame_dt=4 / 24)
    p = W.Params()
    off = W.Params(strength=0.0)
    ratio = _edge_weights(q, k, meta, p) / _edge_weights(q, k, meta, off)
    seg, t = meta["seg"], meta["time_s"].astype(np.float64)
    c = golden_rule["cap"][0]
    N = len(seg)
    n_capped = 0
    for i in range(N):
        for j in range(N):
            r = ratio[0, 1, i, j]
            if seg[i] == W.TARGET and seg[j] == W.GUIDE:
                dt = abs(t[i] - t[j])
                assert r <= 1.0 + 1e-15          # a penalty never raises a weight
                if dt <= golden_rule["window"][0] + 1e-9:
                    assert r == pytest.approx(1.0, rel=1e-12)
                if dt >= golden_rule["cap_reached_at_s"][0] + 0.001:
                    assert r == pytest.approx(math.exp(-c), rel=1e-9)   # capped, not masked
                    n_capped += 1
            else:
                assert r == pytest.approx(1.0, rel=1e-12), (i, j)
    assert n_capped > 0          # the case exercises the cap (7 frames at 4/24 s)


# ---------------------------------------------------------------------------------------
# P6: key partitions merged by log-sum-exp reproduce the dense result
# ---------------------------------------------------------------------------------------
def test_partition_lse_merge_equals_dense():
    # The pages' backend evaluates the rule as attention-with-LSE over key partitions and
    # merges the contributions exactly ("Three backends"; "Common issues": "exact Flash
    # Partitions and LSE merging").  Merge the oracle's own logit rows by partitions
    # (zero-bias keys, capped keys, the rest; and a random split) and compare with its dense O.
    q, k, v, meta, p = tiny_case(seed=6, frames=7, tpf=2, frame_dt=4 / 24)
    B, H, N, D = q.shape
    O, L = run_all(q, k, v, meta, p)
    rng = np.random.Generator(np.random.PCG64(99))
    for i in range(N):
        s = oracle.logit_row(q, k, "fp64", meta, p, 0, 1, i)
        unb = oracle.logit_row(q, k, "fp64", meta, W.Params(strength=0.0), 0, 1, i)
        d = s - unb
        for parts in ([d == 0, (d != 0) & (d <= -5.999), (d != 0) & (d > -5.999)],
                      list(np.eye(3, dtype=bool)[rng.integers(0, 3, N)].T)):
            lses, outs = [], []
            for mask in parts:
                if not mask.any():
                    continue
                sp = s[mask]
                mx = sp.max()
                e = np.exp(sp - mx)
                lses.append(mx + math.log(e.sum()))
                outs.append((e[:, None] * v[0, 1][mask]).sum(0) / e.sum())
            lses = np.array(lses)
            lse = lses.max() + math.log(np.exp(lses - lses.max()).sum())
            o = sum(math.exp(l_ - lse) * o_ for l_, o_ in zip(lses, outs))
            assert lse == pytest.approx(L[0, 1, i], abs=1e-12)
            np.testing.assert_allclose(o, O[0, 1, i], atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------------------
# P7: brute force in 50-digit arithmetic on a tiny sequence
# ---------------------------------------------------------------------------------------
def test_brute_force_mpmath():
    mpmath = pytest.importorskip("mpmath")
    mpmath.mp.dps = 50
    q, k, v, meta, p = tiny_case(seed=7, frames=5, tpf=1, D=4, H=1, frame_dt=4 / 24,
                                 extra_other=False)
    B, H, N, D = q.shape
    O, L = run_all(q, k, v, meta, p)
    f32 = lambda x: mpmath.mpf(float(np.float32(x)))
    window, falloff, strength, cap = (f32(x) for x in (p.window, p.falloff, p.strength, p.cap))
    gains = [f32(g) for g in p.gain]
    seg, t, pic, m = meta["seg"], meta["time_s"], meta["pic"], meta["m"]
    for i in range(N):
        logits = []
        for j in range(N):
            dot = mpmath.fsum(mpmath.mpf(q[0, 0, i, c]) * mpmath.mpf(k[0, 0, j, c])
                              for c in range(D))
            x = dot / mpmath.sqrt(D)
            if seg[i] == W.TARGET and seg[j] == W.GUIDE:
                dt = abs(mpmath.mpf(float(t[i])) - mpmath.mpf(float(t[j])))
                over = max(dt - window, mpmath.mpf(0)) / falloff
                x -= min(strength * over * over, cap)
            if seg[i] == W.TARGET and seg[j] == W.PICTURE:
                x += mpmath.mpf(float(m[i])) * mpmath.log(gains[pic[j] - 1])
            logits.append(x)
        z = mpmath.fsum(mpmath.exp(x) for x in logits)
        assert float(mpmath.log(z)) == pytest.approx(L[0, 0, i], abs=1e-12)
        for c in range(D):
            oc = mpmath.fsum(mpmath.exp(x) * mpmath.mpf(v[0, 0, j, c])
                             for j, x in enumerate(logits)) / z
            assert float(oc) == pytest.approx(O[0, 0, i, c], abs=1e-12)


# ---------------------------------------------------------------------------------------
# P9: invariances the rule implies
# ---------------------------------------------------------------------------------------
def test_time_translation_invariance():
    # Only |output time - guide time| enters ("The temporal rule"): shifting both clocks by the
    # same amount changes nothing.  Times on a dyadic grid keep the shift exact in float32.
    base = dict(seed=8, frames=7, tpf=2, frame_dt=0.125)
    q, k, v, meta, p = tiny_case(**base)
    O1, L1 = run_all(q, k, v, meta, p)
    meta2 = dict(meta)
    ts = meta["time_s"].copy()
    sel = (meta["seg"] == W.TARGET) | (meta["seg"] == W.GUIDE)
    ts[sel] += np.float32(2.0)
    meta2["time_s"] = ts
    O2, L2 = run_all(q, k, v, meta2, p)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


def test_time_reflection_invariance():
    # dt is an absolute difference: reversing the guide clock around a target frame time is the
    # same as mirroring; check |a-b| symmetry by swapping target and guide times.
    q, k, v, meta, p = tiny_case(seed=9, frames=5, tpf=2, frame_dt=0.125, guide_t0=0.25)
    O1, L1 = run_all(q, k, v, meta, p)
    seg = meta["seg"]
    ts = meta["time_s"].copy()
    ts[seg == W.TARGET] *= -1
    ts[seg == W.GUIDE] *= -1
    meta2 = dict(meta, time_s=ts)
    O2, L2 = run_all(q, k, v, meta2, p)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


def test_stored_types_widen_exactly():
    # bf16 / fp16 / fp32 inputs are widened exactly: the oracle on 16-bit patterns equals the
    # oracle on the same values already widened to fp64.
    q, k, v, meta, p = tiny_case(seed=10)
    for name, tdt in (("bf16", torch.bfloat16), ("fp16", torch.float16), ("fp32", torch.float32)):
        ts = [torch.from_numpy(x).to(tdt) for x in (q, k, v)]
        raw = [oracle.torch_to_numpy_raw(t)[0] for t in ts]
        wide = [t.to(torch.float64).numpy() for t in ts]
        O1, L1 = run_all(*raw, meta, p, dtype=name)
        O2, L2 = run_all(*wide, meta, p, dtype="fp64")
        np.testing.assert_array_equal(O1, O2)
        np.testing.assert_array_equal(L1, L2)


def test_batch_strided_metadata():
    # Branch b reads its own metadata set at b*stride; equal sets give equal results.
    q, k, v, meta, p = tiny_case(seed=11, B=2)
    N = len(meta["seg"])
    meta2 = {key: np.concatenate([val, val]) for key, val in meta.items()}
    O1, L1 = run_all(q, k, v, meta, p)
    O2, L2 = run_all(q, k, v, meta2, p, meta_batch_stride=N)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


# ---------------------------------------------------------------------------------------
# packer pins
# ---------------------------------------------------------------------------------------
def test_packer_microbenchmark_length(golden_rule):
    # "On an RTX PRO 6000 Blackwell at 107,126 tokens" ("What the numbers say").
    n = int(golden_rule["microbenchmark_tokens"][0])
    for name in ("micro", "full"):
        meta = oracle.pack_token_meta(W.get(name).segments)
        assert len(meta["seg"]) == n


def test_packer_clock_and_roles(golden_rule):
    # 24 fps on both sides ("Wiring it"); a latent frame's tokens share its time; roles and
    # Picture indices follow the segment order; mask modes follow "Inputs you'll set".
    fps = golden_rule["fps"][0]
    w = W.get("tiny")
    meta = oracle.pack_token_meta(w.segments)
    seg, t, pic, m = meta["seg"], meta["time_s"], meta["pic"], meta["m"]
    assert list(np.bincount(seg, minlength=6)) == [16, 32, 64, 64, 16, 0]
    tgt = np.where(seg == W.TARGET)[0]
    gd = np.where(seg == W.GUIDE)[0]
    for f in range(4):
        expect = np.float32(f * 4 / fps)
        assert np.all(t[tgt[f * 16:(f + 1) * 16]] == expect)
        assert np.all(t[gd[f * 16:(f + 1) * 16]] == expect)
    assert np.all(pic[seg == W.PICTURE] == 1) and np.all(pic[seg != W.PICTURE] == 0)
    np.testing.assert_array_equal(m[tgt], w.segments[2].mask)
    assert np.all(m[seg != W.TARGET] == 1.0)
    # static mask repeats per frame; no mask means weight 1
    full = oracle.pack_token_meta(W.get("full").segments)
    tg = full["m"][full["seg"] == W.TARGET].reshape(26, 2000)
    assert np.all(tg == tg[0]) and 0.0 < tg.min() and tg.max() < 1.0
    rg = oracle.pack_token_meta(W.get("ragged").segments)
    assert np.all(rg["m"] == 1.0)
    gt = rg["time_s"][rg["seg"] == W.GUIDE].reshape(26, 461)
    np.testing.assert_array_equal(gt[:, 0], (np.arange(26) * 4 / fps + 1 / fps).astype(np.float32))


# ---------------------------------------------------------------------------------------
# chained bindings ("Common issues": two subjects are two chained binding nodes; overlapping
# masks combine their log gains)
# ---------------------------------------------------------------------------------------
def _two_bindings(seed, m2_fn):
    q, k, v, meta, _ = tiny_case(seed=seed)
    N = len(meta["seg"])
    rng = np.random.Generator(np.random.PCG64(seed + 50))
    m2 = np.ones(N, dtype=np.float32)
    tgt = meta["seg"] == W.TARGET
    m2[tgt] = m2_fn(rng, int(tgt.sum()))
    meta = dict(meta, m_extra=m2[None, :])
    g1 = (1.25, 0.75) + (1.0,) * 7            # binding 0: Picture 1 chosen
    g2 = (0.9, 1.6) + (0.9,) * 7              # binding 1: Picture 2 chosen
    p = W.Params(gain=g1, extra_gain=(g2,))
    return q, k, meta, p, g1, g2, m2


def test_overlapping_bindings_multiply_gain_powers():
    q, k, meta, p, g1, g2, m2 = _two_bindings(20, lambda rng, n: rng.uniform(0, 1, n))
    neutral = W.Params(p.window, p.falloff, p.strength, p.cap, (1.0,) * 9)
    ratio = _edge_weights(q, k, meta, p) / _edge_weights(q, k, {kk: vv for kk, vv in meta.items() if kk != "m_extra"}, neutral)
    seg, pic, m = meta["seg"], meta["pic"], meta["m"].astype(np.float64)
    f32 = lambda g: np.array([float(np.float32(x)) for x in g])
    a, b = f32(g1), f32(g2)
    N = len(seg)
    for i in range(N):
        for j in range(N):
            if seg[i] == W.TARGET and seg[j] == W.PICTURE:
                expect = a[pic[j] - 1] ** m[i] * b[pic[j] - 1] ** float(m2[i])
            else:
                expect = 1.0
            assert ratio[0, 0, i, j] == pytest.approx(expect, rel=1e-12, abs=0), (i, j)


def test_extra_binding_with_zero_mask_changes_nothing():
    q, k, meta, p, g1, g2, m2 = _two_bindings(21, lambda rng, n: np.zeros(n))
    v = np.random.Generator(np.random.PCG64(9)).standard_normal(q.shape)
    O1, L1 = run_all(q, k, v, meta, p)
    single = W.Params(gain=g1)
    O0, L0 = run_all(q, k, v, {kk: vv for kk, vv in meta.items() if kk != "m_extra"}, single)
    np.testing.assert_array_equal(O1, O0)
    np.testing.assert_array_equal(L1, L0)


def test_disjoint_bindings_act_on_their_own_rows():
    # binding 0 masks the first half of the target rows, binding 1 the second half
    q, k, meta, p, g1, g2, m2 = _two_bindings(22, lambda rng, n: (np.arange(n) >= n // 2).astype(np.float32))
    tgt = np.where(meta["seg"] == W.TARGET)[0]
    m = meta["m"].copy()
    m[tgt] = (np.arange(len(tgt)) < len(tgt) // 2).astype(np.float32)
    meta = dict(meta, m=m)
    v = np.random.Generator(np.random.PCG64(10)).standard_normal(q.shape)
    O, L = run_all(q, k, v, meta, p)
    no_extra = {kk: vv for kk, vv in meta.items() if kk != "m_extra"}
    Oa, La = run_all(q, k, v, no_extra, W.Params(gain=g1))
    m_b = m.copy()
    m_b[tgt] = m2[tgt]
    Ob, Lb = run_all(q, k, v, dict(no_extra, m=m_b), W.Params(gain=g2))
    first, second = tgt[: len(tgt) // 2], tgt[len(tgt) // 2:]
    np.testing.assert_allclose(O[:, :, first], Oa[:, :, first], atol=1e-13, rtol=0)
    np.testing.assert_allclose(O[:, :, second], Ob[:, :, second], atol=1e-13, rtol=0)
    np.testing.assert_allclose(L[:, :, second], Lb[:, :, second], atol=1e-13, rtol=0)
