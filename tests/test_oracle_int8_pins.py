"""Pins of the INT8-QK^T oracle (`oracle/int8_qk.py`) against facts that do not come from it.

The quantiser is checked against: groups it must reproduce exactly (integers already on the
8-bit grid), exact power-of-two scaling, the rounding error bound of uniform symmetric
quantisation, a brute-force nearest-code search with ties to even, block independence of the
K scales, and the zero group.  The composed variant is checked against the plain oracle on
inputs the quantiser reproduces exactly, and against the logit and LSE error bounds that
follow from the per-element quantisation errors.
"""
import numpy as np

import oracle
from oracle import int8_qk as Q8
import workloads as W

RNG = lambda s: np.random.Generator(np.random.PCG64(s))   # noqa: E731


def _grid_group(rng, n, pow2=0):
    """n integers in [-127, 127] with one +-127, times 2**pow2 (exactly on the 8-bit grid)."""
    x = rng.integers(-127, 128, size=n).astype(np.float32)
    x[rng.integers(0, n)] = 127.0 * rng.choice([-1.0, 1.0])
    return (x * np.float32(2.0 ** pow2)).astype(np.float32)


def test_grid_values_are_reproduced_exactly():
    rng = RNG(1)
    for pow2 in (-20, -3, 0, 5):
        x = np.stack([_grid_group(rng, 64, pow2) for _ in range(9)])
        codes, scales = Q8._quantise_groups(x)
        np.testing.assert_array_equal(scales, np.float32(2.0 ** pow2))
        np.testing.assert_array_equal(codes.astype(np.float32) * scales[:, None], x)


def test_power_of_two_scaling_is_exact():
    rng = RNG(2)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    c0, s0 = Q8._quantise_groups(x)
    for e in (-30, -7, 1, 9, 40):
        c, s = Q8._quantise_groups((x * np.float32(2.0 ** e)).astype(np.float32))
        np.testing.assert_array_equal(c, c0)
        np.testing.assert_array_equal(s, (s0 * np.float32(2.0 ** e)).astype(np.float32))


def test_rounding_error_bound_and_range():
    rng = RNG(3)
    x = (rng.standard_normal((64, 128)) * rng.uniform(0.01, 50, (64, 1))).astype(np.float32)
    codes, scales = Q8._quantise_groups(x)
    c = codes.astype(np.float64)
    assert np.all(np.abs(c) <= 127)
    # the element of largest magnitude lands on +-127
    top = np.abs(x).argmax(axis=1)
    np.testing.assert_array_equal(np.abs(c[np.arange(64), top]), 127)
    # |x - code*scale| <= scale/2, up to the float32 roundings of inv and of x*inv
    err = np.abs(x.astype(np.float64) - c * scales[:, None].astype(np.float64))
    bound = scales[:, None].astype(np.float64) * (0.5 + 2.0 ** -16)
    assert np.all(err <= bound)


def _nearest_code_search(p: float) -> int:
    """The integer in [-127, 127] nearest to p, ties to the even one, by exhaustive search."""
    best = None
    for c in range(-127, 128):
        d = abs(p - c)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1]


def test_codes_match_a_brute_force_search_with_ties():
    rng = RNG(4)
    # ties: amax 127 makes inv exactly 1, so k + 0.5 values sit exactly between two codes
    ties = np.array([127.0, 2.5, -2.5, 3.5, -0.5, 0.5, 126.5, -126.5], np.float32)
    groups = [ties] + [rng.standard_normal(8).astype(np.float32) * 3 for _ in range(20)]
    for g in groups:
        codes, scales = Q8._quantise_groups(g[None, :])
        amax = np.float32(np.max(np.abs(g)))
        inv = np.float32(np.float32(127.0) / amax)
        for x, c in zip(g, codes[0]):
            p = float(np.float32(x * inv))
            assert int(c) == _nearest_code_search(p), (x, p, c)
        assert scales[0] == np.float32(amax / np.float32(127.0))


def test_zero_and_negligible_groups():
    x = np.zeros((3, 16), np.float32)
    x[1, 3] = 1e-31
    x[2, 5] = -2e-30
    codes, scales = Q8._quantise_groups(x)
    np.testing.assert_array_equal(codes[:2], 0)
    np.testing.assert_array_equal(scales[:2], 0)
    assert scales[2] > 0 and codes[2, 5] == -127


def test_k_blocks_are_independent_and_the_tail_covers_valid_tokens():
    rng = RNG(5)
    B, H, N, D = 1, 2, 300, 16
    k = rng.standard_normal((B, H, N, D)).astype(np.float32)
    c0, s0 = Q8.quantise_k(k)
    assert s0.shape == (B, H, 3)
    k2 = k.copy()
    k2[:, :, 7, 3] = 1000.0                      # an outlier in block 0 only
    c1, s1 = Q8.quantise_k(k2)
    np.testing.assert_array_equal(s1[:, :, 1:], s0[:, :, 1:])
    np.testing.assert_array_equal(c1[:, :, 128:], c0[:, :, 128:])
    assert np.all(s1[:, :, 0] > s0[:, :, 0])
    # the last block holds tokens 256..299 only
    expect = (np.max(np.abs(k[:, :, 256:, :]), axis=(2, 3)) / np.float32(127)).astype(np.float32)
    np.testing.assert_array_equal(s0[:, :, 2], expect)
    # Q is per token: one outlier changes one row's scale
    cq0, sq0 = Q8.quantise_q(k)
    cq1, sq1 = Q8.quantise_q(k2)
    changed = np.argwhere(sq1 != sq0)
    assert changed.tolist() == [[0, 0, 7], [0, 1, 7]]


def _tiny_meta():
    w = W.get("tiny")
    return w, oracle.pack_token_meta(w.segments)


def test_variant_equals_the_plain_oracle_on_grid_inputs():
    # operands already on the 8-bit grid (per token for Q, per 128-token block for K) are
    # quantised losslessly, so the variant must give the plain rule's result exactly
    w, meta = _tiny_meta()
    rng = RNG(6)
    B, H, N, D = w.B, w.H, w.N, w.D
    q = np.stack([np.stack([np.stack([_grid_group(rng, D, -7) for _ in range(N)])
                            for _ in range(H)]) for _ in range(B)])
    k = np.empty((B, H, N, D), np.float32)
    for b in range(B):
        for h in range(H):
            for j in range(0, N, 128):
                n = min(128, N - j)
                k[b, h, j:j + n] = _grid_group(rng, n * D, -6 - j // 128).reshape(n, D)
    v = rng.standard_normal((B, H, N, D)).astype(np.float32)
    rows = oracle.all_rows(B, H, N)
    O8, L8 = Q8.attention_rows_int8qk(q, k, v, "fp32", meta, w.params, rows)
    O, L = oracle.attention_rows(q, k, v, "fp32", meta, w.params, rows)
    np.testing.assert_array_equal(O8, O)
    np.testing.assert_array_equal(L8, L)


def test_logit_and_lse_errors_within_the_quantisation_bound():
    # |q.k - q^.k^| <= sum_d |q_d| sk/2 + |k_d| sq/2 + sq sk/4 (per-element errors <= scale/2),
    # and the LSE moves by at most the largest logit change
    w, meta = _tiny_meta()
    rng = RNG(7)
    B, H, N, D = w.B, w.H, w.N, w.D
    q = (rng.standard_normal((B, H, N, D)) * 1.5).astype(np.float32)
    k = (rng.standard_normal((B, H, N, D)) * 1.5).astype(np.float32)
    v = rng.standard_normal((B, H, N, D)).astype(np.float32)
    cq, sq = Q8.quantise_q(q)
    ck, sk = Q8.quantise_k(k)
    qd, kd = Q8.dequantise_q(cq, sq), Q8.dequantise_k(ck, sk)
    scale = 1.0 / np.sqrt(D)
    rows = oracle.all_rows(B, H, N)
    _, L8 = Q8.attention_rows_int8qk(q, k, v, "fp32", meta, w.params, rows)
    _, L = oracle.attention_rows(q, k, v, "fp32", meta, w.params, rows)
    q64, k64 = q.astype(np.float64), k.astype(np.float64)
    skt = np.repeat(sk.astype(np.float64), 128, axis=2)[:, :, :N]
    for r, (b, h, i) in enumerate(rows):
        exact = oracle.logit_row(q64, k64, "fp64", meta, w.params, b, h, i)
        quant = oracle.logit_row(np.ascontiguousarray(qd), np.ascontiguousarray(kd), "fp64",
                                 meta, w.params, b, h, i)
        sqi = float(sq[b, h, i])
        bound = scale * (np.abs(q64[b, h, i]).sum() * skt[b, h] / 2
                         + np.abs(k64[b, h]).sum(axis=1) * sqi / 2 + D * sqi * skt[b, h] / 4)
        dl = np.abs(quant - exact)
        assert np.all(dl <= bound * (1 + 1e-9) + 1e-12), r
        assert abs(L8[r] - L[r]) <= dl.max() * (1 + 1e-9) + 1e-12
    # and the bound is not vacuous: the quantised logits do move
    assert np.max(np.abs(L8 - L)) > 0
