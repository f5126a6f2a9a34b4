"""Pins for the oracle: checks against the FP16 format definition, the
hand-worked examples in ``tests/golden``, closed-form error bounds and
ranges, brute force over the whole level-2 domain, and numpy's own integer
matmul.  None of these re-types the oracle's formulas.

Passages pinned: "QServe: W4A8KV4 Quantization and System Co-design for
Efficient LLM Serving" (velog notes), Methods 1) Algorithm: QoQ and
2) System: QServe; same page, Background (no partial-sum dequantization).
"""
import math
import os
from fractions import Fraction

import numpy as np
import warnings
import pytest

import synthetic_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.txt")


def _golden(kind):
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line.startswith(kind + ":"):
                continue
            parts = [p.split() for p in line[len(kind) + 1:].split("|")]
            rows.append(parts)
    assert rows, kind
    return rows


# ---------------------------------------------------------------------------
# FP16 conversions
# ---------------------------------------------------------------------------

def test_fp16_decode_all_patterns(oracle):
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.h2d_array(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.isnan(got[nan]).all()
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_fp16_roundtrip_all_patterns(oracle):
    bits = np.arange(65536, dtype=np.uint16)
    vals = bits.view(np.float16)
    finite = np.isfinite(vals) | np.isinf(vals)
    back = oracle.d2h_array(vals.astype(np.float64))
    assert np.array_equal(back[finite], bits[finite])
    back32 = oracle.f2h_array(vals.astype(np.float32))
    assert np.array_equal(back32[finite], bits[finite])
    # a NaN encodes as a NaN: all-ones exponent and a non-zero fraction
    for enc in (back[~finite], back32[~finite]):
        assert enc.size == 2 * 1023
        assert ((enc & 0x7c00) == 0x7c00).all() and ((enc & 0x03ff) != 0).all()


def test_fp16_ties_go_to_even(oracle):
    # every exact midpoint between consecutive finite FP16 values, from
    # binary64 (numpy converts binary64 -> binary16 directly, RNE)
    pos = np.arange(0, 0x7bff, dtype=np.uint16)
    lo = pos.view(np.float16).astype(np.float64)
    hi = (pos + 1).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2.0
    got = oracle.d2h_array(mid)
    expect = np.where(pos % 2 == 0, pos, pos + 1).astype(np.uint16)
    assert np.array_equal(got, expect)
    # just above / below a midpoint rounds away from / toward lo
    eps = np.abs(mid) * 2.0 ** -40 + 2.0 ** -60
    assert np.array_equal(oracle.d2h_array(mid + eps), (pos + 1).astype(np.uint16))
    assert np.array_equal(oracle.d2h_array(mid - eps), pos)
    assert np.array_equal(oracle.d2h_array(-mid), expect | 0x8000)


def test_fp16_random_floats_match_numpy(oracle):
    rng = np.random.default_rng(123)
    x = np.concatenate([
        rng.standard_normal(400_000).astype(np.float32),
        (rng.standard_normal(200_000) * 1e-5).astype(np.float32),
        (rng.standard_normal(200_000) * 3e4).astype(np.float32),
        rng.uniform(-7e4, 7e4, 100_000).astype(np.float32),
        np.array([65504, 65519.99, 65520, 65536, 1e-8, 2.98e-8, 2.9802322e-08,
                  5.96e-8, -0.0, 0.0], np.float32),
    ])
    with warnings.catch_warnings():
        warnings.simplefilter("ignore", RuntimeWarning)   # overflow to inf
        ref = x.astype(np.float16).view(np.uint16)
        xd = x.astype(np.float64) * (1 + 2.0 ** -30)
        refd = xd.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.f2h_array(x), ref)
    assert np.array_equal(oracle.d2h_array(xd), refd)


# ---------------------------------------------------------------------------
# exact integer round-half-even division
# ---------------------------------------------------------------------------

def test_rne_div_bruteforce(oracle):
    for b in range(1, 21):
        for a in range(-300, 301):
            assert oracle.rne_div(a, b) == round(Fraction(a, b)), (a, b)


# ---------------------------------------------------------------------------
# Level 2 (per group, UINT4 asymmetric)
# ---------------------------------------------------------------------------

def test_level2_hand_examples(oracle):
    for w8, sz, q, dq in _golden("level2"):
        W8 = np.array([[int(v) for v in w8]], np.int8)
        qq, s2, z = oracle.quant_w_level2(W8, 4)
        assert [int(s2[0, 0]), int(z[0, 0])] == [int(v) for v in sz], w8
        assert qq[0].tolist() == [int(v) for v in q], w8
        d = oracle.dequant_w(qq, s2, z, 4)
        assert d[0].tolist() == [int(v) for v in dq], w8


def _level2_domain_groups(G=128):
    """Groups covering every (min, max, w) with -119 <= min <= 0 <= max <= 119
    and min <= w <= max: each group holds min and max plus a slice of the
    values in between."""
    groups = []
    for mn in range(-119, 1):
        for mx in range(0, 120):
            vals = np.arange(mn, mx + 1, dtype=np.int16)
            for start in range(0, len(vals), G - 2):
                chunk = vals[start:start + G - 2]
                g = np.full(G, mn, np.int16)
                g[1] = mx
                g[2:2 + len(chunk)] = chunk
                groups.append(g)
    return np.stack(groups).astype(np.int8)


@pytest.fixture(scope="module")
def level2_domain(oracle):
    W8 = _level2_domain_groups()
    q, s2, z = oracle.quant_w_level2(W8, 128)
    dq = oracle.dequant_w(q, s2, z, 128)
    return W8, q, s2[:, 0].astype(np.int32), z[:, 0].astype(np.int32), dq


def test_level2_bruteforce_half_step_bound(level2_domain):
    W8, q, s2, z, dq = level2_domain
    err2 = 2 * np.abs(W8.astype(np.int32) - dq.astype(np.int32))
    assert (err2 <= s2[:, None]).all()          # |W8 - dq| <= s2 / 2


def test_level2_bruteforce_ranges(level2_domain):
    W8, q, s2, z, dq = level2_domain
    assert q.min() >= 0 and q.max() <= 15
    assert z.min() >= 0 and z.max() <= 15
    assert s2.min() >= 1 and s2.max() <= 16
    assert (q.astype(np.int32) * s2[:, None]).max() <= 240   # fits a byte lane
    assert (z * s2).max() <= 240
    d = dq.astype(np.int32)
    # dq stays inside INT8: the protective range 119 gives |dq| <= 121
    assert d.min() == -121 and d.max() == 121


def test_level2_bruteforce_scale_is_minimal(level2_domain):
    W8, q, s2, z, dq = level2_domain
    w = W8.astype(np.int32)
    rng_ = np.maximum(w.max(1), 0) - np.minimum(w.min(1), 0)
    # 15 steps of s2 cover the range, and 15 steps of s2 - 1 do not
    assert (15 * s2 >= rng_).all()
    small = s2 > 1
    assert (15 * (s2[small] - 1) < rng_[small]).all()
    # lossless whenever the range fits 15 unit steps
    lossless = rng_ <= 15
    assert np.array_equal(dq[lossless], W8[lossless])


def test_level2_groups_are_independent(level2_domain, oracle):
    # Rows of several groups: each group's (q, s2, z, dq) must be exactly
    # what that group gives alone, in its own place along K, for G = 128 and
    # for G = 64 (where each half of a 128-wide domain group is its own group).
    W8, q, s2, z, dq = level2_domain
    n = (W8.shape[0] // 4) * 4
    rows = W8[:n].reshape(n // 4, 4 * 128)
    qr, s2r, zr = oracle.quant_w_level2(rows, 128)
    assert np.array_equal(qr, q[:n].reshape(n // 4, 512))
    assert np.array_equal(s2r.astype(np.int32), s2[:n].reshape(n // 4, 4))
    assert np.array_equal(zr.astype(np.int32), z[:n].reshape(n // 4, 4))
    dqr = oracle.dequant_w(qr, s2r, zr, 128)
    assert np.array_equal(dqr, dq[:n].reshape(n // 4, 512))
    halves = W8[:n].reshape(2 * n, 64)
    qh, s2h, zh = oracle.quant_w_level2(halves, 64)
    q64, s264, z64 = oracle.quant_w_level2(rows, 64)
    assert np.array_equal(q64, qh.reshape(n // 4, 512))
    assert np.array_equal(s264, s2h.reshape(n // 4, 8))
    assert np.array_equal(z64, zh.reshape(n // 4, 8))
    assert np.array_equal(oracle.dequant_w(q64, s264, z64, 64),
                          oracle.dequant_w(qh, s2h, zh, 64).reshape(n // 4, 512))


def test_level2_full_range_reduces_to_grid(oracle):
    # every group spans exactly [-119, 119]: s2 = 16, z = 7 and the result is
    # the nearest multiple of 16 (ties to even multiple), clipped to 7 steps
    rng = np.random.default_rng(5)
    W8 = rng.integers(-119, 120, size=(64, 128)).astype(np.int8)
    W8[:, 0] = -119
    W8[:, 1] = 119
    q, s2, z = oracle.quant_w_level2(W8, 128)
    assert (s2 == 16).all() and (z == 7).all()
    dq = oracle.dequant_w(q, s2, z, 128).astype(np.int32)
    grid = 16 * np.array([[round(Fraction(int(v), 16)) for v in r] for r in W8])
    assert np.array_equal(dq, np.clip(grid, -112, 128))


# ---------------------------------------------------------------------------
# Level 1 (per output channel, symmetric INT8 with FP16 scale)
# ---------------------------------------------------------------------------

def test_level1_hand_examples(oracle):
    for w, s1h, w8 in _golden("level1"):
        W = np.array([[float(v) for v in w]], np.float16)
        assert np.array_equal(W.astype(np.float64)[0], [float(v) for v in w])
        s1, W8 = oracle.quant_w_level1(W)
        assert int(s1.view(np.uint16)[0]) == int(s1h[0], 16)
        assert W8[0].tolist() == [int(v) for v in w8]


def test_level1_bounds_and_symmetry(oracle):
    W = si.weights(si.TINY, seed=3)
    s1, W8 = oracle.quant_w_level1(W)
    Wf = W.astype(np.float64)
    s = s1.astype(np.float64)
    w8 = W8.astype(np.int32)
    amax = np.abs(Wf).max(1)
    # the row maximum lands on the edge of the protective range
    assert (np.abs(w8).max(1) >= 118).all() and np.abs(w8).max() <= 119
    # sign preserved
    assert (np.sign(w8) * np.sign(Wf) >= 0).all()
    # round-trip error: half a step, plus the slack of rounding s1 to FP16
    slack = np.maximum(amax - 119 * s, 0)
    err = np.abs(Wf - w8 * s[:, None])
    assert (err <= s[:, None] / 2 + slack[:, None] + 1e-12).all()
    assert (slack <= 0.06 * s).all()
    # the FP16 scale is within half an FP16 step of amax / 119
    ulp = np.spacing(s1.astype(np.float16)).astype(np.float64)
    assert (np.abs(s - amax / 119) <= ulp / 2 + 1e-12).all()
    # negation symmetry and exact power-of-two scaling
    s1n, W8n = oracle.quant_w_level1(-W)
    assert np.array_equal(s1n, s1) and np.array_equal(W8n, -W8)
    s1d, W8d = oracle.quant_w_level1((W.astype(np.float32) * 4).astype(np.float16))
    assert np.array_equal(s1d.astype(np.float64), 4 * s) and np.array_equal(W8d, W8)


def test_level1_tiny_scale_guard(oracle):
    W = np.zeros((2, 8), np.float16)
    W[1, 3] = np.float16(2.0 ** -24)           # smallest subnormal
    s1, W8 = oracle.quant_w_level1(W)
    assert s1.view(np.uint16).tolist() == [0x3c00, 0x0001]
    assert W8[1, 3] == 1 and W8[0].tolist() == [0] * 8


def test_level1_subnormal_scale_keeps_protective_range(oracle):
    # Row maxima of k * 2^-24 for every k up to the first normal binary16
    # values: there the FP16 scale fp16(amax / 119) can round down by far more
    # than half a step, and only the clamp keeps the codes inside the
    # protective range of +-119 (a code of 120 or more would push level-2 dq
    # past INT8).
    k = np.arange(1, 2048, dtype=np.float64)
    W = np.zeros((k.size, 4), np.float16)
    W[:, 0] = (k * 2.0 ** -24).astype(np.float16)
    W[:, 1] = (-k * 2.0 ** -24).astype(np.float16)
    W[:, 2] = (k * 2.0 ** -25).astype(np.float16)
    assert np.array_equal(W[:, 0].astype(np.float64), k * 2.0 ** -24)
    s1, W8 = oracle.quant_w_level1(W)
    w8 = W8.astype(np.int32)
    assert np.abs(w8).max() == 119
    assert np.array_equal(w8[:, 1], -w8[:, 0])
    # amax / 119 is below 18 quanta of 2^-24, so the FP16 scale is that many
    # quanta rounded to nearest (never a tie: 119 is odd), or the smallest
    # positive FP16 value where that rounds to 0
    s = s1.astype(np.float64)
    assert np.array_equal(s, np.maximum(1, np.round(k / 119)) * 2.0 ** -24)
    # where rounding the scale cost more than half a code, the code saturates
    ratio = k * 2.0 ** -24 / s
    assert (w8[ratio >= 119.5, 0] == 119).all()
    assert (ratio >= 119.5).any()


# ---------------------------------------------------------------------------
# Per-token activations
# ---------------------------------------------------------------------------

def test_act_hand_examples(oracle):
    for x, sxh, x8 in _golden("act"):
        X = np.array([[float(v) for v in x]], np.float16)
        X8, sx = oracle.quant_act(X)
        assert int(sx.view(np.uint16)[0]) == int(sxh[0], 16)
        assert X8[0].tolist() == [int(v) for v in x8]


def test_act_bounds(oracle):
    X = si.activations(si.TINY, 16, seed=0)
    X8, sx = oracle.quant_act(X)
    Xf = X.astype(np.float64)
    s = sx.astype(np.float64)
    x8 = X8.astype(np.int32)
    amax = np.abs(Xf).max(1)
    assert (np.abs(x8).max(1) >= 126).all() and np.abs(x8).max() <= 127
    slack = np.maximum(amax - 127 * s, 0)
    err = np.abs(Xf - x8 * s[:, None])
    assert (err <= s[:, None] / 2 + slack[:, None] + 1e-12).all()
    X8n, sxn = oracle.quant_act(-X)
    assert np.array_equal(X8n, -X8) and np.array_equal(sxn, sx)


def test_act_subnormal_scale_stays_symmetric(oracle):
    # As for the weights: with a subnormal FP16 scale, X / sx can exceed 127
    # by far; the codes must still stay in the symmetric range [-127, 127].
    k = np.arange(1, 2048, dtype=np.float64)
    X = np.zeros((k.size, 3), np.float16)
    X[:, 0] = (-k * 2.0 ** -24).astype(np.float16)
    X[:, 1] = (k * 2.0 ** -25).astype(np.float16)
    X8, sx = oracle.quant_act(X)
    x8 = X8.astype(np.int32)
    assert x8.min() == -127 and x8.max() <= 127
    X8n, sxn = oracle.quant_act(-X)
    assert np.array_equal(X8n.astype(np.int32), -x8) and np.array_equal(sxn, sx)
    ratio = k * 2.0 ** -24 / sx.astype(np.float64)
    assert (x8[ratio >= 127.5, 0] == -127).all()
    assert (ratio >= 127.5).any()


# ---------------------------------------------------------------------------
# Integer GEMM and epilogue
# ---------------------------------------------------------------------------

def test_int_gemm_matches_numpy_int64(oracle):
    rng = np.random.default_rng(11)
    for M, N, K in [(1, 1, 1), (3, 5, 7), (17, 33, 256), (16, 128, 512)]:
        X8 = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
        dq = rng.integers(-121, 122, size=(N, K), dtype=np.int8)
        ref = X8.astype(np.int64) @ dq.astype(np.int64).T
        assert np.array_equal(oracle.int_gemm(X8, dq), ref)
        ms = rng.integers(0, M, 50)
        ns = rng.integers(0, N, 50)
        assert np.array_equal(oracle.int_gemm_at(X8, dq, ms, ns), ref[ms, ns])


def test_int_gemm_bruteforce_tiny(oracle):
    rng = np.random.default_rng(12)
    X8 = rng.integers(-127, 128, size=(3, 9), dtype=np.int8)
    dq = rng.integers(-121, 122, size=(4, 9), dtype=np.int8)
    acc = oracle.int_gemm(X8, dq)
    for m in range(3):
        for n in range(4):
            s = 0
            for k in range(9):
                s += int(X8[m, k]) * int(dq[n, k])
            assert acc[m, n] == s


def test_int_gemm_one_hot_columns(oracle):
    rng = np.random.default_rng(13)
    K, N = 256, 64
    dq = rng.integers(-121, 122, size=(N, K), dtype=np.int8)
    ks = rng.choice(K, 32, replace=False)
    X8 = np.zeros((32, K), np.int8)
    X8[np.arange(32), ks] = 1
    acc = oracle.int_gemm(X8, dq)
    assert np.array_equal(acc, dq[:, ks].T.astype(np.int32))


def test_int_gemm_extreme_fits_int32(oracle):
    K = 16384
    X8 = np.full((1, K), -127, np.int8)
    dq = np.full((2, K), 121, np.int8)
    dq[1] = -121
    acc = oracle.int_gemm(X8, dq)
    assert acc.tolist() == [[-127 * 121 * K, 127 * 121 * K]]


def test_int_gemm_reports_int32_overflow(oracle):
    # 127 * 127 * K fits INT32 up to K = 133144 and not beyond: the bound on
    # K that keeps the INT32 accumulator exact for any INT8 operands.
    for K, fits in ((133144, True), (133145, False)):
        X8 = np.full((1, K), 127, np.int8)
        dq = np.full((2, K), 127, np.int8)
        dq[1] = -127
        if fits:
            acc = oracle.int_gemm(X8, dq)
            assert acc.tolist() == [[127 * 127 * K, -127 * 127 * K]]
        else:
            with pytest.raises(OverflowError):
                oracle.int_gemm(X8, dq)


def test_epilogue_matches_numpy(oracle):
    rng = np.random.default_rng(14)
    M, N = 7, 33
    acc = rng.integers(-2 ** 27, 2 ** 27, size=(M, N)).astype(np.int32)
    sx = (rng.uniform(0.5, 1.5, M) * 1e-2).astype(np.float16)
    s1 = (rng.uniform(0.5, 1.5, N) * 1e-3).astype(np.float16)
    Y = oracle.epilogue(acc, sx, s1)
    ref = (acc.astype(np.float64) * sx.astype(np.float64)[:, None]
           * s1.astype(np.float64)[None, :]).astype(np.float16)
    assert np.array_equal(Y.view(np.uint16), ref.view(np.uint16))


# ---------------------------------------------------------------------------
# End to end on the small workload: the quantized product stays within the
# analytic error bound of the unquantized X @ W^T.
# ---------------------------------------------------------------------------

def test_end_to_end_error_bound_tiny(oracle):
    L = si.TINY
    W = si.weights(L, seed=0)
    X = si.activations(L, 16, seed=0)
    Wq = oracle.quantize_weights(W, L.group)
    X8, sx, acc, Y = oracle.w4a8_forward(X, Wq["dq"], Wq["s1"])
    Xf = X.astype(np.float64)
    Wf = W.astype(np.float64)
    s1 = Wq["s1"].astype(np.float64)
    s2 = np.repeat(Wq["s2"].astype(np.float64), L.group, axis=1)
    sxf = sx.astype(np.float64)
    exact = Xf @ Wf.T
    amax_w = np.abs(Wf).max(1)
    amax_x = np.abs(Xf).max(1)
    dW = s1[:, None] * (0.5 + s2 / 2) + np.maximum(amax_w - 119 * s1, 0)[:, None]
    dX = sxf[:, None] / 2 + np.maximum(amax_x - 127 * sxf, 0)[:, None]
    bound = (np.abs(Xf) @ dW.T + dX * np.abs(Wf).sum(1)[None, :]
             + dX * dW.sum(1)[None, :])
    bound += np.abs(exact) * 2.0 ** -11 + 2.0 ** -24 * 4
    Yf = Y.astype(np.float64)
    assert (np.abs(Yf - exact) <= bound).all()
    # and the result tracks the exact product: 16 levels per group give a
    # relative error near step / sqrt(12) of the weights, about 12 % here
    rel = np.linalg.norm(Yf - exact) / np.linalg.norm(exact)
    assert rel < 0.2
    # the scaled INT32 accumulator agrees with Y
    ref = acc.astype(np.float64) * sxf[:, None] * s1[None, :]
    assert np.array_equal(Y.view(np.uint16), ref.astype(np.float16).view(np.uint16))


def test_planted_mistakes_are_caught(oracle):
    """A transposed operand or a dropped zero term in dq breaks the pins."""
    L = si.TINY
    W = si.weights(L, seed=0)
    Wq = oracle.quantize_weights(W, L.group)
    q, s2, z = Wq["q"], Wq["s2"], Wq["z"]
    # dropping the zero term (dq = q*s2) leaves the half-step bound
    bad = (q.astype(np.int32) * np.repeat(s2, L.group, 1).astype(np.int32))
    err2 = 2 * np.abs(Wq["W8"].astype(np.int32) - bad)
    assert not (err2 <= np.repeat(s2, L.group, 1)).all()
    # a transposed weight operand breaks the one-hot column identity
    X8 = np.eye(L.K, dtype=np.int8)[:8]
    acc = oracle.int_gemm(X8, Wq["dq"])
    assert np.array_equal(acc, Wq["dq"][:, :8].T.astype(np.int32))
    assert not np.array_equal(acc, Wq["dq"][:8, :].astype(np.int32)[:, :Wq["dq"].shape[0]])


# ---------------------------------------------------------------------------
# Per-input-channel smoothing ("Part5 LLM部署技术", 1.1 权重-激活联合量化：
# SmoothQuant): calibration maxima, X / s and W * s, migration strength 0.5
# ---------------------------------------------------------------------------

def _hex16(h):
    return np.array([int(h, 16)], np.uint16).view(np.float16)


def test_smoothing_hand_examples(oracle):
    for (ax, aw), (sh,) in _golden("smooth_factor"):
        Xc = np.array([[float(ax)]], np.float16)
        W = np.array([[float(aw)]], np.float16)
        s = oracle.smooth_factors(Xc, W)
        assert s.view(np.uint16)[0] == int(sh, 16), (ax, aw, s)
    for (wh, sh), (outh,) in _golden("smooth_weight"):
        got = oracle.smooth_weights(_hex16(wh).reshape(1, 1), _hex16(sh))
        assert got.view(np.uint16)[0, 0] == int(outh, 16), (wh, sh)
    for (xh, sh), (outh,) in _golden("smooth_act"):
        got = oracle.smooth_act(_hex16(xh).reshape(1, 1), _hex16(sh))
        assert got.view(np.uint16)[0, 0] == int(outh, 16), (xh, sh)


def test_smoothing_by_one_is_identity(oracle):
    """Every finite FP16 value is unchanged by the factor 1."""
    bits = np.arange(65536, dtype=np.uint16)
    vals = bits.view(np.float16)
    vals = vals[np.isfinite(vals)].reshape(1, -1)
    ones = np.ones(vals.shape[1], np.float16)
    assert np.array_equal(oracle.smooth_weights(vals, ones).view(np.uint16), vals.view(np.uint16))
    assert np.array_equal(oracle.smooth_act(vals, ones).view(np.uint16), vals.view(np.uint16))


def test_smoothing_by_powers_of_two_is_exact(oracle):
    """A factor 2^e scales exactly wherever the result stays a normal FP16
    number: W * 2^e and X / 2^e."""
    rng = np.random.default_rng(5)
    vals = rng.uniform(-2.0, 2.0, (7, 64)).astype(np.float16)
    vals[np.abs(vals) < 2.0 ** -10] = 0.5
    for e in (-3, -1, 1, 4):
        s = np.full(64, 2.0 ** e, np.float16)
        w = oracle.smooth_weights(vals, s).astype(np.float64)
        x = oracle.smooth_act(vals, s).astype(np.float64)
        assert np.array_equal(w, vals.astype(np.float64) * 2.0 ** e)
        assert np.array_equal(x, vals.astype(np.float64) * 2.0 ** -e)


def test_smoothing_balances_channel_maxima(oracle):
    """The factor makes the largest smoothed activation and the largest
    smoothed weight of each channel equal (both sqrt(ax * aw)), up to the
    FP16 roundings, and leaves each channel's balance point at the geometric
    mean -- the migration of difficulty with strength 0.5."""
    L = si.LLAMA3_8B_QKV
    Xc = si.activations(L, 16, seed=3)[:, :512]
    W = si.weights(L, seed=0)[:256, :512]
    s = oracle.smooth_factors(Xc, W)
    Xp = oracle.smooth_act(Xc, s).astype(np.float64)
    Wp = oracle.smooth_weights(W, s).astype(np.float64)
    mx = np.abs(Xp).max(0)
    mw = np.abs(Wp).max(0)
    geo = np.sqrt(np.abs(Xc.astype(np.float64)).max(0) * np.abs(W.astype(np.float64)).max(0))
    assert np.all(np.abs(np.log(mx / mw)) <= 4 * 2.0 ** -10)
    assert np.all(np.abs(np.log(mx / geo)) <= 3 * 2.0 ** -10)
    # the outlier channels of the activation recipe get the largest factors
    ax = np.abs(Xc.astype(np.float64)).max(0)
    top = np.argsort(ax)[-5:]
    assert np.all(s.astype(np.float64)[top] > np.median(s.astype(np.float64)))


def test_smoothing_keeps_the_product(oracle):
    """X' . W'^T equals X . W^T up to the FP16 roundings of the smoothed
    operands: every term x_k w_k moves by at most 2^-10 of |x_k w_k|
    (one rounding on each side, each at most 2^-11 relative)."""
    rng = np.random.default_rng(11)
    X = rng.standard_normal((5, 96)).astype(np.float16)
    X[:, 7] *= np.float16(30)
    W = (rng.standard_normal((6, 96)) * 0.02).astype(np.float16)
    s = oracle.smooth_factors(X, W)
    Xp = oracle.smooth_act(X, s).astype(np.float64)
    Wp = oracle.smooth_weights(W, s).astype(np.float64)
    Xd, Wd = X.astype(np.float64), W.astype(np.float64)
    diff = np.abs(Xp @ Wp.T - Xd @ Wd.T)
    bound = (np.abs(Xd) @ np.abs(Wd).T) * (2.0 ** -10 + 2.0 ** -20)
    assert np.all(diff <= bound)


def test_smoothing_moves_outliers_from_activations_to_weights(oracle):
    """What the page states the method does: the activations' channel
    maxima become flatter (the recipe's x20 outlier channels shrink to about
    sqrt(20) of the typical channel) while the weights' channel maxima
    spread by the same factor."""
    L = si.LLAMA3_8B_QKV
    K, N = 1024, 256
    W = si.weights(L, seed=0)[:N, :K]
    X = si.activations(L, 64, seed=4)[:, :K]
    s = oracle.smooth_factors(X, W)

    def spread(a):
        m = np.abs(a.astype(np.float64)).max(0)
        return m.max() / np.median(m)
    rx, rxs = spread(X), spread(oracle.smooth_act(X, s))
    rw, rws = spread(W), spread(oracle.smooth_weights(W, s))
    assert rx > 10 and rxs < rx / 2
    assert rws > rw
    assert abs(np.log(rxs / np.sqrt(rx * rw))) < np.log(2)


# ---------------------------------------------------------------------------
# SiLU(gate) * up (the step between the gate_up and down projections)
# ---------------------------------------------------------------------------

def test_silu_mul_hand_examples(oracle):
    for (g, u), (hh,) in _golden("silu_mul"):
        h = oracle.silu_mul(np.array([float(g)], np.float16), np.array([float(u)], np.float16))
        assert h.view(np.uint16)[0] == int(hh, 16), (g, u, h)


def test_silu_odd_part_is_the_identity(oracle):
    """silu(x) - silu(-x) = x exactly (sigma(x) + sigma(-x) = 1), so with
    u = 1 the two FP16 results differ by x up to their two roundings."""
    g = np.random.default_rng(2).uniform(-12, 12, 4000).astype(np.float16)
    one = np.ones_like(g)
    hp = oracle.silu_mul(g, one).astype(np.float64)
    hn = oracle.silu_mul(-g, one).astype(np.float64)
    ulp = np.spacing(np.abs(hp).astype(np.float16)).astype(np.float64) + \
        np.spacing(np.abs(hn).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs((hp - hn) - g.astype(np.float64)) <= ulp)


def test_silu_limits_and_linearity_in_up(oracle):
    g = np.array([30.0, 60.0, -30.0, -60.0], np.float16)
    u = np.array([1.5, -2.0, 3.0, 1.0], np.float16)
    h = oracle.silu_mul(g, u).astype(np.float64)
    assert h[0] == 45.0 and h[1] == -120.0          # silu(x) = x for large x
    assert abs(h[2]) <= 2.0 ** -24 and h[3] == 0.0  # vanishes for very negative x
    # scaling up by a power of two scales h exactly (away from under/overflow)
    g2 = np.random.default_rng(4).uniform(-6, 6, 500).astype(np.float16)
    u2 = np.random.default_rng(5).uniform(0.5, 2, 500).astype(np.float16)
    a = oracle.silu_mul(g2, u2).astype(np.float64)
    b = oracle.silu_mul(g2, (u2.astype(np.float64) * 4).astype(np.float16)).astype(np.float64)
    keep = np.abs(a) > 2.0 ** -12
    assert np.array_equal(b[keep], 4 * a[keep])


# ---------------------------------------------------------------------------
# 4-bit KV cache and decode attention over it ("QServe: Cuantificación
# W4A8KV4 ...", abstract: the 4-bit KV cache; velog notes, Insight: the fused,
# memory-bound attention).  The cache format is a reading: x^ = s * q + m per
# (token, KV head) vector, q = clamp(rne((x - min) / s), 0, 15).
# ---------------------------------------------------------------------------

def test_kv4_hand_examples(oracle):
    for x, q, sm in _golden("kv4_quant"):
        X = np.array([float(v) for v in x], np.float16)[None, :]
        qq, s, m = oracle.kv4_quant(X)
        assert qq[0].tolist() == [int(v) for v in q], x
        assert int(s.view(np.uint16)[0]) == int(sm[0], 16), x
        assert int(m.view(np.uint16)[0]) == int(sm[1], 16), x


def test_kv4_codes_are_the_nearest_level(oracle):
    """Brute force over the 16 levels: every code is the level nearest to x
    (ties aside), the minimum gets code 0, and |x - x^| <= s / 2 where s is
    a normal FP16 number."""
    rng = np.random.default_rng(11)
    X = (rng.standard_normal((400, 8)) * rng.choice([0.01, 1.0, 30.0], (400, 1))).astype(np.float16)
    q, s, m = oracle.kv4_quant(X)
    assert q.max() <= 15
    xh = oracle.kv4_dequant(q, s, m)
    x = X.astype(np.float64)
    sv = s.astype(np.float64)[:, None]
    levels = sv[:, :, None] * np.arange(16)[None, None, :] + m.astype(np.float64)[:, None, None]
    dist = np.abs(x[:, :, None] - levels)
    best = dist.min(axis=2)
    own = np.abs(x - xh)
    assert np.all(own <= best * (1 + 1e-6) + 1e-30)
    assert np.all(q[np.arange(400), x.argmin(axis=1)] == 0)
    normal = sv[:, 0] >= 2.0 ** -14
    assert np.all(own[normal] <= 0.5 * sv[normal] * (1 + 2.0 ** -10))


def _attn_inputs(oracle, rng, B, Hq, Hkv, L, d):
    Q = rng.standard_normal((B, Hq, d)).astype(np.float16)
    K = rng.standard_normal((B, Hkv, L, d)).astype(np.float16)
    V = rng.standard_normal((B, Hkv, L, d)).astype(np.float16)
    qk, sk, mk = oracle.kv4_quant(K)
    qv, sv, mv = oracle.kv4_quant(V)
    return Q, [qk, sk, mk, qv, sv, mv]


def test_kv4_attention_single_token_returns_its_value(oracle):
    """softmax over one token is 1: out = v^ exactly."""
    rng = np.random.default_rng(1)
    Q, c = _attn_inputs(oracle, rng, 2, 4, 2, 5, 16)
    out, out64 = oracle.kv4_decode_attention(Q, *c, np.array([1, 1], np.int32))
    vh = oracle.kv4_dequant(c[3], c[4], c[5])
    for h in range(4):
        assert np.array_equal(out64[:, h], vh[:, h // 2, 0])


def test_kv4_attention_equal_keys_average_the_values(oracle):
    rng = np.random.default_rng(2)
    Q, c = _attn_inputs(oracle, rng, 1, 2, 1, 7, 16)
    for a in c[:3]:
        a[:, :, 1:] = a[:, :, :1]            # every key equal to the first
    out, out64 = oracle.kv4_decode_attention(Q, *c, np.array([7], np.int32))
    vh = oracle.kv4_dequant(c[3], c[4], c[5])
    ref = vh[0, 0].mean(axis=0)
    for h in range(2):
        assert np.allclose(out64[0, h], ref, rtol=1e-12, atol=1e-12)


def test_kv4_attention_two_tokens_logistic(oracle):
    """Keys 0 and e_0 (d = 4), values 0 and 3 e_0: the weight of the second
    token is the logistic function of q_0 / sqrt(4)."""
    d, L = 4, 2
    qk = np.zeros((1, 1, L, d), np.uint8)
    qk[0, 0, 1, 0] = 1
    qv = np.zeros((1, 1, L, d), np.uint8)
    qv[0, 0, 1, 0] = 3
    one = np.full((1, 1, L), 1.0, np.float16)
    zero = np.zeros((1, 1, L), np.float16)
    for a in (0.75, -2.0, 5.5):
        Q = np.array([[[a, 0.3, -1, 2]]], np.float16)
        out, out64 = oracle.kv4_decode_attention(Q, qk, one, zero, qv, one, zero,
                                                 np.array([2], np.int32))
        p1 = 1.0 / (1.0 + math.exp(-float(np.float16(a)) / 2.0))
        assert abs(out64[0, 0, 0] - 3.0 * p1) <= 1e-12
        assert np.all(out64[0, 0, 1:] == 0.0)


def test_kv4_attention_grouped_heads(oracle):
    """Query heads 0, 1 read KV head 0 and heads 2, 3 read KV head 1: with
    every value of a KV head equal to a constant, its query heads return it."""
    rng = np.random.default_rng(3)
    Q, c = _attn_inputs(oracle, rng, 1, 4, 2, 6, 16)
    c[3][:] = 0                                 # codes 0: v^ = m
    c[5][0, 0, :] = 1.5
    c[5][0, 1, :] = -0.25
    out, out64 = oracle.kv4_decode_attention(Q, *c, np.array([6], np.int32))
    assert np.allclose(out64[0, :2], 1.5, rtol=1e-14, atol=0)
    assert np.allclose(out64[0, 2:], -0.25, rtol=1e-14, atol=0)


def test_kv4_attention_masks_tokens_past_the_length(oracle):
    rng = np.random.default_rng(4)
    Q, c = _attn_inputs(oracle, rng, 3, 2, 2, 9, 16)
    seq = np.array([9, 4, 0], np.int32)
    out_a, a64 = oracle.kv4_decode_attention(Q, *c, seq)
    for arr in c:
        arr[1, :, 4:] = arr[1, :, 4:][..., ::-1] if arr.ndim == 4 else arr[1, :, 4:] * 3
    out_b, b64 = oracle.kv4_decode_attention(Q, *c, seq)
    assert np.array_equal(a64, b64)
    assert np.all(a64[2] == 0.0) and np.all(out_a.view(np.uint16)[2] == 0)


def test_kv4_attention_invariances(oracle):
    """Shifting every key by the same vector t * 1 shifts all scores of a head
    alike (softmax unchanged); permuting the tokens changes nothing; shifting
    every value by t shifts the output by t."""
    rng = np.random.default_rng(5)
    Q, c = _attn_inputs(oracle, rng, 2, 4, 1, 11, 16)
    seq = np.array([11, 8], np.int32)
    _, base = oracle.kv4_decode_attention(Q, *c, seq)
    c2 = [a.copy() for a in c]
    c2[2] = (c2[2].astype(np.float64) + 0.5).astype(np.float16)
    _, shifted = oracle.kv4_decode_attention(Q, *c2, seq)
    assert np.allclose(shifted, base, rtol=0, atol=1e-9)
    perm = rng.permutation(8)
    c3 = [a.copy() for a in c]
    for a in c3:
        a[1, :, :8] = a[1][:, perm]
    _, permuted = oracle.kv4_decode_attention(Q, *c3, seq)
    assert np.allclose(permuted, base, rtol=0, atol=1e-12)
    c4 = [a.copy() for a in c]
    c4[5] = (c4[5].astype(np.float64) + 2.0).astype(np.float16)
    exact = np.all(c4[5].astype(np.float64) == c[5].astype(np.float64) + 2.0)
    assert exact
    _, vshift = oracle.kv4_decode_attention(Q, *c4, seq)
    assert np.allclose(vshift, base + 2.0, rtol=0, atol=1e-9)
