"""Pins for oracle.int4 (the INT4 variant of the SVDQuant layer): exact cases where
quantization loses nothing, the rounding rule on ties, the group layout, the
quantizer's error bound, a pure-Python brute force of the whole layer, and
planted mistakes that the pins must catch."""

import numpy as np
import pytest

import bruteforce as BF
from oracle import formats as F
from oracle import int4 as I4
from oracle import svdquant as S


def _grid_rows(rows, K, seed, exp_lo=-6, exp_hi=3):
    # every group of 64 holds integers -7..7 (one +-7 per group) times a power of two
    # per group: nothing is rounded by the quantizer and the scale is that power of two
    g = np.random.default_rng(seed)
    q = g.integers(-7, 8, (rows, K))
    q[:, ::64] = np.where(g.random((rows, K // 64)) < 0.5, -7, 7)
    p = 2.0 ** g.integers(exp_lo, exp_hi, (rows, K // 64))
    return (q * np.repeat(p, 64, axis=1)).astype(np.float32), q, p


def test_grid_values_are_kept_exactly():
    t, q, p = _grid_rows(5, 192, seed=1)
    codes, sb = I4.int4_quantize(t)
    np.testing.assert_array_equal(codes, q)
    np.testing.assert_array_equal(F.bf16_from_bits(sb), p.astype(np.float32))
    np.testing.assert_array_equal(I4.int4_dequantize(codes, sb), t.astype(np.float64))


def test_ties_round_to_even_and_zero_groups_stay_zero():
    # amax 7 -> s = 1: the halves are ties
    row = np.zeros(128, np.float32)
    row[:10] = [7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, 6.5, -6.5]
    codes, sb = I4.int4_quantize(row[None, :])
    np.testing.assert_array_equal(codes[0, :10], [7, 0, 2, 2, 0, -2, -2, 4, 6, -6])
    assert F.bf16_from_bits(sb)[0, 0] == 1.0
    assert sb[0, 1] == 0 and np.all(codes[0, 64:] == 0)  # the all-zero group


def test_scale_rounding_never_pushes_a_code_past_7():
    # amax / 7 rounded down to bf16 makes amax / s slightly above 7: still code 7
    g = np.random.default_rng(2)
    t = (g.standard_normal((64, 64)) * np.exp(g.uniform(-20, 20, (64, 1)))).astype(np.float32)
    codes, sb = I4.int4_quantize(t)
    assert codes.min() >= -7 and codes.max() <= 7
    s = F.bf16_from_bits(sb).astype(np.float64)
    rounded_down = s < np.max(np.abs(t), axis=1, keepdims=True) / 7.0
    assert rounded_down.any()  # the case occurs in this sample
    np.testing.assert_array_equal(np.abs(codes[np.arange(64), np.argmax(np.abs(t), axis=1)]), 7)


def test_groups_are_64_consecutive_elements_of_a_row():
    t, _, _ = _grid_rows(2, 256, seed=3)
    t2 = t.copy()
    t2[0, 64:128] *= 1024.0  # a large group leaves its neighbours' scales alone
    _, s1 = I4.int4_quantize(t)
    _, s2 = I4.int4_quantize(t2)
    assert s2[0, 1] != s1[0, 1]
    np.testing.assert_array_equal(np.delete(s2, 1, axis=1), np.delete(s1, 1, axis=1))


def test_error_within_half_a_step():
    g = np.random.default_rng(4)
    t = (g.standard_normal((8, 320)) * 3.0).astype(np.float32)
    codes, sb = I4.int4_quantize(t)
    s = np.repeat(F.bf16_from_bits(sb).astype(np.float64), 64, axis=1)
    err = np.abs(I4.int4_dequantize(codes, sb) - t.astype(np.float64))
    # half a step, plus the float32 rounding of t * (1 / s) (relative 2^-23 of at most 7.03)
    assert np.all(err <= s * (0.5 + 2.0 ** -20))


def test_matches_brute_force_quantizer():
    g = np.random.default_rng(5)
    t = (g.standard_normal((3, 128)) * np.array([[1e-3], [1.0], [300.0]])).astype(np.float32)
    codes, sb = I4.int4_quantize(t)
    want_c, want_s = BF.int4_quantize_rows(t.astype(np.float64).tolist())
    np.testing.assert_array_equal(codes, np.array(want_c))
    np.testing.assert_array_equal(F.bf16_from_bits(sb).astype(np.float64), np.array(want_s))


def _exact_layer_inputs(M, N, K, seed):
    # lambda = 1 (equal column maxima of X and W) and both operands on the INT4 grid:
    # the rank-0 layer is then lossless and Y = X W^T exactly
    X, _, _ = _grid_rows(M, K, seed, exp_lo=-2, exp_hi=2)
    W, _, _ = _grid_rows(N, K, seed + 1, exp_lo=-8, exp_hi=-4)
    X[0, :] = 7.0 * 2.0 ** 1  # the column maxima ...
    W[0, :] = 7.0 * 2.0 ** 1  # ... are equal, so lambda_j = 1
    return X, W


def test_lossless_operands_give_the_exact_product():
    X, W = _exact_layer_inputs(4, 12, 128, seed=6)
    amax = np.max(np.abs(X), axis=0).astype(np.float32)
    L = I4.prepare(W, amax, 0)
    assert np.all(L.lam == 1.0)
    y = I4.forward(L, X)
    np.testing.assert_array_equal(y, X.astype(np.float64) @ W.T.astype(np.float64))


def test_error_bound_of_section_4_1():
    g = np.random.default_rng(7)
    M, N, K = 6, 16, 128
    X = g.standard_normal((M, K)).astype(np.float32)
    W = (g.standard_normal((N, K)) * 0.05).astype(np.float32)
    L = I4.prepare(W, np.max(np.abs(X), axis=0).astype(np.float32), 0)
    act = I4.quantize_act(L, X)
    qx = I4.int4_dequantize(act.codes, act.scales)
    xh = act.x_hat.astype(np.float64)
    what = L.R.T  # W_hat (rank 0: R^T = W diag(lambda))
    bound = S.error_bound(xh, what.T, qx, L.deq_w.T)
    assert S.quant_error(xh @ what.T, I4.linear(L, act)) <= bound


@pytest.mark.parametrize("rank,with_bias,gelu", [(0, False, False), (4, True, False), (8, True, True)])
def test_matches_brute_force_layer(rank, with_bias, gelu):
    g = np.random.default_rng(10 + rank)
    M, N, K = 3, 5, 128
    W = (g.standard_normal((N, K)) * 0.05).astype(np.float32)
    W = F.bf16(W)
    X = F.bf16(g.standard_normal((M, K)).astype(np.float32) * 2.0)
    X[:, 7] *= 20.0  # an outlier channel for the smoothing to move
    amax = np.max(np.abs(X), axis=0).astype(np.float32)
    L1 = F.bf16(g.standard_normal((K, rank)).astype(np.float32) * 0.1).astype(np.float64)
    L2 = F.bf16(g.standard_normal((rank, N)).astype(np.float32) * 0.1).astype(np.float64)
    b = F.bf16(g.standard_normal(N).astype(np.float32) * 0.1).astype(np.float64) if with_bias else None
    L = I4.prepare(W, amax, rank, bias=b, factors=(L1, L2))
    want = BF.int4_layer_forward(W.astype(np.float64).tolist(), X.astype(np.float64).tolist(), amax.tolist(),
                                 L1.tolist(), L2.tolist(), None if b is None else b.tolist(), gelu)
    np.testing.assert_array_equal(L.lam, np.array(want["lam"], np.float32))
    np.testing.assert_array_equal(L.w_codes, np.array(want["w_codes"]))
    np.testing.assert_array_equal(F.bf16_from_bits(L.w_scales).astype(np.float64), np.array(want["w_scales"]))
    act = I4.quantize_act(L, X)
    np.testing.assert_array_equal(act.codes, np.array(want["a_codes"]))
    np.testing.assert_array_equal(F.bf16_from_bits(act.scales).astype(np.float64), np.array(want["a_scales"]))
    np.testing.assert_allclose(act.lr, np.array(want["lr"]), rtol=1e-12, atol=1e-12)
    y = I4.linear(L, act, S.EPI_GELU_TANH if gelu else S.EPI_NONE)
    np.testing.assert_allclose(y, np.array(want["Y"]), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ mutations


def _pins_fail():
    failed = 0
    for t in (test_grid_values_are_kept_exactly, test_ties_round_to_even_and_zero_groups_stay_zero,
              test_groups_are_64_consecutive_elements_of_a_row, test_matches_brute_force_quantizer,
              test_lossless_operands_give_the_exact_product, lambda: test_matches_brute_force_layer(4, True, False)):
        try:
            t()
        except AssertionError:
            failed += 1
    return failed


_orig_quantize = I4.int4_quantize


def _q_max_8(t):  # scales from amax / 8
    t = np.asarray(t, np.float32)
    rows, k = t.shape
    g = t.reshape(rows, k // 64, 64)
    sb = F.bf16_bits((np.max(np.abs(g), axis=2) / np.float32(8)).astype(np.float32))
    s = F.bf16_from_bits(sb)
    rcp = np.where(s == 0, 0, 1 / np.where(s == 0, 1, s)).astype(np.float32)
    q = np.clip(np.rint((g * rcp[..., None]).astype(np.float32)), -7, 7).astype(np.int8)
    return q.reshape(rows, k), sb


def _floor_rounding(t):
    codes, sb = _orig_quantize(t)
    t = np.asarray(t, np.float32)
    rows, k = t.shape
    s = np.repeat(F.bf16_from_bits(sb), 64, axis=1)
    rcp = np.where(s == 0, 0, 1 / np.where(s == 0, 1, s)).astype(np.float32)
    return np.clip(np.floor((t * rcp).astype(np.float32) + 0.5), -7, 7).astype(np.int8), sb


def _groups_of_16(t):
    t = np.asarray(t, np.float32)
    rows, k = t.shape
    g = t.reshape(rows, k // 16, 16)
    sb16 = F.bf16_bits((np.max(np.abs(g), axis=2) / np.float32(7)).astype(np.float32))
    s = F.bf16_from_bits(sb16)
    rcp = np.where(s == 0, 0, 1 / np.where(s == 0, 1, s)).astype(np.float32)
    q = np.clip(np.rint((g * rcp[..., None]).astype(np.float32)), -7, 7).astype(np.int8)
    return q.reshape(rows, k), sb16[:, ::4]


def _linear_drops_low_rank(layer, act, epilogue=0, rows=None):
    y = I4.int4_dequantize(act.codes, act.scales) @ layer.deq_w.T
    return y + (0 if layer.bias is None else layer.bias[None, :])


@pytest.mark.parametrize("fn", [_q_max_8, _floor_rounding, _groups_of_16])
def test_planted_quantizer_mistakes_are_caught(monkeypatch, fn):
    monkeypatch.setattr(I4, "int4_quantize", fn)
    assert _pins_fail() >= 1


def test_planted_linear_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(I4, "linear", _linear_drops_low_rank)
    assert _pins_fail() >= 1
