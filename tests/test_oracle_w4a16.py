"""Pins for oracle.w4a16 (the W4A16 layer: 4-bit NVFP4 weights, 16-bit
activations, an activation-aware per-channel scale s): exact cases where
quantization loses nothing, the quantizer's error bound, a pure-Python brute
force, and planted mistakes."""

import numpy as np
import pytest

import bruteforce as BF
from oracle import formats as F
from oracle import svdquant as S
from oracle import w4a16 as W4


def _grid_weights(N, K, seed, scale_pow=0):
    # every 16-block holds E2M1 grid values times 448 * 2^p, with one 6 per
    # block, so g = 2^p, every block scale is 448 and nothing is rounded
    g = np.random.default_rng(seed)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    W = grid[g.integers(0, 8, (N, K))] * np.where(g.random((N, K)) < 0.5, -1.0, 1.0)
    W[:, ::16] = 6.0
    return (W * 448.0 * 2.0 ** scale_pow).astype(np.float32)


def _f16_exact_x(M, K, seed):
    # values exactly representable in f16 (and bf16): 8 significant bits, no tiny magnitudes
    X = np.random.default_rng(seed).standard_normal((M, K)).astype(np.float32)
    X = np.where(np.abs(X) < 1e-2, np.float32(0.0), X).astype(np.float16).astype(np.float32)
    return (np.round(X * 64.0) / 64.0).astype(np.float32)


def test_exact_weights_give_the_exact_product():
    W = _grid_weights(24, 64, seed=1, scale_pow=-12)
    X = _f16_exact_x(5, 64, seed=2)
    L = W4.prepare(W)
    assert L.g == np.float32(2.0 ** -12)
    assert np.all(L.scales == F.e4m3_encode(np.float32(448.0)))
    np.testing.assert_array_equal(np.float64(L.g) * L.deq, W.astype(np.float64))
    np.testing.assert_allclose(W4.linear(L, X), X.astype(np.float64) @ W.T.astype(np.float64), rtol=1e-12,
                               atol=1e-12)


def test_power_of_two_channel_scales_cancel():
    # W' = W diag(s) and X diag(s)^-1 with s a power of two per channel: the
    # grid weights become W' = W s, still exact; Y must equal X W^T
    K = 64
    s = (2.0 ** np.random.default_rng(3).integers(-3, 4, K)).astype(np.float32)
    Wp = _grid_weights(16, K, seed=4, scale_pow=-10)
    W = (Wp / s[None, :]).astype(np.float32)
    X = _f16_exact_x(3, K, seed=5)
    L = W4.prepare(W, s=s)
    np.testing.assert_array_equal(np.float64(L.g) * L.deq, Wp.astype(np.float64))
    np.testing.assert_allclose(W4.linear(L, X), X.astype(np.float64) @ W.T.astype(np.float64), rtol=1e-12,
                               atol=1e-12)


def test_error_within_half_a_grid_step_per_weight():
    g = np.random.default_rng(6)
    W = (g.standard_normal((32, 128)) * 0.02).astype(np.float32)
    X = g.standard_normal((4, 128)).astype(np.float32)
    L = W4.prepare(W)
    wq = np.float64(L.g) * L.deq
    # E2M1 steps are at most 2 (between 4 and 6) in units of the block's d = scale * g
    d = np.repeat(F.e4m3_decode(L.scales).astype(np.float64), 16, axis=1) * np.float64(L.g)
    assert np.all(np.abs(wq - W) <= 1.0 * d + 1e-30)
    bound = np.abs(X).astype(np.float64) @ (1.0 * d).T
    assert np.all(np.abs(W4.linear(L, X) - X.astype(np.float64) @ W.T.astype(np.float64)) <= bound + 1e-12)


@pytest.mark.parametrize("seed,with_s,with_bias", [(0, False, False), (1, True, False), (2, True, True)])
def test_matches_brute_force(seed, with_s, with_bias):
    g = np.random.default_rng(seed)
    N, K, M = 6, 32, 3
    W = (g.standard_normal((N, K)) * 0.05).astype(np.float32)
    X = g.standard_normal((M, K)).astype(np.float32)
    s = (0.5 + g.random(K)).astype(np.float32) if with_s else np.ones(K, np.float32)
    b = g.standard_normal(N) * 0.01 if with_bias else None
    want = BF.w4a16_forward(W.tolist(), X.tolist(), s.tolist(), None if b is None else b.tolist())
    L = W4.prepare(W, s=s if with_s else None, bias=b)
    assert L.g == np.float32(want["g"])
    np.testing.assert_array_equal(L.codes, np.array(want["codes"]))
    np.testing.assert_array_equal(L.scales, np.array(want["scales"]))
    np.testing.assert_allclose(W4.linear(L, X), np.array(want["Y"]), rtol=1e-12, atol=1e-12)


def test_activation_operand_rounds_to_f16_and_saturates():
    x = np.array([[1.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 7e4, -1e6, 2.0 ** -25, 3 * 2.0 ** -25]],
                 np.float32)
    got = W4.act_operand(x, np.ones(x.shape[1], np.float32)).astype(np.float64)[0]
    np.testing.assert_array_equal(got, [1.0, 1.0, 1.0 + 2.0 ** -9, 65504.0, -65504.0, 0.0, 2.0 ** -23])
    for v in x[0]:  # the brute force's rounding agrees
        assert BF.f16r(float(v)) == float(W4.act_operand(np.array([[v]], np.float32), np.ones(1, np.float32))[0, 0])


def test_rejects_bad_scales_and_shapes():
    with pytest.raises(ValueError):
        W4.prepare(np.zeros((4, 20), np.float32))
    with pytest.raises(ValueError):
        W4.prepare(np.zeros((4, 32), np.float32), s=np.zeros(32, np.float32))


# ------------------------------------------------------------------ mutations


def _pins_fail():
    failed = 0
    for t in (test_exact_weights_give_the_exact_product, test_power_of_two_channel_scales_cancel,
              lambda: test_matches_brute_force(2, True, True)):
        try:
            t()
        except AssertionError:
            failed += 1
    return failed


def _linear_times_s(layer, X, rows=None):  # multiplies by s instead of dividing
    Xt = W4.act_operand(X, 1.0 / layer.inv_s).astype(np.float64)
    return np.float64(layer.g) * (Xt @ layer.deq.T) + (0 if layer.bias is None else layer.bias[None, :])


def _linear_no_g(layer, X, rows=None):
    Xt = W4.act_operand(X, layer.inv_s).astype(np.float64)
    return Xt @ layer.deq.T + (0 if layer.bias is None else layer.bias[None, :])


def _linear_no_bias(layer, X, rows=None):
    Xt = W4.act_operand(X, layer.inv_s).astype(np.float64)
    return np.float64(layer.g) * (Xt @ layer.deq.T)


@pytest.mark.parametrize("fn", [_linear_times_s, _linear_no_g, _linear_no_bias])
def test_planted_mistakes_are_caught(monkeypatch, fn):
    monkeypatch.setattr(W4, "linear", fn)
    assert _pins_fail() >= 1


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(N=st.integers(1, 5), kb=st.integers(1, 3), M=st.integers(1, 3), seed=st.integers(0, 10_000),
       with_s=st.booleans(), with_bias=st.booleans(), wscale=st.sampled_from([1e-3, 0.05, 20.0]))
def test_matches_brute_force_on_random_layers(N, kb, M, seed, with_s, with_bias, wscale):
    K = 16 * kb
    g = np.random.default_rng(seed)
    W = (g.standard_normal((N, K)) * wscale).astype(np.float32)
    X = g.standard_normal((M, K)).astype(np.float32)
    s = (0.25 + 2 * g.random(K)).astype(np.float32) if with_s else np.ones(K, np.float32)
    b = g.standard_normal(N) * 0.01 if with_bias else None
    want = BF.w4a16_forward(W.tolist(), X.tolist(), s.tolist(), None if b is None else b.tolist())
    L = W4.prepare(W, s=s if with_s else None, bias=b)
    np.testing.assert_array_equal(L.codes, np.array(want["codes"]))
    np.testing.assert_array_equal(L.scales, np.array(want["scales"]))
    np.testing.assert_allclose(W4.linear(L, X), np.array(want["Y"]), rtol=1e-11, atol=1e-11)
