"""Pins for the fused MLP pair of the oracle (oracle.svdquant.mlp_pair).

The pair is fc1 (tanh-GELU epilogue) whose bf16 output feeds fc2's activation quantization
(Diffusers/Nunchaku page, the fused GELU/MLP path).  Pinned against the pure-Python brute force
of both layers on tiny shapes, with the hidden state rounded to bf16 in between, and against
planted mistakes: a pair that skips the bf16 rounding of the hidden state, or quantizes it under
fc1's smoothing instead of fc2's, must fail the pin."""

import numpy as np
import pytest

import bruteforce as BF
from bit_w4a4_quantized_b200 import workloads as WL
from oracle import formats as F
from oracle import svdquant as S


def _factors(W, amax, r):
    lam, _ = S.smoothing_factors(amax, np.max(np.abs(W), 0))
    if not r:
        return np.zeros((W.shape[1], 0)), np.zeros((0, W.shape[0]))
    l1, l2, _ = S.low_rank_factors(lam.astype(np.float64)[:, None] * W.T.astype(np.float64), r)
    return S.bf16_from_f64(l1), S.bf16_from_f64(l2)


def _pair_case(M, K1, N1, N2, r, seed):
    X = WL.make_x(M, K1, seed=seed, n_outlier=2).astype(np.float32)
    W1 = WL.make_w(N1, K1, seed=seed, n_outlier=2).astype(np.float32)
    W2 = WL.make_w(N2, N1, seed=seed + 1, n_outlier=0).astype(np.float32)
    b1 = WL.make_bias(N1, seed).astype(np.float64)
    amax1 = np.max(np.abs(X), axis=0)
    f1 = _factors(W1, amax1, r)
    fc1 = S.prepare(W1, amax1, r, bias=b1, factors=f1)
    # fc2 is calibrated on the hidden state it will see (the oracle's own fc1 output)
    h_cal = S.bf16_from_f64(S.forward(fc1, X, S.EPI_GELU_TANH)).astype(np.float32)
    amax2 = np.max(np.abs(h_cal), axis=0)
    f2 = _factors(W2, amax2, r)
    fc2 = S.prepare(W2, amax2, r, factors=f2)
    return X, W1, W2, b1, amax1, amax2, f1, f2, fc1, fc2


def check_pair_against_bruteforce(M, K1, N1, N2, r, seed):
    X, W1, W2, b1, amax1, amax2, f1, f2, fc1, fc2 = _pair_case(M, K1, N1, N2, r, seed)
    h, act2, y = S.mlp_pair(fc1, fc2, X)
    ref1 = BF.layer_forward(W1.tolist(), X.tolist(), amax1.tolist(), f1[0].tolist(), f1[1].tolist(), b1.tolist(),
                            gelu=True)
    h_bf = [[BF.bf16r(v) for v in row] for row in ref1["Y"]]
    ref2 = BF.layer_forward(W2.tolist(), h_bf, amax2.tolist(), f2[0].tolist(), f2[1].tolist(), None, gelu=False)
    assert h.astype(np.float64).tolist() == h_bf
    assert act2.x_hat.astype(np.float64).tolist() == ref2["x_hat"]
    assert act2.codes.tolist() == ref2["a_codes"]
    assert act2.scales.tolist() == ref2["a_scales"]
    lr = np.array(ref2["lr"]) if r else np.zeros((M, 0))
    np.testing.assert_allclose(act2.lr, lr, rtol=1e-12, atol=1e-12 * max(np.abs(lr).max(initial=0), 1e-300))
    yr = np.array(ref2["Y"])
    np.testing.assert_allclose(y, yr, rtol=1e-12, atol=1e-12 * np.abs(yr).max())


@pytest.mark.parametrize("M,K1,N1,N2,r", [(3, 32, 48, 5, 2), (2, 16, 32, 4, 0), (4, 48, 64, 3, 3)])
def test_pair_matches_bruteforce(M, K1, N1, N2, r):
    check_pair_against_bruteforce(M, K1, N1, N2, r, seed=M + K1 + N1)


def test_pair_is_the_composition_of_the_two_layers():
    """mlp_pair is fc2's forward on fc1's bf16 GELU output, on a workload-shaped case."""
    X, W1, W2, b1, amax1, amax2, f1, f2, fc1, fc2 = _pair_case(16, 256, 512, 256, 16, seed=9)
    h, act2, y = S.mlp_pair(fc1, fc2, X)
    np.testing.assert_array_equal(h, S.bf16_from_f64(S.forward(fc1, X, S.EPI_GELU_TANH)).astype(np.float32))
    np.testing.assert_array_equal(y, S.forward(fc2, h))
    assert np.max(np.abs(h)) > 0 and np.any(act2.codes != 0)


ORIG_BF16 = S.bf16_from_f64
ORIG_QUANT = S.quantize_act


def _mut_no_rounding(x):
    return np.asarray(x, dtype=np.float64)


def test_planted_mistake_unrounded_hidden_state_is_caught(monkeypatch):
    monkeypatch.setattr(S, "bf16_from_f64", _mut_no_rounding)
    with pytest.raises(AssertionError):
        check_pair_against_bruteforce(3, 32, 48, 5, 2, seed=83)


def test_planted_mistake_wrong_smoothing_is_caught(monkeypatch):
    """fc2 quantizing h with every smoothing factor 1 instead of its own: the codes differ from
    the brute force.  Only fc2's call is changed (fc2's input width is fc1's N1 = 48 here)."""
    def mutant(layer, X):
        if layer.inv_lam.shape[0] != 48:
            return ORIG_QUANT(layer, X)
        orig_inv = layer.inv_lam
        try:
            layer.inv_lam = np.ones_like(orig_inv)
            return ORIG_QUANT(layer, X)
        finally:
            layer.inv_lam = orig_inv

    monkeypatch.setattr(S, "quantize_act", mutant)
    with pytest.raises(AssertionError):
        check_pair_against_bruteforce(3, 32, 48, 5, 2, seed=83)


from gpu_cases import PAIR_TOL  # noqa: E402  (the GPU pair against the oracle's pair, max-norm)


def test_pair_output_moves_with_last_ulp_changes_of_the_hidden_state():
    """Why the composed pair gets a wider bound against the oracle than one layer does: fc2's
    4-bit quantizer turns one-ulp changes of the bf16 hidden state into whole-code flips.  Moving
    5-50 % of the hidden values by one ulp (what a float32 GPU with a hardware tanh does to the
    float64 oracle's hidden state) moves the oracle's own pair output by a few percent of its max;
    the GPU tests' pair bound PAIR_TOL sits above every case measured here."""
    g = np.random.default_rng(0)
    worst = 0.0
    for (M, K1, N1, N2, r) in [(64, 256, 640, 256, 16), (48, 512, 512, 320, 0)]:
        X, W1, W2, b1, amax1, amax2, f1, f2, fc1, fc2 = _pair_case(M, K1, N1, N2, r, seed=N1 + r)
        h, _, y = S.mlp_pair(fc1, fc2, X)
        bits = F.bf16_bits(h).astype(np.int32)
        for frac in (0.05, 0.2, 0.5):
            flip = (g.random(h.shape) < frac) & ((bits & 0x7FFF) != 0)
            step = np.where(g.random(h.shape) < 0.5, 1, -1)
            hp = F.bf16_from_bits(np.where(flip, bits + step, bits).astype(np.uint16))
            err = S.max_rel_err(S.forward(fc2, hp), y)
            assert err > 1e-3  # the flips do reach the output
            worst = max(worst, err)
    assert worst < PAIR_TOL, worst
