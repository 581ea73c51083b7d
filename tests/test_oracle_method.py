"""Pins for oracle.svdquant: closed forms, LAPACK cross-checks, the page's
worked example, a pure-Python brute force on tiny shapes, the error bound of
section 4.1 and the qualitative claims of section 4.2 (SVDQuant summary page).
Mutation tests at the end plant mistakes in the oracle and check that a pin
catches each one."""

import json
import os

import numpy as np
import pytest
import scipy.linalg
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import bruteforce as BF
from bit_w4a4_quantized_b200 import workloads as WL
from oracle import formats as F
from oracle import svdquant as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- quantizer


def test_worked_outlier_example():
    ex = json.load(open(os.path.join(GOLDEN, "outlier_example.json")))
    block = np.zeros((1, 16), np.float32)
    block[0, :6] = np.float32(ex["page_input"])
    g = S.global_scale(np.max(np.abs(block)))
    codes, scales = S.nvfp4_quantize(block, g)
    deq = S.nvfp4_dequantize(codes, scales)[0, :6] * np.float64(g)
    np.testing.assert_allclose(deq, ex["expected_dequantized"], atol=1e-6)
    assert list(np.signbit(deq)) == ex["expected_negative_zero"]
    assert np.max(F.e2m1_decode(codes)) == ex["q_max"]


def _edge_blocks():
    g = np.random.default_rng(11)
    blocks = [g.standard_normal(16) * 10.0 ** g.integers(-3, 3) for _ in range(300)]
    blocks.append(np.zeros(16))
    blocks.append(np.full(16, -0.0))
    blocks.append(np.r_[1e-30, np.zeros(15)])  # scale underflows to 0
    blocks.append(np.r_[5.0, -0.1, 0.1, np.zeros(13)])
    blocks.append(g.standard_normal(16) * 1e-6)  # tiny block next to big ones
    blocks.append(np.r_[300.0, -300.0, g.standard_normal(14)])
    return np.array(blocks, dtype=np.float32)


def test_quantizer_matches_bruteforce():
    t = _edge_blocks()
    for g in (S.global_scale(np.max(np.abs(t))), np.float32(0.37), np.float32(1.0)):
        codes, scales = S.nvfp4_quantize(t, g)
        for i, row in enumerate(t):
            bc, bs = BF.quantize_block([float(v) for v in row], float(g))
            assert bs == scales[i, 0], (i, g)
            assert bc == codes[i].tolist(), (i, g)


def test_quantizer_error_within_half_grid_spacing():
    t = _edge_blocks()
    g = S.global_scale(np.max(np.abs(t)))
    codes, scales = S.nvfp4_quantize(t, g)
    d = (F.e4m3_decode(scales[:, 0]).astype(np.float32) * g).astype(np.float64)
    for i in range(t.shape[0]):
        if d[i] == 0:
            assert np.all(F.e2m1_decode(codes[i]) == 0)
            continue
        v = np.abs(t[i].astype(np.float64)) / d[i]
        q = np.abs(F.e2m1_decode(codes[i]))
        half = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
        bound = np.where(v > 6, v - 6, half) * (1 + 1e-6)
        assert np.all(np.abs(q - v) <= bound + 1e-12)


@settings(max_examples=60, deadline=None)
@given(seed=st.integers(0, 2**31 - 1), log_scale=st.floats(-20, 20), spread=st.integers(0, 12),
       zeros=st.floats(0, 0.5))
def test_quantizer_error_bound_on_random_blocks(seed, log_scale, spread, zeros):
    """Every element lands within half the local E2M1 grid spacing of t / d
    (0.25 below 2, 0.5 below 4, 1 above), or on 6 when t / d exceeds 6; a block
    with d = 0 has only zero codes.  Random magnitudes over 40 binades, blocks
    whose scales differ by up to 2^12, and exact zeros."""
    g0 = np.random.default_rng(seed)
    t = g0.standard_normal((8, 256)) * np.exp2(log_scale)
    t = t * np.exp2(g0.integers(-spread, spread + 1, size=(8, 16, 1))).repeat(16, axis=2).reshape(8, 256)
    t[g0.random(t.shape) < zeros] = 0.0
    t = t.astype(np.float32)
    g = S.global_scale(np.max(np.abs(t)))
    codes, scales = S.nvfp4_quantize(t, g)
    d = (F.e4m3_decode(scales).astype(np.float32) * g).astype(np.float64)  # [8, 16]
    v = np.abs(t.astype(np.float64)).reshape(8, 16, 16)
    q = np.abs(F.e2m1_decode(codes)).reshape(8, 16, 16)
    zero = d == 0
    assert np.all(q[zero] == 0)
    r = v[~zero] / d[~zero][:, None]
    half = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0))
    bound = np.where(r > 6, r - 6, half) * (1 + 1e-6)
    assert np.all(np.abs(q[~zero] - r) <= bound + 1e-12)


def test_scales_fit_e4m3_under_global_scale():
    t = np.random.default_rng(5).standard_normal((64, 256)).astype(np.float32) * 7
    g = S.global_scale(np.max(np.abs(t)))
    _, scales = S.nvfp4_quantize(t, g)
    assert np.all(F.e4m3_decode(scales) <= 448.0)
    # the block holding the tensor max gets the largest scale code (448)
    assert np.max(scales) == 0x7E


@settings(max_examples=60, deadline=None)
@given(seed=st.integers(0, 2**31 - 1), log_scale=st.floats(-12, 12), heavy=st.booleans())
def test_quantizer_is_idempotent_on_normal_scales(seed, log_scale, heavy):
    """Q(deq(Q(t)) g) = Q(t) on every block whose E4M3 scale is normal: each
    block's largest element lands on code 6 (the E4M3 rounding of the scale is
    within 1/16, so amax / d stays in [5.65, 6.4)), the dequantized block's
    maximum is then exactly 6 d, and every code value survives the round trip.
    A scale computed with a q_max other than 6 breaks it (the largest code is
    then not 6); errors in d alone are left to the brute force and the error
    bound above, since a consistently rescaled d still round-trips."""
    g0 = np.random.default_rng(seed)
    t = g0.standard_normal((16, 128)) * np.exp2(log_scale)
    if heavy:
        t = t * np.exp2(g0.integers(-8, 9, size=(16, 8, 1))).repeat(16, axis=2).reshape(16, 128)
    t = t.astype(np.float32)
    g = S.global_scale(np.max(np.abs(t)))
    codes, scales = S.nvfp4_quantize(t, g)
    deq = (S.nvfp4_dequantize(codes, scales) * np.float64(g)).astype(np.float32)
    codes2, scales2 = S.nvfp4_quantize(deq, g)
    normal = F.e4m3_decode(scales) >= 2.0**-6
    assert np.any(normal)
    blk = np.repeat(normal, 16, axis=1)
    np.testing.assert_array_equal(scales2[normal], scales[normal])
    np.testing.assert_array_equal(codes2[blk], codes[blk])
    top = np.max(np.abs(F.e2m1_decode(codes)).reshape(16, 8, 16), axis=2)
    assert np.all(top[normal] == 6.0)


# ---------------------------------------------------------------- smoothing


def test_smoothing_preserves_product_and_balances():
    g = np.random.default_rng(6)
    X = WL.make_x(32, 64, seed=9).astype(np.float64)
    W = WL.make_w(48, 64, seed=9).astype(np.float64)
    a = np.max(np.abs(X), axis=0).astype(np.float32)
    w = np.max(np.abs(W), axis=0).astype(np.float32)
    lam, inv = S.smoothing_factors(a, w)
    Xh = X / lam.astype(np.float64)
    Wh_t = lam.astype(np.float64)[:, None] * W.T
    np.testing.assert_allclose(Xh @ Wh_t, X @ W.T, rtol=1e-12, atol=1e-12)
    # migration strength 1/2: per channel max|X_hat| == max|W_hat|
    np.testing.assert_allclose(np.max(np.abs(Xh), 0), np.max(np.abs(Wh_t), 1), rtol=2e-7)
    # zero channels get lambda = 1
    a0 = a.copy()
    a0[3] = 0
    lam0, _ = S.smoothing_factors(a0, w)
    assert lam0[3] == 1.0
    del g


# ---------------------------------------------------------------- low rank


def _what(K=96, N=80, seed=7):
    W = WL.make_w(N, K, seed=seed).astype(np.float64)
    X = WL.make_x(64, K, seed=seed).astype(np.float64)
    lam, _ = S.smoothing_factors(np.max(np.abs(X), 0), np.max(np.abs(W), 0))
    return lam.astype(np.float64)[:, None] * W.T


def test_svd_singular_values_match_second_lapack_driver():
    A = _what()
    _, _, s = S.low_rank_factors(A, 8)
    s2 = scipy.linalg.svd(A, compute_uv=False, lapack_driver="gesvd")
    np.testing.assert_allclose(s, s2, rtol=1e-10, atol=1e-12 * s2[0])


def test_eckart_young_and_orthonormal_rows():
    A = _what()
    for r in (1, 4, 16):
        l1, l2, s = S.low_rank_factors(A, r)
        res = np.linalg.norm(S.residual(A, l1, l2))
        np.testing.assert_allclose(res, np.sqrt(np.sum(s[r:] ** 2)), rtol=1e-10)
        np.testing.assert_allclose(l2 @ l2.T, np.eye(r), atol=1e-12)
        np.testing.assert_allclose(l1.T @ l1, np.diag(s[:r] ** 2), rtol=1e-10, atol=1e-10 * s[0] ** 2)


def test_exact_rank_r_weight_has_zero_residual():
    g = np.random.default_rng(8)
    A = g.standard_normal((96, 6)) @ g.standard_normal((6, 80))
    l1, l2, _ = S.low_rank_factors(A, 6)
    assert np.linalg.norm(S.residual(A, l1, l2)) / np.linalg.norm(A) < 1e-12


def test_decomposition_identity_before_quantization():
    A = _what()
    X = WL.make_x(16, 96, seed=3).astype(np.float64)
    l1, l2, _ = S.low_rank_factors(A, 8)
    l1b, l2b = S.bf16_from_f64(l1), S.bf16_from_f64(l2)
    R = S.residual(A, l1b, l2b)
    np.testing.assert_allclose(X @ l1b @ l2b + X @ R, X @ A, rtol=1e-11, atol=1e-11 * np.abs(X @ A).max())


# ----------------------------------------------------- whole-layer brute force


def _tiny_case(M, K, N, r, seed, bias, gelu):
    X = WL.make_x(M, K, seed=seed, n_outlier=2).astype(np.float32)
    W = WL.make_w(N, K, seed=seed, n_outlier=2).astype(np.float32)
    amax = np.max(np.abs(X), axis=0)
    b = WL.make_bias(N, seed).astype(np.float64) if bias else None
    lam, _ = S.smoothing_factors(amax, np.max(np.abs(W), 0))
    if r:
        l1, l2, _ = S.low_rank_factors(lam.astype(np.float64)[:, None] * W.T.astype(np.float64), r)
        l1b, l2b = S.bf16_from_f64(l1), S.bf16_from_f64(l2)
    else:
        l1b, l2b = np.zeros((K, 0)), np.zeros((0, N))
    return X, W, amax, l1b, l2b, b


def check_layer_against_bruteforce(M=3, K=32, N=5, r=2, seed=1, bias=True, gelu=False):
    X, W, amax, l1b, l2b, b = _tiny_case(M, K, N, r, seed, bias, gelu)
    layer = S.prepare(W, amax, r, bias=b, factors=(l1b, l2b))
    act = S.quantize_act(layer, X)
    y = S.linear(layer, act, S.EPI_GELU_TANH if gelu else S.EPI_NONE)
    ref = BF.layer_forward(W.tolist(), X.tolist(), amax.tolist(), l1b.tolist(), l2b.tolist(),
                           None if b is None else b.tolist(), gelu)
    assert layer.lam.tolist() == ref["lam"]
    assert float(layer.g_w) == ref["g_w"] and float(layer.g_a) == ref["g_a"]
    assert layer.w_codes.tolist() == ref["w_codes"]
    assert layer.w_scales.tolist() == ref["w_scales"]
    assert act.codes.tolist() == ref["a_codes"]
    assert act.scales.tolist() == ref["a_scales"]
    assert act.x_hat.astype(np.float64).tolist() == ref["x_hat"]
    yr = np.array(ref["Y"])
    np.testing.assert_allclose(y, yr, rtol=1e-12, atol=1e-12 * np.abs(yr).max())


@pytest.mark.parametrize("M,K,N,r,bias,gelu", [
    (3, 32, 5, 2, True, False),
    (4, 48, 7, 0, False, False),
    (2, 64, 3, 3, False, True),
    (5, 16, 4, 1, True, True),
])
def test_layer_matches_bruteforce(M, K, N, r, bias, gelu):
    check_layer_against_bruteforce(M, K, N, r, seed=M + K, bias=bias, gelu=gelu)


# ------------------------------------------------- section 4.1 bound, claims


def _small_spec_layer(spec, M=128, rank=None):
    X = spec.x(M).astype(np.float32)
    W = spec.w().astype(np.float32)
    amax = np.max(np.abs(X), axis=0)
    r = spec.rank if rank is None else rank
    return X, W, S.prepare(W, amax, r)


def test_error_bound_of_section_4_1_holds():
    X, W, layer = _small_spec_layer(WL.CFG1, rank=0)
    act = S.quantize_act(layer, X)
    Xh = act.x_hat.astype(np.float64)
    Wh_t = layer.R  # rank 0: R == W_hat^T
    QX = S.nvfp4_dequantize(act.codes, act.scales) * np.float64(layer.g_a)
    QW = (S.nvfp4_dequantize(layer.w_codes, layer.w_scales) * np.float64(layer.g_w)).T
    E = S.quant_error(Xh @ Wh_t, QX @ QW)
    assert E <= S.error_bound(Xh, Wh_t, QX, QW)
    assert E > 0


@pytest.mark.parametrize("spec", [WL.CFG1, WL.CFG2, WL.CFG3_FC1, WL.CFG4, WL.sweep_spec(256, 3072, 32)],
                         ids=lambda s: s.name)
def test_low_rank_branch_does_not_increase_error(spec):
    """Section 4.2: the low-rank branch absorbs the outliers smoothing moved into
    W, so the layer error with it is no worse than plain smoothed W4A4.

    64 rows of each workload; the attention projection at its full K x N, the
    other wide layers on their first 1024 output rows (a full LAPACK SVD of
    3072 x 12288 would dominate the CPU suite)."""
    M = 64 if spec.K > 1024 else spec.M
    X = spec.x(M).astype(np.float32)
    W = spec.w().astype(np.float32)
    if spec is not WL.CFG2:
        W = W[:1024]
    amax = np.max(np.abs(X), axis=0)
    XW = X.astype(np.float64) @ W.T.astype(np.float64)
    y0 = S.forward(S.prepare(W, amax, 0), X)
    y1 = S.forward(S.prepare(W, amax, spec.rank), X)
    assert S.quant_error(XW, y1) <= S.quant_error(XW, y0)


def test_rank_zero_is_plain_smoothed_w4a4():
    X, W, layer = _small_spec_layer(WL.CFG1, rank=0)
    lam = layer.lam.astype(np.float64)
    np.testing.assert_array_equal(layer.R, lam[:, None] * W.T.astype(np.float64))
    act = S.quantize_act(layer, X)
    assert act.lr.shape == (X.shape[0], 0)
    y = S.linear(layer, act)
    QX = S.nvfp4_dequantize(act.codes, act.scales)
    QW = S.nvfp4_dequantize(layer.w_codes, layer.w_scales)
    ref = layer.alpha * QX @ QW.T
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-13 * np.abs(ref).max())


def test_lora_adds_x_a_b():
    spec = WL.CFG1
    X, W, layer = _small_spec_layer(spec, M=64)
    A, B = WL.make_lora(spec.K, spec.N, 16, seed=0)
    y0 = S.forward(layer, X)
    S.attach_lora(layer, A.astype(np.float32), B.astype(np.float32), scale=0.5)
    assert layer.L1.shape == (spec.K, spec.rank + 16)
    y1 = S.forward(layer, X)
    want = 0.5 * X.astype(np.float64) @ A.astype(np.float64) @ B.astype(np.float64)
    got = y1 - y0
    assert np.max(np.abs(got - want)) <= 2e-2 * np.max(np.abs(want))
    S.detach_lora(layer)
    np.testing.assert_array_equal(S.forward(layer, X), y0)


def test_gelu_matches_torch():
    x = np.linspace(-8, 8, 4001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    np.testing.assert_allclose(S.gelu_tanh(x), ref, rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------ planted mistakes


def _mut_residual_sign(w_hat_t, l1, l2):
    r = np.array(w_hat_t, dtype=np.float64, copy=True)
    for j in range(l1.shape[1]):
        r += np.outer(l1[:, j], l2[j, :])
    return r


def _mut_smoothing_inverted(act_amax, w_amax):
    lam, inv = ORIG_SMOOTH(act_amax, w_amax)
    return inv, lam


ORIG_SMOOTH = S.smoothing_factors
ORIG_LINEAR = S.linear


def _mut_linear_no_lowrank(layer, act, epilogue=S.EPI_NONE, rows=None):
    act2 = S.Act(act.x_hat, act.codes, act.scales, act.lr * 0)
    return ORIG_LINEAR(layer, act2, epilogue, rows)


def _mut_quant_division(t, g):
    t = np.asarray(t, dtype=np.float32)
    rows, k = t.shape
    blocks = t.reshape(rows, k // 16, 16)
    amax = np.max(np.abs(blocks), axis=2)
    c = np.float32(1.0) / np.float32(6.0 * g)
    s_code = F.e4m3_encode((amax * c).astype(np.float32))
    d = (F.e4m3_decode(s_code).astype(np.float32) * g).astype(np.float32)
    q = F.e2m1_encode((blocks / np.where(d == 0, 1, d)[..., None]).astype(np.float32) * 1.02)
    return q.reshape(rows, k), s_code


@pytest.mark.parametrize("name,target,mutant", [
    ("residual sign", "residual", _mut_residual_sign),
    ("inverted smoothing", "smoothing_factors", _mut_smoothing_inverted),
    ("dropped low-rank term", "linear", _mut_linear_no_lowrank),
    ("perturbed element scaling", "nvfp4_quantize", _mut_quant_division),
])
def test_planted_mistake_is_caught(monkeypatch, name, target, mutant):
    monkeypatch.setattr(S, target, mutant)
    with pytest.raises(AssertionError):
        check_layer_against_bruteforce(3, 32, 5, 2, seed=35, bias=True, gelu=False)


def test_prepare_on_sampled_outputs_matches_the_whole_layer():
    """The restriction to some output features gives exactly those features of the whole layer."""
    g = np.random.default_rng([11, 1])
    K, N, r = 128, 96, 16
    W = F.bf16(g.normal(0, 0.02, (N, K)).astype(np.float32)).astype(np.float64)
    X = F.bf16(g.normal(0, 1, (8, K)).astype(np.float32))
    amax = np.max(np.abs(X.astype(np.float32)), 0)
    b = F.bf16(g.normal(0, 0.01, N).astype(np.float32)).astype(np.float64)
    whole = S.prepare(W, amax, r, bias=b)
    cols = np.array([0, 5, 17, 64, 95])
    part = S.prepare(W, amax, r, bias=b, factors=(whole.L1, whole.L2), out_rows=cols)
    assert part.N == len(cols) and part.g_w == whole.g_w
    np.testing.assert_array_equal(part.w_codes, whole.w_codes[cols])
    np.testing.assert_array_equal(part.w_scales, whole.w_scales[cols])
    np.testing.assert_array_equal(part.L2, whole.L2[:, cols])
    y_whole = S.forward(whole, X)
    np.testing.assert_array_equal(S.forward(part, X), y_whole[:, cols])
