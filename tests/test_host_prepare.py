"""Host preparation (C++) against the oracle, without a GPU.

With the same low-rank factors (computed by the oracle's LAPACK SVD and given
to the library as a checkpoint would), every prepared quantity is a function
of the inputs with exactly defined float32 / float64 arithmetic, so the
library must match the oracle bit for bit: lambda, R, the weight codes and
block scales, g_w and g_a.  The library's own randomized SVD is checked for
quality against LAPACK (singular values, Eckart-Young residual)."""

import numpy as np
import pytest
import scipy.linalg

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from oracle import formats as F
from oracle import svdquant as S


def _oracle_factors(W, amax, r):
    lam, _ = S.smoothing_factors(amax, np.max(np.abs(W), 0))
    l1, l2, s = S.low_rank_factors(lam.astype(np.float64)[:, None] * W.T.astype(np.float64), r)
    return S.bf16_from_f64(l1), S.bf16_from_f64(l2), s


def _case(spec, M=None, N=None):
    X = spec.x(M).astype(np.float32)
    W = spec.w()
    if N is not None:
        W = W[:N]
    return X, W, np.max(np.abs(X), axis=0)


CASES = [
    ("cfg1", WL.CFG1, None, None),
    ("cfg2_rows", WL.CFG2, 256, 512),
    ("sweep_r0", WL.sweep_spec(256, 3072, 0), 64, 256),
    ("cfg4_rank32", WL.CFG4, 64, 320),
]


@pytest.mark.parametrize("name,spec,M,N", CASES, ids=[c[0] for c in CASES])
def test_prepare_with_given_factors_is_bit_exact(name, spec, M, N):
    X, W, amax = _case(spec, M, N)
    Wf = W.astype(np.float32)
    r = spec.rank
    if r:
        l1b, l2b, _ = _oracle_factors(Wf, amax, r)
        factors = (l1b, l2b)
        lib_factors = (F.bf16_bits(l1b.astype(np.float32)), F.bf16_bits(l2b.astype(np.float32)))
    else:
        factors, lib_factors = None, None
    ref = S.prepare(Wf, amax, r, bias=None, factors=factors)
    layer = svdq.Layer(W, amax, r, factors=lib_factors, keep_r=True, threads=4)

    np.testing.assert_array_equal(layer.export(svdq.EXPORT_LAMBDA), ref.lam)
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_INV_LAMBDA), ref.inv_lam)
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_R), ref.R.astype(np.float32))
    g_a, g_w, alpha, inv_alpha = layer.export(svdq.EXPORT_SCALARS)
    assert g_w == ref.g_w and g_a == ref.g_a
    assert alpha == np.float32(ref.g_a * ref.g_w)
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_W_CODES), F.pack_e2m1(ref.w_codes))
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_W_SCALES), ref.w_scales)
    if r:
        np.testing.assert_array_equal(F.bf16_from_bits(layer.export(svdq.EXPORT_L1)), l1b.astype(np.float32))
        np.testing.assert_array_equal(F.bf16_from_bits(layer.export(svdq.EXPORT_L2)), l2b.astype(np.float32))


def test_prepare_is_independent_of_thread_count():
    X, W, amax = _case(WL.CFG1)
    a = svdq.Layer(W, amax, 16, threads=1, keep_r=True)
    b = svdq.Layer(W, amax, 16, threads=7, keep_r=True)
    for what in (svdq.EXPORT_L1, svdq.EXPORT_L2, svdq.EXPORT_W_CODES, svdq.EXPORT_W_SCALES, svdq.EXPORT_SIGMA):
        np.testing.assert_array_equal(a.export(what), b.export(what))


@pytest.mark.parametrize("name,spec,M,N", [
    ("cfg1", WL.CFG1, None, None),
    ("cfg2_cols", WL.CFG2, 128, 1024),
    ("sweep_r64", WL.sweep_spec(256, 3072, 64), 64, 512),
], ids=lambda c: c if isinstance(c, str) else "")
def test_library_svd_quality_against_lapack(name, spec, M, N):
    X, W, amax = _case(spec, M, N)
    Wf = W.astype(np.float32)
    r = spec.rank
    layer = svdq.Layer(W, amax, r, threads=8)
    lam = layer.export(svdq.EXPORT_LAMBDA).astype(np.float64)
    A = lam[:, None] * Wf.T.astype(np.float64)
    s = scipy.linalg.svd(A, compute_uv=False, lapack_driver="gesvd")
    sig = layer.export(svdq.EXPORT_SIGMA)
    # Ritz values from a subspace never exceed the true singular values
    # (interlacing); the well-separated leading ones are found to high accuracy
    assert np.all(sig <= s[:r] * (1 + 1e-12))
    lead = s[:r] > 1.5 * s[r]
    np.testing.assert_allclose(sig[lead], s[:r][lead], rtol=1e-6)
    tail = np.sqrt(np.sum(s[r:] ** 2))
    r_f64, r_bf16 = layer.export(svdq.EXPORT_RESID_NORM)
    # Eckart-Young: no rank-r factorization beats the tail; ours is within 1 %
    assert tail * (1 - 1e-12) <= r_f64 <= 1.01 * tail
    # bf16 rounding of the factors adds at most ~2^-8 relative of ||L1 L2||
    assert r_bf16 <= r_f64 + 2 * 2.0**-8 * np.sqrt(np.sum(s[:r] ** 2))
    # L2 rows orthonormal up to bf16 rounding
    l2 = F.bf16_from_bits(layer.export(svdq.EXPORT_L2)).astype(np.float64)
    np.testing.assert_allclose(l2 @ l2.T, np.eye(r), atol=2e-2)


def test_library_svd_exact_rank():
    g = np.random.default_rng(3)
    K, N, r = 256, 192, 16
    W = (g.standard_normal((N, r)) @ g.standard_normal((r, K)) * 0.05).astype(np.float32)
    Wb = WL.to_bf16(W)
    amax = np.ones(K, np.float32)
    layer = svdq.Layer(Wb, amax, r, threads=4)
    r_f64, _ = layer.export(svdq.EXPORT_RESID_NORM)
    A = layer.export(svdq.EXPORT_LAMBDA).astype(np.float64)[:, None] * Wb.astype(np.float64).T
    # bf16 rounding of W makes it full rank, but only barely: the tail is tiny
    s = scipy.linalg.svd(A, compute_uv=False)
    assert r_f64 <= 1.01 * np.sqrt(np.sum(s[r:] ** 2))
    assert r_f64 < 1e-2 * np.linalg.norm(A)


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=20, deadline=None)
@given(kt=st.integers(1, 3), nt=st.integers(1, 2), r=st.sampled_from([0, 16]), seed=st.integers(0, 10_000),
       wscale=st.sampled_from([1e-6, 0.02, 50.0]), zero_cols=st.integers(0, 3))
def test_prepare_is_bit_exact_on_random_layers(kt, nt, r, seed, wscale, zero_cols):
    # zero activation channels and zero weight columns (lambda = 1 there), weights from
    # E4M3-subnormal block scales to large ones, ranks 0 and 16
    K, N = 64 * kt, 64 * nt
    g = np.random.default_rng(seed)
    W = WL.to_bf16(g.standard_normal((N, K)) * wscale)
    amax = np.abs(g.standard_normal(K) * 3.0).astype(np.float32)
    cols = g.choice(K, size=zero_cols, replace=False)
    if zero_cols:
        amax[cols[: (zero_cols + 1) // 2]] = 0.0
        Wz = W.astype(np.float32)
        Wz[:, cols[(zero_cols + 1) // 2:]] = 0.0
        W = WL.to_bf16(Wz)
    amax = WL.to_bf16(amax).astype(np.float32)  # calibration maxima of bf16 activations
    Wf = W.astype(np.float32)
    if r:
        l1b, l2b, _ = _oracle_factors(Wf, amax, r)
        factors = (l1b, l2b)
        lib_factors = (F.bf16_bits(l1b.astype(np.float32)), F.bf16_bits(l2b.astype(np.float32)))
    else:
        factors, lib_factors = None, None
    ref = S.prepare(Wf, amax, r, bias=None, factors=factors)
    layer = svdq.Layer(W, amax, r, factors=lib_factors, keep_r=True, threads=2)
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_LAMBDA), ref.lam)
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_R), ref.R.astype(np.float32))
    g_a, g_w, _, _ = layer.export(svdq.EXPORT_SCALARS)
    assert g_w == ref.g_w and g_a == ref.g_a
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_W_CODES), F.pack_e2m1(ref.w_codes))
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_W_SCALES), ref.w_scales)
    layer.close()


def test_all_zero_calibration_batch():
    """A layer calibrated on an all-zero batch: lambda = 1 on every channel
    (either maximum 0) and the activation tensor scale falls back to 1, on both
    sides, bit for bit."""
    W = WL.make_w(192, 256, seed=62)
    Wf = W.astype(np.float32)
    amax = np.zeros(256, np.float32)
    l1b, l2b, _ = _oracle_factors(Wf, amax, 16)
    ref = S.prepare(Wf, amax, 16, factors=(l1b, l2b))
    assert np.all(ref.lam == 1.0) and ref.g_a == 1.0
    layer = svdq.Layer(W, amax, 16, factors=(F.bf16_bits(l1b.astype(np.float32)), F.bf16_bits(l2b.astype(np.float32))),
                       threads=2)
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_LAMBDA), ref.lam)
    g_a, g_w, alpha, _ = layer.export(svdq.EXPORT_SCALARS)
    assert g_a == 1.0 and g_w == ref.g_w and alpha == np.float32(ref.g_a * ref.g_w)
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_W_CODES), F.pack_e2m1(ref.w_codes))
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_W_SCALES), ref.w_scales)


def test_host_quantizer_rounds_every_e2m1_tie_like_the_oracle():
    """Rank 0 and lambda = 1 make R^T = W.  With max|W| = 2.625 the tensor scale
    is 2^-10, and a block whose largest value is 1.5 gets the block scale 256, so
    d = 0.25 and each weight times 1/d is exact: the weights 0.0625, 0.1875,
    0.3125, 0.4375, 0.625, 0.875 and 1.25 land on the E2M1 ties 0.25 ... 5 (ties
    go to the even code), and their bf16 neighbours one step off them."""
    from ml_dtypes import bfloat16

    K, N = 64, 64
    ties = np.array([0.0625, 0.1875, 0.3125, 0.4375, 0.625, 0.875, 1.25], np.float32)
    bits = ties.astype(bfloat16).view(np.uint16)
    below = (bits - 1).view(bfloat16).astype(np.float32)  # the bf16 neighbours of each tie
    above = (bits + 1).view(bfloat16).astype(np.float32)
    vals = np.concatenate([ties, below, above])  # 21 values
    W = np.zeros((N, K), np.float32)
    for n in range(N):
        for b in range(K // 16):
            blk = np.zeros(16, np.float32)
            blk[0] = 1.5  # block maximum: scale 256, d = 0.25
            pick = np.random.default_rng([n, b]).choice(vals.size, 15, replace=False)
            blk[1:] = vals[pick] * np.where(np.random.default_rng([b, n]).random(15) < 0.5, -1, 1)
            W[n, 16 * b:16 * b + 16] = blk
    W[0, 0] = 2.625  # the tensor maximum: g_w = 2^-10
    Wb = W.astype(bfloat16)
    assert np.array_equal(Wb.astype(np.float32), W)
    amax = np.max(np.abs(W), axis=0)  # act_amax = max|W_:,j| gives lambda = 1
    ref = S.prepare(W, amax, 0)
    assert np.all(ref.lam == 1.0) and ref.g_w == np.float32(2.0**-10)
    assert np.count_nonzero(ref.w_scales == 0x78) > N  # E4M3 256: d = 0.25 on those blocks
    layer = svdq.Layer(Wb, amax, 0, threads=3)
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_W_CODES), F.pack_e2m1(ref.w_codes))
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_W_SCALES), ref.w_scales)
    # the ties themselves went to the even code (0.25 -> 0, 0.75 -> 2, 1.25 -> 2, 1.75 -> 4, 2.5 -> 4, 3.5 -> 6, 5 -> 6)
    deq_rows = ref.w_codes.reshape(N, K // 16, 16)
    Wr = np.abs(W.reshape(N, K // 16, 16))
    want = {0.0625: 0, 0.1875: 2, 0.3125: 2, 0.4375: 4, 0.625: 4, 0.875: 6, 1.25: 6}
    for v, code in want.items():
        sel = (Wr == np.float32(v)) & (ref.w_scales[..., None] == 0x78)
        assert np.any(sel)
        assert np.all((deq_rows[sel] & 7) == code), v
