"""Host preparation of the INT4 layer (C++) against oracle.int4, without a GPU.

With the same low-rank factors, the INT4 codes and bf16 group scales of R^T are
exactly defined float32 decisions, so the library must match the oracle bit for
bit.  The power-of-two prescales of the kernel's f16 operands are checked
against their definition (the weights' largest value q s 2^e_w in (2^14, 2^15],
the calibration maximum of X_hat times 2^e_a in (2^10, 2^11]), and the layer
must survive a blob round trip unchanged."""

import numpy as np
import pytest

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from oracle import formats as F
from oracle import int4 as I4
from oracle import svdquant as S


def _oracle_factors(W, amax, r):
    lam, _ = S.smoothing_factors(amax, np.max(np.abs(W), 0))
    l1, l2, _ = S.low_rank_factors(lam.astype(np.float64)[:, None] * W.T.astype(np.float64), r)
    return S.bf16_from_f64(l1), S.bf16_from_f64(l2)


def _nibbles(packed):
    """int8 codes [N, K] from two's-complement nibbles, element 2i in the low nibble."""
    u = F.unpack_e2m1(packed).astype(np.int16)
    return np.where(u >= 8, u - 16, u).astype(np.int8)


CASES = [
    ("cfg1", WL.CFG1, None, None),
    ("cfg2_rows", WL.CFG2, 256, 512),
    ("rank0", WL.sweep_spec(256, 3072, 0), 64, 256),
    ("cfg4_rank32", WL.CFG4, 64, 320),
]


@pytest.mark.parametrize("name,spec,M,N", CASES, ids=[c[0] for c in CASES])
def test_int4_prepare_with_given_factors_is_bit_exact(name, spec, M, N):
    X = spec.x(M).astype(np.float32)
    W = spec.w() if N is None else spec.w()[:N]
    amax = np.max(np.abs(X), axis=0)
    r = spec.rank
    factors = _oracle_factors(W.astype(np.float32), amax, r) if r else None
    lib_factors = None if not r else (F.bf16_bits(factors[0].astype(np.float32)),
                                      F.bf16_bits(factors[1].astype(np.float32)))
    ref = I4.prepare(W.astype(np.float32), amax, r, factors=factors)
    layer = svdq.Layer(W, amax, r, factors=lib_factors, threads=4, fmt=svdq.FMT_INT4)
    assert layer.info().format == svdq.FMT_INT4
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_LAMBDA), ref.lam)
    np.testing.assert_array_equal(_nibbles(layer.export(svdq.EXPORT_W_CODES)), ref.w_codes)
    np.testing.assert_array_equal(layer.export(svdq.EXPORT_W_SCALES), ref.w_scales)

    # the prescales: powers of two at their stated ranges
    g_a, g_w, alpha, inv_alpha = (float(v) for v in layer.export(svdq.EXPORT_SCALARS))
    e_w, e_a = -np.log2(g_w), -np.log2(g_a)
    assert e_w == round(e_w) and e_a == round(e_a) and alpha == g_a * g_w and inv_alpha == 1.0 / alpha
    top_w = 7.0 * np.max(F.bf16_from_bits(ref.w_scales).astype(np.float64)) / g_w
    assert 2.0 ** 14 < top_w <= 2.0 ** 15
    xh_max = np.max(F.bf16((amax * ref.inv_lam).astype(np.float32)).astype(np.float64))
    assert 2.0 ** 10 < xh_max / g_a <= 2.0 ** 11


def test_int4_blob_round_trip_keeps_every_export():
    spec = WL.CFG1
    X = spec.x().astype(np.float32)
    W = spec.w()
    a = svdq.Layer(W, np.max(np.abs(X), axis=0), spec.rank, threads=4, fmt=svdq.FMT_INT4)
    b = svdq.Layer.from_blob(a.serialize())
    assert b.fmt == svdq.FMT_INT4
    for what in (svdq.EXPORT_LAMBDA, svdq.EXPORT_L1, svdq.EXPORT_L2, svdq.EXPORT_W_CODES, svdq.EXPORT_W_SCALES,
                 svdq.EXPORT_SCALARS):
        np.testing.assert_array_equal(a.export(what), b.export(what))


def test_int4_act_buffer_has_the_nvfp4_size():
    spec = WL.CFG1
    X = spec.x().astype(np.float32)
    W = spec.w()
    amax = np.max(np.abs(X), axis=0)
    a = svdq.Layer(W, amax, spec.rank, threads=4, fmt=svdq.FMT_INT4)
    b = svdq.Layer(W, amax, spec.rank, threads=4)
    for M in (1, 300, 4096):
        assert a.act_buffer_bytes(M) == b.act_buffer_bytes(M)
    assert a.device_bytes == b.device_bytes


def test_unknown_format_is_refused():
    spec = WL.CFG1
    W = spec.w()
    with pytest.raises(svdq.SvdqError):
        svdq.Layer(W, np.ones(W.shape[1], np.float32), 0, fmt=7)
