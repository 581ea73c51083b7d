"""The W4A16 layer's host half (no GPU): the library's NVFP4 quantization of
W diag(s) equals the oracle's bit for bit, and bad descriptors are refused."""

import ctypes

import numpy as np
import pytest

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from oracle import formats as F
from oracle import w4a16 as W4


@pytest.mark.parametrize("K,N,with_s,with_bias", [(64, 1, False, False), (256, 37, True, True),
                                                  (3072, 96, True, False), (1024, 300, False, True)])
def test_host_quantization_is_bit_exact(K, N, with_s, with_bias):
    W = WL.make_w(N, K, seed=31)
    s = WL.make_awq_scales(K, seed=31) if with_s else None
    b = WL.make_bias(N, seed=31) if with_bias else None
    L = svdq.W4A16Layer(W, s=s, bias=b)
    ref = W4.prepare(W.astype(np.float32), s=s, bias=None if b is None else b.astype(np.float32))
    np.testing.assert_array_equal(L.export(svdq.EXPORT_W_CODES), F.pack_e2m1(ref.codes))
    np.testing.assert_array_equal(L.export(svdq.EXPORT_W_SCALES), ref.scales)
    assert L.export(svdq.EXPORT_SCALARS)[0] == ref.g
    np.testing.assert_array_equal(L.export(svdq.EXPORT_INV_LAMBDA), ref.inv_s)
    L.close()


def test_bad_descriptors_are_refused():
    lib = svdq.lib()
    W = WL.make_w(8, 64, seed=1).view(np.uint16)
    for K, N in [(32, 8), (96, 8), (64, 0), (12288 + 64, 8)]:
        d = svdq.W4A16Desc()
        d.K, d.N, d.W = K, N, W.ctypes.data
        assert lib.svdq_w4a16_device_bytes(ctypes.byref(d)) == 0
        h = ctypes.c_void_p()
        assert lib.svdq_w4a16_prepare_host(ctypes.byref(d), ctypes.byref(h)) == svdq.ERR_UNSUPPORTED_SHAPE
    d = svdq.W4A16Desc()
    d.K, d.N, d.W = 64, 8, W.ctypes.data
    bad_s = np.zeros(64, np.float32)
    d.s = bad_s.ctypes.data
    h = ctypes.c_void_p()
    assert lib.svdq_w4a16_prepare_host(ctypes.byref(d), ctypes.byref(h)) == svdq.ERR_INVALID_ARGUMENT
    d.s = None
    d.W = None
    assert lib.svdq_w4a16_prepare_host(ctypes.byref(d), ctypes.byref(h)) == svdq.ERR_INVALID_ARGUMENT
    assert lib.svdq_w4a16_linear(None, None, 1, None, None) == svdq.ERR_INVALID_ARGUMENT
    lib.svdq_w4a16_destroy(None)


def test_host_only_layer_cannot_launch():
    L = svdq.W4A16Layer(WL.make_w(8, 64, seed=2))
    assert svdq.lib().svdq_w4a16_linear(L._h, 16, 1, 16, None) == svdq.ERR_INVALID_ARGUMENT
    assert "uploaded" in svdq.last_error()
    with pytest.raises(svdq.SvdqError):
        L.export(svdq.EXPORT_L1)


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(kt=st.integers(1, 4), n=st.integers(1, 40), seed=st.integers(0, 10_000), with_s=st.booleans(),
       scale=st.sampled_from([1e-4, 0.02, 3.0, 200.0]))
def test_host_quantization_matches_the_oracle_on_random_layers(kt, n, seed, with_s, scale):
    # any K that is a multiple of 64, any N, weights over several orders of magnitude
    K = 64 * kt
    g = np.random.default_rng(seed)
    W = WL.to_bf16(g.standard_normal((n, K)) * scale)
    s = (np.exp(g.uniform(-2, 2, K))).astype(np.float32) if with_s else None
    L = svdq.W4A16Layer(W, s=s)
    ref = W4.prepare(W.astype(np.float32), s=s)
    np.testing.assert_array_equal(L.export(svdq.EXPORT_W_CODES), F.pack_e2m1(ref.codes))
    np.testing.assert_array_equal(L.export(svdq.EXPORT_W_SCALES), ref.scales)
    assert L.export(svdq.EXPORT_SCALARS)[0] == ref.g
    L.close()


def test_modulation_workloads_stay_in_the_f16_operand_range():
    """The W4A16 layer rounds x / s to f16 (not bf16): values above 65504 would saturate and values below
    2^-14 would lose bits.  Every modulation workload's nonzero |x / s| lies inside [2^-14, 65504] up to a
    handful of tiny values, so the f16 operand changes nothing there."""
    from bit_w4a4_quantized_b200 import workloads as WL

    for N in (18432, 9216):
        for M in (1, 2, 4, 8):
            spec = WL.w4a16_spec(M, N=N)
            x = spec.x().astype(np.float64)
            inv = (np.float32(1.0) / spec.s().astype(np.float32)).astype(np.float64)
            v = np.abs(x * inv[None, :])
            assert v.max() < 65504.0
            nz = v[v > 0]
            assert np.mean(nz < 2.0**-14) < 1e-3
