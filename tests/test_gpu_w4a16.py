"""GPU parity of the W4A16 layer (4-bit NVFP4 weights, bf16 activations, an
activation-aware scale s per input channel) against oracle.w4a16.

Codes and scales are checked bit for bit on the host (tests/test_w4a16_host.py);
here Y is compared with max|Y - Y_ref| / max|Y_ref| <= 1e-2 over several row
counts (the kernel takes X 8 rows per launch), ragged N, the smallest and the
largest K, bias and s, and the FLUX-like modulation shape on sampled output
features."""

import numpy as np
import pytest
import torch

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from gpu_cases import assert_y_close, y_to_f64
from oracle import svdquant as S
from oracle import w4a16 as W4

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()


def _case(M, K, N, seed, with_s, with_bias):
    X = WL.make_x(M, K, seed=seed, n_outlier=0)
    W = WL.make_w(N, K, seed=seed)
    s = WL.make_awq_scales(K, seed=seed) if with_s else None
    b = WL.make_bias(N, seed=seed) if with_bias else None
    return X, W, s, b


@pytest.mark.parametrize("M,K,N,with_s,with_bias", [
    (1, 64, 1, False, False), (1, 3072, 257, True, True), (2, 256, 96, True, False), (3, 1024, 130, False, True),
    (4, 512, 64, True, True), (5, 3072, 200, True, False), (8, 768, 33, False, False), (13, 2048, 48, True, True),
])
def test_parity(M, K, N, with_s, with_bias):
    X, W, s, b = _case(M, K, N, 41 + M, with_s, with_bias)
    L = svdq.W4A16Layer(W, s=s, bias=b, device="cuda")
    Y = L.linear(_dev(X))
    torch.cuda.synchronize()
    ref = W4.prepare(W.astype(np.float32), s=s, bias=None if b is None else b.astype(np.float32))
    want = W4.linear(ref, X.astype(np.float32))
    err = assert_y_close(y_to_f64(Y), want)
    L.poll_status()
    print(f"W4A16 M{M} K{K} N{N}: max rel err {err:.2e}")


@pytest.mark.parametrize("M,K,N", [(3, 4096, 200), (1, 12288, 40), (8, 12288, 40), (9, 12288, 17)])
def test_largest_k_and_several_passes_over_k(M, K, N):
    """K above 3072 takes each row tile through several stages of the weight ring
    (48 tiles of 16 x 64 per stage; K = 4096: a partial second stage); K = 12288
    is the largest K the layer takes, and 8 rows of it the largest shared-memory
    request (x~ 196 KB, one CTA per SM with a ring of smaller stages).  Nine rows
    run as one 8-row launch on the tensor cores and one 1-row launch on the CUDA
    cores.  No bounded wait may have given up."""
    X, W, s, b = _case(M, K, N, 51 + M, True, True)
    L = svdq.W4A16Layer(W, s=s, bias=b, device="cuda")
    Y = L.linear(_dev(X))
    torch.cuda.synchronize()
    ref = W4.prepare(W.astype(np.float32), s=s, bias=b.astype(np.float32))
    assert_y_close(y_to_f64(Y), W4.linear(ref, X.astype(np.float32)))
    L.poll_status()


@pytest.mark.parametrize("M", [1, 2, 4])
def test_modulation_shape_on_sampled_features(M):
    spec = WL.w4a16_spec(M)
    X, W, s, b = spec.x(), spec.w(), spec.s(), spec.b()
    L = svdq.W4A16Layer(W, s=s, bias=b, device="cuda")
    Y = y_to_f64(L.linear(_dev(X)))
    torch.cuda.synchronize()
    g = np.random.default_rng([7, WL.STREAM_SAMPLE])
    cols = np.sort(np.concatenate([[0, spec.N - 1], g.choice(spec.N, 512, replace=False)]))
    ref = W4.prepare(W.astype(np.float32), s=s, bias=b.astype(np.float32), rows=cols)
    want = W4.linear(ref, X.astype(np.float32))
    err = assert_y_close(Y[:, cols], want)
    print(f"W4A16 modulation M{M}: max rel err {err:.2e}")


def test_deterministic_and_bad_arguments():
    X, W, s, b = _case(3, 256, 40, 5, True, True)
    L = svdq.W4A16Layer(W, s=s, bias=b, device="cuda")
    Xd = _dev(X)
    Y1 = L.linear(Xd)
    Y2 = L.linear(Xd)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    lib = svdq.lib()
    Y = torch.empty((3, 40), dtype=torch.bfloat16, device="cuda")
    assert lib.svdq_w4a16_linear(L._h, Xd.data_ptr(), 0, Y.data_ptr(), None) == svdq.ERR_INVALID_ARGUMENT
    assert lib.svdq_w4a16_linear(L._h, Xd.data_ptr() + 2, 1, Y.data_ptr(), None) == svdq.ERR_INVALID_ARGUMENT
    assert lib.svdq_w4a16_linear(L._h, None, 1, Y.data_ptr(), None) == svdq.ERR_INVALID_ARGUMENT
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    assert lib.svdq_w4a16_upload(L._h, small.data_ptr(), 16, None) == svdq.ERR_BUFFER_TOO_SMALL
