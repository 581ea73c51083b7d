"""GPU parity on the degenerate inputs of the method, through the C ABI.

- Zero blocks: a 16-element block of X_hat whose maximum is 0 gets the E4M3
  scale 0 and all codes 0 (reciprocal taken as 0), a zero channel gets
  lambda = 1, and a zero row of X gives Y = b exactly, since every term of the
  accumulator is 0 (SVDQuant summary page, section 3 "Quantization
  preliminary": s = max|X| / q_max, here per block).
- An all-zero calibration batch: the activation tensor scale falls back to 1.
- Activations beyond the calibrated maximum: the activation tensor scale is
  static, so larger runtime values saturate, the block scale at E4M3's 448 and
  the elements at E2M1's +-6, on both sides.
- An empty batch is refused before any launch.
- Exact E2M1 ties and exact E4M3 ties of the block scale: the device
  conversions take each tie to the even code, as the oracle does.

Codes and scales are compared bit for bit, Y within the layer tolerance."""

import numpy as np
import pytest
import torch
from ml_dtypes import bfloat16

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from gpu_cases import Case, assert_y_close, check_act, check_y, y_to_f64
from oracle import formats as F
from oracle import svdquant as S

pytestmark = pytest.mark.gpu


def _dev(X):
    return torch.from_numpy(X.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()


def _zeroed_x(M, K, seed):
    X = WL.make_x(M, K, seed=seed).astype(np.float32)
    g = np.random.default_rng([seed, 99])
    blocks = X.reshape(M, K // 16, 16)
    blocks[g.random((M, K // 16)) < 0.1] = 0.0  # a tenth of the blocks
    X[[0, M // 3, M - 1]] = 0.0  # whole rows
    X[:, 32:48] = 0.0  # whole channels (lambda = 1)
    return X.astype(bfloat16)


@pytest.mark.parametrize("r", [0, 32])
def test_zero_rows_channels_and_blocks(r):
    M, K, N = 200, 512, 384
    X = _zeroed_x(M, K, seed=61 + r)
    bias = WL.make_bias(N, seed=61)
    case = Case(X, WL.make_w(N, K, seed=61), r, bias=bias)
    assert case.ref.lam[32] == 1.0
    act, Y = case.run()
    ref = check_act(case, act)
    assert np.count_nonzero(ref.scales == 0) > M  # zero blocks were exercised
    check_y(case, Y, ref)
    Yb = Y.view(torch.int16).cpu().numpy().view(np.uint16)
    want = np.asarray(bias).view(np.uint16)
    for m in (0, M // 3, M - 1):
        np.testing.assert_array_equal(Yb[m], want)


def test_all_zero_calibration_batch_gives_the_bias():
    M, K, N = 130, 256, 192
    X = np.zeros((M, K), dtype=bfloat16)
    bias = WL.make_bias(N, seed=62)
    case = Case(X, WL.make_w(N, K, seed=62), 16, bias=bias)
    assert case.ref.g_a == 1.0
    act, Y = case.run()
    ref = check_act(case, act)
    assert not np.any(ref.codes) and not np.any(ref.scales)
    np.testing.assert_array_equal(Y.view(torch.int16).cpu().numpy().view(np.uint16),
                                  np.broadcast_to(np.asarray(bias).view(np.uint16), (M, N)))


@pytest.mark.parametrize("factor", [8.0, 64.0])
def test_activations_beyond_calibration_saturate(factor):
    M, K, N, r = 160, 768, 256, 16
    X = WL.make_x(M, K, seed=63)
    case = Case(X, WL.make_w(N, K, seed=63), r)
    Xs = (X.astype(np.float32) * np.float32(factor)).astype(bfloat16)  # a power of two: exact in bf16
    act, Y = case.run(X=_dev(Xs))
    codes, scales, lr = case.unpack(act, M)
    ref = S.quantize_act(case.ref, Xs.astype(np.float32))
    assert np.count_nonzero(ref.scales == 0x7E) > 0  # block scales saturated at 448
    top = np.float64(6 * 448) * np.float64(case.ref.g_a)  # the largest value Q can represent
    assert np.max(np.abs(ref.x_hat)) > 1.5 * top  # elements saturated at +-6
    np.testing.assert_array_equal(codes, F.pack_e2m1(ref.codes))
    np.testing.assert_array_equal(scales, ref.scales)
    lr_gpu = F.bf16_from_bits(lr).astype(np.float64) * case.ref.alpha
    assert np.max(np.abs(lr_gpu - ref.lr)) <= 2.0**-7 * np.max(np.abs(ref.lr))
    assert_y_close(y_to_f64(Y), S.linear(case.ref, ref))


def test_empty_batch_is_refused():
    case = Case(WL.make_x(64, 256, seed=64), WL.make_w(256, 256, seed=64), 16)
    with pytest.raises(svdq.SvdqError) as e:
        case.layer.quantize_act(case.Xd[:0])
    assert e.value.status == svdq.ERR_INVALID_ARGUMENT
    act = case.layer.quantize_act(case.Xd)
    Y = torch.empty((64, 256), dtype=torch.bfloat16, device="cuda")
    lib = svdq.lib()
    assert lib.svdq_w4a4_linear(case.layer._h, act.data_ptr(), act.numel(), 0, Y.data_ptr(), 0, None) == \
        svdq.ERR_INVALID_ARGUMENT
    # the layer still runs
    Y = case.layer.linear(act, 64)
    torch.cuda.synchronize()
    check_y(case, Y, check_act(case, act))


def _w4a16_check(X, W, s=None, bias=None):
    from oracle import w4a16 as W4

    L = svdq.W4A16Layer(W, s=s, bias=bias, device="cuda")
    Y = L.linear(_dev(X))
    torch.cuda.synchronize()
    ref = W4.prepare(W.astype(np.float32), s=s, bias=None if bias is None else bias.astype(np.float32))
    want = W4.linear(ref, X.astype(np.float32))
    assert_y_close(y_to_f64(Y), want)
    return Y, ref


@pytest.mark.parametrize("M", [1, 5])
def test_w4a16_zero_weight_rows_and_blocks_give_the_bias(M):
    """W4A16: zero weight blocks get the scale 0; an all-zero output row gives
    Y = b exactly; an all-zero W falls back to the tensor scale 1."""
    K, N = 512, 96
    W = WL.make_w(N, K, seed=65).astype(np.float32)
    g = np.random.default_rng([65, 99])
    W.reshape(N, K // 16, 16)[g.random((N, K // 16)) < 0.2] = 0.0
    W[[3, 40, N - 1]] = 0.0
    W = W.astype(bfloat16)
    bias = WL.make_bias(N, seed=65)
    X = WL.make_x(M, K, seed=65, n_outlier=0)
    Y, ref = _w4a16_check(X, W, s=WL.make_awq_scales(K, seed=65), bias=bias)
    assert np.count_nonzero(ref.scales == 0) > 3 * K // 16
    Yb = Y.view(torch.int16).cpu().numpy().view(np.uint16)
    for n in (3, 40, N - 1):
        np.testing.assert_array_equal(Yb[:, n], np.asarray(bias).view(np.uint16)[n])
    Z = np.zeros((N, K), dtype=bfloat16)
    Y0, ref0 = _w4a16_check(X, Z, bias=bias)
    assert ref0.g == 1.0
    np.testing.assert_array_equal(Y0.view(torch.int16).cpu().numpy().view(np.uint16),
                                  np.broadcast_to(np.asarray(bias).view(np.uint16), (M, N)))


@pytest.mark.parametrize("M", [1, 3])
def test_w4a16_activations_beyond_f16_saturate(M):
    """W4A16: x / s is rounded to f16 saturating at +-65504 on both sides."""
    K, N = 256, 64
    X = (WL.make_x(M, K, seed=66, n_outlier=0).astype(np.float32) * np.float32(2.0**17)).astype(bfloat16)
    from oracle import w4a16 as W4

    s = WL.make_awq_scales(K, seed=66)
    assert np.count_nonzero(np.abs(W4.act_operand(X.astype(np.float32), np.float32(1.0) / s)) == 65504.0) > 0
    _w4a16_check(X, WL.make_w(N, K, seed=66), s=s)


def test_qkv_norm_rope_on_zero_heads():
    """The fused Q/K RMSNorm + rotary epilogue on zero rows (no bias): every
    head's sum of squares is 0, eps keeps the norm finite, and the row stays
    0; other rows carry zero blocks and channels."""
    from test_gpu_qkv import _check, _inputs, _run, _v_passes_through

    M, K, C = 200, 512, 256
    X = _zeroed_x(M, K, seed=67)
    case = Case(X, WL.make_w(3 * C, K, seed=67), 16)
    host, dev = _inputs(M, seed=67)
    act, Yf, Yp = _run(case, dev, M)
    _check(case, Yf, check_act(case, act), host)
    _v_passes_through(Yf, Yp)
    for m in (0, M // 3, M - 1):
        assert not torch.any(Yf[m].float() != 0).item()


def _tie_inputs(M=64, K=128, N=64):
    """X whose blocks have the maximum 1.5 and values on (or one bf16 step off)
    the E2M1 ties after scaling, with max|X| = 2.625; W's column maxima equal
    X's, so lambda = 1, x_hat = x, g_a = 2^-10, the block scale is 256 and
    1/d = 4 exactly."""
    ties = np.array([0.0625, 0.1875, 0.3125, 0.4375, 0.625, 0.875, 1.25], np.float32)
    bits = ties.astype(bfloat16).view(np.uint16)
    vals = np.concatenate([ties, (bits - 1).view(bfloat16).astype(np.float32),
                           (bits + 1).view(bfloat16).astype(np.float32)])
    X = np.zeros((M, K), np.float32)
    g = np.random.default_rng(71)
    for m in range(M):
        for b in range(K // 16):
            X[m, 16 * b] = 1.5
            X[m, 16 * b + 1:16 * b + 16] = vals[g.choice(vals.size, 15, replace=False)] * np.where(
                g.random(15) < 0.5, -1, 1)
    X[0, 0] = 2.625
    W = WL.make_w(N, K, seed=71).astype(np.float32)
    W[0] = np.max(np.abs(X), axis=0)
    return X.astype(bfloat16), W.astype(bfloat16), ties


def test_activation_codes_on_exact_e2m1_ties():
    """Kernel 1's hardware conversion (round to nearest even, satfinite) takes
    every E2M1 tie to the even code, as the oracle's reading does: 0.25 -> 0,
    0.75 -> 2, 1.25 -> 2, 1.75 -> 4, 2.5 -> 4, 3.5 -> 6, 5 -> 6."""
    X, W, ties = _tie_inputs()
    case = Case(X, W, 0)
    assert np.all(case.ref.lam == 1.0) and case.ref.g_a == np.float32(2.0**-10)
    act, Y = case.run()
    ref = check_act(case, act)  # codes and scales bit for bit
    check_y(case, Y, ref)
    blocks = np.abs(X.astype(np.float32)).reshape(X.shape[0], -1, 16)
    codes = ref.codes.reshape(blocks.shape)
    on_256 = (ref.scales == 0x78)[..., None]
    for v, code in zip(ties, (0, 2, 2, 4, 4, 6, 6)):
        sel = (blocks == v) & on_256
        assert np.count_nonzero(sel) > 100
        assert np.all((codes[sel] & 7) == code), v


def _e4m3_tie_inputs(N=64, K=128):
    """Block maxima on every E4M3 midpoint (normal binades 2^-6 .. 2^7 and the
    subnormal range), bf16-exact; one extra row holds the tensor maximum 448, so
    g_a = f32(1/6), 6 g_a rounds to 1 and the block scale is E4M3(block max)
    itself.  W's column maxima equal X's (lambda = 1)."""
    mids = [(2.0**e * (1 + m / 8 + 1 / 16), m) for e in range(-6, 8) for m in range(8)]
    mids += [((m + 0.5) * 2.0**-9, m) for m in range(8)]
    per_row = K // 16
    M = (len(mids) + per_row - 1) // per_row + 1
    g = np.random.default_rng(72)
    X = np.zeros((M, K), np.float32)
    for i, (v, _) in enumerate(mids):
        m, b = divmod(i, per_row)
        blk = np.float32(v) * g.uniform(-1, 1, 16).astype(np.float32)
        blk[g.integers(16)] = v if g.random() < 0.5 else -v
        X[m, 16 * b:16 * b + 16] = blk
    X[M - 1, 0] = 448.0
    X = X.astype(bfloat16)
    W = WL.make_w(N, K, seed=72).astype(np.float32)
    W[0] = np.max(np.abs(X.astype(np.float32)), axis=0)
    return X, W.astype(bfloat16), mids


def test_block_scales_on_exact_e4m3_ties():
    """Kernel 1's E4M3 block scale (round to nearest even, satfinite) on block
    maxima that sit exactly between two E4M3 values: the even mantissa wins,
    in the normal binades and among the subnormal scales (the midpoint 2^-10
    goes to the scale 0, whose block then has all codes 0)."""
    X, W, mids = _e4m3_tie_inputs()
    case = Case(X, W, 0)
    assert np.all(case.ref.lam == 1.0)
    assert np.float32(np.float32(1.0) / np.float32(np.float32(6.0) * case.ref.g_a)) == 1.0
    act, Y = case.run()
    ref = check_act(case, act)  # codes and scales bit for bit
    check_y(case, Y, ref)
    scale = F.e4m3_decode(ref.scales)
    per_row = X.shape[1] // 16
    for i, (v, m) in enumerate(mids):
        r, b = divmod(i, per_row)
        if v < 2.0**-6:
            lo, hi = m * 2.0**-9, (m + 1) * 2.0**-9
        else:
            e = np.floor(np.log2(v))
            lo, hi = 2.0**e * (1 + m / 8), 2.0**e * (1 + (m + 1) / 8)
        assert scale[r, b] == (lo if m % 2 == 0 else hi), (v, scale[r, b])
