"""GPU parity of the fused MLP pair (svdq_w4a4_linear_mlp): fc1's output tile turned straight
into fc2's activation buffer (Diffusers/Nunchaku page, the fused GELU/MLP path).

Three comparisons:
  * against the library's own unfused path (fc1's kernel 2 writing Y1, then fc2's kernel 1 on
    it): the fused codes and block scales must be the same bytes, lr' within bf16 rounding --
    the fusion moves fc2's quantization, it must not change it;
  * against the oracle's pair (oracle.svdquant.mlp_pair): codes and scales bit-exact on every
    16-element block whose hidden values the GPU's fc1 reproduced exactly, and fc2's output
    within the pair bound (PAIR_TOL).  Such blocks are few: the GPU's GELU uses the hardware tanh
    approximation and its sums are float32, so most 16-value blocks of the bf16 hidden state
    hold at least one value one ulp off the float64 oracle's (the unfused path shares this;
    its codes are pinned to the oracle on given inputs by the kernel-1 tests);
  * shapes: several tiles, a ragged last weight tile of fc1 (N1 % 256 = 128), fc2 with no ranks,
    fc2 with a LoRA attached, and the full MLP workload on sampled rows."""

import numpy as np
import pytest
import torch

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from gpu_cases import LR_TOL, PAIR_TOL, Case, assert_y_close, y_to_f64
from oracle import formats as F
from oracle import svdquant as S

pytestmark = pytest.mark.gpu


def _to_bf16(a):
    return WL.to_bf16(np.asarray(a, np.float32))


def _pair(M, K1, N1, N2, r1, r2, seed, lora=0, cal_rows=None):
    X = WL.make_x(M, K1, seed=seed)
    W1 = WL.make_w(N1, K1, seed=seed)
    W2 = WL.make_w(N2, N1, seed=seed + 1, n_outlier=0)
    fc1 = Case(X, W1, r1, bias=WL.make_bias(N1, seed))
    # fc2 is calibrated on the oracle's hidden state (on a row sample for large M)
    Xc = fc1.X32 if cal_rows is None else fc1.X32[cal_rows]
    h_cal = S.bf16_from_f64(S.forward(fc1.ref, Xc, S.EPI_GELU_TANH)).astype(np.float32)
    fc2 = Case(_to_bf16(h_cal), W2, r2, rank_capacity=r2 + lora)
    return fc1, fc2


def _unfused(fc1, fc2, M):
    act1 = fc1.layer.quantize_act(fc1.Xd)
    Y1 = fc1.layer.linear(act1, M, epilogue=svdq.EPI_GELU_TANH)
    act2_ref = fc2.layer.quantize_act(Y1)
    return act1, Y1, act2_ref


def _check_pair(fc1, fc2, M, rows=None):
    act1, Y1, act2_ref = _unfused(fc1, fc2, M)
    act2 = fc1.layer.linear_mlp(act1, M, fc2.layer)
    Y2 = fc2.layer.linear(act2, M)
    Y2_ref = fc2.layer.linear(act2_ref, M)
    torch.cuda.synchronize()
    fc1.layer.poll_status()
    fc2.layer.poll_status()
    # 1. the library's own unfused path: same bytes
    c_f, s_f, lr_f = fc2.layer.act_unpack(act2.cpu().numpy(), M)
    c_u, s_u, lr_u = fc2.layer.act_unpack(act2_ref.cpu().numpy(), M)
    np.testing.assert_array_equal(c_f, c_u)
    np.testing.assert_array_equal(s_f, s_u)
    if lr_u.shape[1]:
        a = F.bf16_from_bits(lr_f).astype(np.float64)
        b = F.bf16_from_bits(lr_u).astype(np.float64)
        assert np.max(np.abs(a - b)) <= LR_TOL * max(np.max(np.abs(b)), 1e-30)
    # 2. the oracle's pair, on `rows`
    sel = np.arange(M) if rows is None else rows
    h, act2_o, y2_o = S.mlp_pair(fc1.ref, fc2.ref, fc1.X32[sel])
    y1 = Y1.float().cpu().numpy()[sel]
    same = (y1.reshape(len(sel), -1, 16) == h.reshape(len(sel), -1, 16)).all(axis=2)  # blocks with equal inputs
    codes_o = F.pack_e2m1(act2_o.codes).reshape(len(sel), -1, 8)
    cf = c_f[sel].reshape(len(sel), -1, 8)
    assert np.array_equal(cf[same], codes_o[same])
    assert np.array_equal(s_f[sel][same], act2_o.scales[same])
    # fc2's output: both layer bounds against the unfused pair (the same hidden state), and the
    # pair bound against the oracle's pair, whose hidden state differs from the GPU's by last-ulp
    # values that fc2's 4-bit quantizer turns into whole-code flips (PAIR_TOL is derived from the
    # oracle's own sensitivity to such changes, tests/test_oracle_mlp.py)
    assert_y_close(y_to_f64(Y2), y_to_f64(Y2_ref))
    err = S.max_rel_err(y_to_f64(Y2)[sel], y2_o)
    assert err <= PAIR_TOL, err
    return same.mean()


def test_pair_several_tiles_and_a_ragged_weight_tile():
    fc1, fc2 = _pair(300, 256, 640, 256, 16, 32, seed=61)
    _check_pair(fc1, fc2, 300)


def test_pair_with_no_ranks_in_fc2():
    fc1, fc2 = _pair(130, 512, 512, 320, 32, 0, seed=62)
    assert fc1.layer.mlp_workspace_bytes(fc2.layer, 130) == 0
    _check_pair(fc1, fc2, 130)


def test_pair_with_a_lora_on_fc2():
    fc1, fc2 = _pair(200, 256, 768, 256, 16, 32, seed=63, lora=16)
    A, B = WL.make_lora(768, 256, 16, seed=63)
    to = lambda a: torch.from_numpy(a.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    fc2.layer.lora_swap(to(A), to(B))
    S.attach_lora(fc2.ref, A.astype(np.float32), B.astype(np.float32))
    _check_pair(fc1, fc2, 200)


def test_fused_pair_is_deterministic_and_reuses_its_workspace():
    fc1, fc2 = _pair(257, 256, 512, 256, 16, 32, seed=64)
    act1 = fc1.layer.quantize_act(fc1.Xd)
    ws = torch.empty(fc1.layer.mlp_workspace_bytes(fc2.layer, 257), dtype=torch.uint8, device="cuda")
    a = fc1.layer.linear_mlp(act1, 257, fc2.layer, workspace=ws).clone()
    ws.fill_(0xFF)  # garbage left in the scratch must not matter
    b = fc1.layer.linear_mlp(act1, 257, fc2.layer, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_mlp_arguments_are_checked():
    fc1, fc2 = _pair(64, 128, 512, 256, 16, 16, seed=65)
    act1 = fc1.layer.quantize_act(fc1.Xd)
    with pytest.raises(svdq.SvdqError) as e:  # fc2's K must be fc1's N
        fc2.layer.linear_mlp(fc2.layer.quantize_act(fc2.Xd), 64, fc1.layer)
    assert e.value.status == svdq.ERR_UNSUPPORTED_SHAPE
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(svdq.SvdqError) as e:
        fc1.layer.linear_mlp(act1, 64, fc2.layer, workspace=small)
    assert e.value.status == svdq.ERR_BUFFER_TOO_SMALL


def test_mlp_workload_sampled_rows():
    """The MLP pair of the workload (M = 4608, fc1 3072 -> 12288 with GELU, fc2 12288 -> 3072,
    rank 32): all rows against the unfused library path, sampled rows against the oracle."""
    s1, s2 = WL.CFG3_FC1, WL.CFG3_FC2
    g = np.random.default_rng([3, WL.STREAM_SAMPLE])
    rows = np.sort(np.concatenate([[0, s1.M - 1], g.choice(s1.M, size=96, replace=False)]))
    X = s1.x()
    fc1 = Case(X, s1.w(), s1.rank)
    h_cal = S.bf16_from_f64(S.forward(fc1.ref, fc1.X32[rows], S.EPI_GELU_TANH)).astype(np.float32)
    fc2 = Case(_to_bf16(h_cal), s2.w(), s2.rank)
    frac = _check_pair(fc1, fc2, s1.M, rows=rows)
    print(f"MLP pair: {frac:.5f} of fc2's blocks had bit-identical hidden inputs")
