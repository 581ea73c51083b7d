"""GPU parity of the INT4 layer (--precision int4) against oracle.int4.

The oracle prepares the layer with the same low-rank factors as the library,
so kernel 1's INT4 codes and bf16 group scales must agree bit for bit, lr'
within its bf16 rounding, and Y within the layer tolerance.  Nothing expected
here comes from the CUDA path."""

import types

import numpy as np
import pytest
import torch

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from gpu_cases import LR_TOL, assert_y_close, oracle_factors, y_to_f64
from oracle import formats as F
from oracle import int4 as I4
from oracle import svdquant as S

pytestmark = pytest.mark.gpu


class Int4Case:
    """Oracle INT4 layer + library INT4 layer built from the same inputs and factors."""

    def __init__(self, X, W, r, bias=None, rank_capacity=None):
        self.X = X
        self.X32 = X.astype(np.float32)
        self.W32 = W.astype(np.float32)
        self.amax = np.max(np.abs(self.X32), axis=0)
        l1b, l2b = oracle_factors(self.W32, self.amax, r)
        b64 = None if bias is None else bias.astype(np.float64)
        self.ref = I4.prepare(self.W32, self.amax, r, bias=b64, factors=(l1b, l2b))
        lib_factors = None
        if r:
            lib_factors = (F.bf16_bits(l1b.astype(np.float32)), F.bf16_bits(l2b.astype(np.float32)))
        self.layer = svdq.Layer(W, self.amax, r, rank_capacity=rank_capacity, bias=bias, factors=lib_factors,
                                device="cuda", fmt=svdq.FMT_INT4)
        self.alpha = float(self.layer.export(svdq.EXPORT_SCALARS)[2])
        self.Xd = torch.from_numpy(X.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()

    def run(self, epilogue=svdq.EPI_NONE):
        act = self.layer.quantize_act(self.Xd)
        Y = self.layer.linear(act, self.Xd.shape[0], epilogue=epilogue)
        torch.cuda.synchronize()
        return act, Y

    def check_act(self, act, rows=None):
        M = self.X.shape[0]
        codes, scales, lr = self.layer.act_unpack(act.cpu().numpy(), M)
        sel = slice(None) if rows is None else rows
        ref = I4.quantize_act(self.ref, self.X32[sel])
        u = F.unpack_e2m1(codes[sel]).astype(np.int16)
        np.testing.assert_array_equal(np.where(u >= 8, u - 16, u), ref.codes)
        np.testing.assert_array_equal(scales[sel], ref.scales)
        if self.ref.L1.shape[1]:
            lr_gpu = F.bf16_from_bits(lr[sel]).astype(np.float64) * self.alpha
            den = max(np.max(np.abs(ref.lr)), 1e-30)
            assert np.max(np.abs(lr_gpu - ref.lr)) <= LR_TOL * den
        return ref

    def check_y(self, Y, ref_act, epilogue=S.EPI_NONE, rows=None):
        y = y_to_f64(Y)
        if rows is not None:
            y = y[rows]
        return assert_y_close(y, I4.linear(self.ref, ref_act, epilogue))


def _spec_case(spec, M=None, **kw):
    return Int4Case(spec.x(M), spec.w(), spec.rank, bias=spec.b(), **kw)


def _rows(M, n=256, seed=0):
    g = np.random.default_rng([seed, WL.STREAM_SAMPLE])
    return np.sort(np.concatenate([[0, M - 1], g.choice(M, size=min(n, M), replace=False)]))


def test_int4_small_layer_bit_exact_codes_and_output():
    case = _spec_case(WL.CFG1)
    act, Y = case.run()
    case.check_y(Y, case.check_act(act))
    case.layer.poll_status()


@pytest.mark.parametrize("M", [1, 127, 129, 385])
def test_int4_ragged_rows(M):
    case = _spec_case(WL.CFG1, M=M)
    act, Y = case.run()
    case.check_y(Y, case.check_act(act))


@pytest.mark.parametrize("K,N,r", [(64, 64, 16), (128, 320, 0), (320, 192, 32), (768, 512, 48)])
def test_int4_small_and_ragged_k_n(K, N, r):
    X = WL.make_x(130, K, seed=K + N + 1)
    W = WL.make_w(N, K, seed=K + N + 1)
    case = Int4Case(X, W, r, bias=WL.make_bias(N, 6))
    act, Y = case.run()
    case.check_y(Y, case.check_act(act))


def test_int4_gelu_epilogue_with_bias():
    X = WL.make_x(300, 512, seed=8)
    W = WL.make_w(512, 512, seed=8)
    case = Int4Case(X, W, 32, bias=WL.make_bias(512, 8))
    act, Y = case.run(epilogue=svdq.EPI_GELU_TANH)
    case.check_y(Y, case.check_act(act), epilogue=S.EPI_GELU_TANH)


def test_int4_attention_projection_full():
    case = _spec_case(WL.CFG2)
    act, Y = case.run()
    err = case.check_y(Y, case.check_act(act))
    print(f"int4 attention projection max rel err {err:.3e}")
    case.layer.poll_status()


def test_int4_mlp_fc1_sampled_rows():
    spec = WL.CFG3_FC1
    case = _spec_case(spec)
    act, Y = case.run(epilogue=svdq.EPI_GELU_TANH)
    rows = _rows(spec.M, seed=7)
    case.check_y(Y, case.check_act(act, rows), epilogue=S.EPI_GELU_TANH, rows=rows)


def test_int4_deterministic_across_runs():
    case = _spec_case(WL.CFG2, M=512)
    act1, Y1 = case.run()
    act2, Y2 = case.run()
    for a, b in zip(case.layer.act_unpack(act1.cpu().numpy(), 512), case.layer.act_unpack(act2.cpu().numpy(), 512)):
        np.testing.assert_array_equal(a, b)
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_int4_lora_attach():
    spec = WL.CFG1
    case = _spec_case(spec, rank_capacity=spec.rank + 16)
    g = np.random.default_rng(9)
    A = WL.to_bf16(g.standard_normal((spec.K, 16)) * 0.05)
    B = WL.to_bf16(g.standard_normal((16, spec.N)) * 0.05)
    Ad = torch.from_numpy(A.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    Bd = torch.from_numpy(B.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    case.layer.lora_swap(Ad, Bd)
    # the adapter joins the branch as for NVFP4 (R untouched): L1' = [L1 | bf16(lambda A)], L2' = [L2 ; B]
    holder = S.attach_lora(types.SimpleNamespace(lam=case.ref.lam), A.astype(np.float32), B.astype(np.float32))
    case.ref.L1 = np.concatenate([case.ref.L1, holder.L1_lora], axis=1)
    case.ref.L2 = np.concatenate([case.ref.L2, holder.L2_lora], axis=0)
    act, Y = case.run()
    case.check_y(Y, case.check_act(act))


def test_int4_layer_from_a_blob_gives_the_same_output():
    case = _spec_case(WL.CFG1)
    act, Y = case.run()
    other = svdq.Layer.from_blob(case.layer.serialize(), device="cuda")
    act2 = other.quantize_act(case.Xd)
    Y2 = other.linear(act2, case.Xd.shape[0])
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


def test_int4_fused_epilogues_are_refused():
    case = _spec_case(WL.CFG1)
    act, _ = case.run()
    with pytest.raises(svdq.SvdqError) as e:
        case.layer.linear_mlp(act, case.Xd.shape[0], case.layer)
    assert e.value.status == svdq.ERR_INVALID_ARGUMENT and "NVFP4" in str(e.value)
    M = case.Xd.shape[0]
    rope = torch.zeros(svdq.rope_packed_bytes(M) // 4, dtype=torch.float32, device="cuda")
    nq = torch.ones(128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(svdq.SvdqError) as e:
        case.layer.linear_qkv_norm_rope(act, M, nq, nq, rope)
    assert e.value.status == svdq.ERR_INVALID_ARGUMENT and "NVFP4" in str(e.value)


def test_int4_zero_rows_give_the_bias():
    """All-zero rows: every group's scale is 0 and every code 0 (oracle and kernel alike), so Y is the bias."""
    spec = WL.CFG1
    X = spec.x()
    X[5:70] = 0
    case = Int4Case(X, spec.w(), spec.rank, bias=WL.make_bias(spec.N, 3))
    act, Y = case.run()
    ref = case.check_act(act)
    assert np.all(ref.codes[5:70] == 0) and np.all(ref.scales[5:70] == 0)
    case.check_y(Y, ref)


def test_int4_inputs_far_above_calibration_stay_finite():
    """The kernel's f16 operand holds q s 2^e_a with e_a set from the calibration maximum; a row 1000 times
    above it saturates there (a documented limit of the INT4 path) and must not turn into inf or NaN.
    Rows inside the range still match the oracle."""
    spec = WL.CFG1
    X = spec.x()
    case = Int4Case(X, spec.w(), spec.rank)
    Xbig = X.astype(np.float32)
    Xbig[3] *= 1000.0
    Xd = torch.from_numpy(WL.to_bf16(Xbig).view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    act = case.layer.quantize_act(Xd)
    Y = case.layer.linear(act, Xd.shape[0])
    torch.cuda.synchronize()
    y = y_to_f64(Y)
    assert np.all(np.isfinite(y))
    rows = np.array([r for r in range(X.shape[0]) if r != 3])
    ref = I4.quantize_act(case.ref, WL.to_bf16(Xbig).astype(np.float32)[rows])
    assert_y_close(y[rows], I4.linear(case.ref, ref))
    case.layer.poll_status()
