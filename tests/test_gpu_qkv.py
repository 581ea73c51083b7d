"""GPU parity of the fused QKV epilogue (per-head RMSNorm of Q and K and their
rotary turn, Diffusers/Nunchaku page, fused-QKV section) against the oracle.

The expected values are the oracle layer's output rounded to bf16, then
oracle.qkv.  Q, K and V are compared separately with the layer tolerance
(max|err| / max|ref| <= 1e-2 each), because normalized Q/K values and raw V
values have different scales.  V must also equal the plain layer's output
bit for bit: the epilogue passes it through."""

import numpy as np
import pytest
import torch

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from gpu_cases import Case, assert_y_close, check_act, y_to_f64
from oracle import qkv as QO
from oracle import svdquant as S

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _inputs(M, seed):
    nq, nk = WL.make_norm_weights(QO.HEAD_DIM, seed)
    rope = WL.make_rope(M, QO.HEAD_DIM)
    dev = lambda a: torch.from_numpy(a.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    return (nq, nk, rope), (dev(nq), dev(nk), svdq.rope_pack(torch.from_numpy(rope).cuda()))


def _check(case, Yf, ref_act, host, rows=None):
    nq, nk, rope = host
    y_lin = S.bf16_from_f64(S.linear(case.ref, ref_act))
    rp = rope if rows is None else rope[rows]
    want = QO.qkv_norm_rope(y_lin, nq.astype(np.float64), nk.astype(np.float64), rp, eps=EPS)
    got = y_to_f64(Yf)
    if rows is not None:
        got = got[rows]
    C = want.shape[1] // 3
    errs = []
    for part in range(3):
        cols = slice(part * C, (part + 1) * C)
        err = assert_y_close(got[:, cols], want[:, cols])
        errs.append(err)
    return errs


def _run(case, dev, M):
    act = case.layer.quantize_act(case.Xd)
    Yf = case.layer.linear_qkv_norm_rope(act, M, *dev, eps=EPS)
    Yp = case.layer.linear(act, M)
    torch.cuda.synchronize()
    return act, Yf, Yp


def _v_passes_through(Yf, Yp):
    C = Yf.shape[1] // 3
    assert torch.equal(Yf[:, 2 * C:].view(torch.int16), Yp[:, 2 * C:].view(torch.int16))


@pytest.mark.parametrize("M,K,C,r,bias", [(200, 256, 256, 16, True), (129, 512, 384, 32, False),
                                          (1, 256, 128, 0, True), (300, 768, 640, 48, False)])
def test_small_and_ragged(M, K, C, r, bias):
    # C = N / 3 columns per part: 384 and 640 put Q/K/V borders inside 256-column tiles
    N = 3 * C
    X = WL.make_x(M, K, seed=21)
    W = WL.make_w(N, K, seed=21)
    b = WL.make_bias(N, seed=21) if bias else None
    case = Case(X, W, r, bias=b)
    host, dev = _inputs(M, seed=21)
    act, Yf, Yp = _run(case, dev, M)
    errs = _check(case, Yf, check_act(case, act), host)
    _v_passes_through(Yf, Yp)
    case.layer.poll_status()
    print(f"M{M} K{K} N{N} r{r}: max rel err Q {errs[0]:.2e} K {errs[1]:.2e} V {errs[2]:.2e}")


def test_qkv_workload_with_lora_sampled_rows():
    spec = WL.CFG4
    case = Case(spec.x(), spec.w(), spec.rank, bias=spec.b(), rank_capacity=spec.rank + spec.lora_rank)
    A, B = spec.lora()
    to_dev = lambda a: torch.from_numpy(a.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    case.layer.lora_swap(to_dev(A), to_dev(B))
    S.attach_lora(case.ref, A.astype(np.float32), B.astype(np.float32))
    host, dev = _inputs(spec.M, seed=spec.seed)
    act, Yf, Yp = _run(case, dev, spec.M)
    g = np.random.default_rng([6, WL.STREAM_SAMPLE])
    rows = np.sort(np.concatenate([[0, spec.M - 1], g.choice(spec.M, 256, replace=False)]))
    errs = _check(case, Yf, check_act(case, act, rows), host, rows)
    _v_passes_through(Yf, Yp)
    case.layer.poll_status()
    print(f"QKV M{spec.M}: max rel err Q {errs[0]:.2e} K {errs[1]:.2e} V {errs[2]:.2e}")


def test_rope_pack_layout():
    # the packed table holds the same values in (row tile, chunk of 2 pairs, row) order
    M = 300
    rope = WL.make_rope(M, QO.HEAD_DIM)
    packed = svdq.rope_pack(torch.from_numpy(rope).cuda()).cpu().numpy().view(np.float32)
    MT = 2 * ((M + 255) // 256)
    assert packed.size == MT * 32 * 128 * 4 == svdq.rope_packed_bytes(M) // 4
    p = packed.reshape(MT, 32, 128, 4)
    full = np.zeros((MT * 128, 64, 2), np.float32)
    full[:M] = rope
    want = full.reshape(MT, 128, 32, 4).transpose(0, 2, 1, 3)
    np.testing.assert_array_equal(p, want)


def test_deterministic():
    case = Case(WL.make_x(256, 256, seed=22), WL.make_w(3 * 256, 256, seed=22), 16)
    host, dev = _inputs(256, seed=22)
    _, Y1, _ = _run(case, dev, 256)
    _, Y2, _ = _run(case, dev, 256)
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_bad_arguments_are_refused():
    M = 64
    host, (nq, nk, rope) = _inputs(M, seed=23)
    odd = Case(WL.make_x(M, 256, seed=23), WL.make_w(256, 256, seed=23), 16)  # N = 256: not 3 x heads
    act = odd.layer.quantize_act(odd.Xd)
    with pytest.raises(svdq.SvdqError) as e:
        odd.layer.linear_qkv_norm_rope(act, M, nq, nk, rope)
    assert e.value.status == svdq.ERR_UNSUPPORTED_SHAPE
    case = Case(WL.make_x(M, 256, seed=23), WL.make_w(3 * 128, 256, seed=23), 16)
    act = case.layer.quantize_act(case.Xd)
    with pytest.raises(svdq.SvdqError) as e:
        case.layer.linear_qkv_norm_rope(act, M, nq, nk, rope, head_dim=64)
    assert e.value.status == svdq.ERR_UNSUPPORTED_SHAPE
    for kw in (dict(norm_q=None), dict(rope=None), dict(eps=-1.0), dict(eps=float("inf")),
               dict(rope=torch.empty(rope.numel() + 4, dtype=torch.uint8, device="cuda")[4:])):
        args = dict(norm_q=nq, norm_k=nk, rope=rope, eps=EPS)
        args.update(kw)
        with pytest.raises(svdq.SvdqError) as e:
            case.layer.linear_qkv_norm_rope(act, M, args["norm_q"], nk, args["rope"], eps=args["eps"])
        assert e.value.status == svdq.ERR_INVALID_ARGUMENT
    with pytest.raises(svdq.SvdqError) as e:  # a table packed for fewer rows
        case.layer.linear_qkv_norm_rope(act, M, nq, nk, rope[:svdq.rope_packed_bytes(1) // 2])
    assert e.value.status == svdq.ERR_BUFFER_TOO_SMALL
    # still usable afterwards
    Y = case.layer.linear_qkv_norm_rope(act, M, nq, nk, rope)
    torch.cuda.synchronize()
    _check(case, Y, check_act(case, act), host)
    case.layer.poll_status()
