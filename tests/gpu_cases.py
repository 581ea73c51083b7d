"""Shared helpers of the GPU parity tests, __graft_entry__.smoke() and bench.py.

One case = one layer of a workload.  The oracle computes the low-rank factors
(LAPACK SVD) and every expected value; the library receives the same factors
(as a checkpoint would give them), so codes and scales must agree bit for bit
and outputs within the layer tolerance.  Nothing expected here comes from the
CUDA path.
"""

import numpy as np
import torch

from bit_w4a4_quantized_b200 import svdq
from oracle import formats as F
from oracle import svdquant as S

Y_TOL = 1e-2       # max|Y - Y_ref| / max|Y_ref| (the layer tolerance)
ROW_TOL = 1e-2     # the same bound per row, each row against its own max (floored at 0.1 rms of Y_ref)
PAIR_TOL = 0.08    # a fused MLP pair's output against the oracle's pair (max-norm); derived from the oracle's
                   # own sensitivity to one-ulp hidden-state changes in tests/test_oracle_mlp.py
LR_TOL = 2.0**-7   # lr' is rounded to bf16 once: relative error <= 2^-9, margin for fp32 sums


def oracle_factors(W32, amax, r):
    if r == 0:
        K, N = W32.shape[1], W32.shape[0]
        return np.zeros((K, 0)), np.zeros((0, N))
    lam, _ = S.smoothing_factors(amax, np.max(np.abs(W32), 0))
    l1, l2, _ = S.low_rank_factors(lam.astype(np.float64)[:, None] * W32.T.astype(np.float64), r)
    return S.bf16_from_f64(l1), S.bf16_from_f64(l2)


class Case:
    """Oracle layer + library layer built from the same inputs and factors."""

    def __init__(self, X, W, r, bias=None, rank_capacity=None, device="cuda"):
        self.X = X  # ml_dtypes bf16 [M, K]
        self.W = W
        self.X32 = X.astype(np.float32)
        self.W32 = W.astype(np.float32)
        self.amax = np.max(np.abs(self.X32), axis=0)
        self.r = r
        l1b, l2b = oracle_factors(self.W32, self.amax, r)
        b64 = None if bias is None else bias.astype(np.float64)
        self.ref = S.prepare(self.W32, self.amax, r, bias=b64, factors=(l1b, l2b))
        lib_factors = None
        if r:
            lib_factors = (F.bf16_bits(l1b.astype(np.float32)), F.bf16_bits(l2b.astype(np.float32)))
        self.layer = svdq.Layer(W, self.amax, r, rank_capacity=rank_capacity, bias=bias, factors=lib_factors,
                                device=device)
        self.Xd = torch.from_numpy(X.view(np.uint16).astype(np.int16)).view(torch.bfloat16).to(device)

    def run(self, epilogue=svdq.EPI_NONE, X=None):
        Xd = self.Xd if X is None else X
        act = self.layer.quantize_act(Xd)
        Y = self.layer.linear(act, Xd.shape[0], epilogue=epilogue)
        torch.cuda.synchronize()
        return act, Y

    def unpack(self, act, M):
        return self.layer.act_unpack(act.cpu().numpy(), M)


def y_to_f64(Y):
    return Y.float().cpu().numpy().astype(np.float64)


def check_act(case, act, rows=None):
    """Codes and scales bit-exact, lr' within bf16 tolerance (optionally on a row subset)."""
    M = case.X.shape[0]
    codes, scales, lr = case.unpack(act, M)
    X32 = case.X32 if rows is None else case.X32[rows]
    ref = S.quantize_act(case.ref, X32)
    sel = slice(None) if rows is None else rows
    np.testing.assert_array_equal(codes[sel], F.pack_e2m1(ref.codes))
    np.testing.assert_array_equal(scales[sel], ref.scales)
    if case.ref.L1.shape[1]:
        lr_gpu = F.bf16_from_bits(lr[sel]).astype(np.float64) * case.ref.alpha
        den = max(np.max(np.abs(ref.lr)), 1e-30)
        assert np.max(np.abs(lr_gpu - ref.lr)) <= LR_TOL * den
    return ref


def row_rel_err(y, y_ref):
    """max over rows i of max_j|y - y_ref|_ij / max(max_j|y_ref|_ij, 0.1 rms(y_ref)).

    The global bound divides by the tensor's max, which a few outlier rows set; a whole tile of
    small outputs could be off by percents of its own scale under it.  Here each row answers to
    its own scale, floored at a tenth of the tensor's rms so that rows of near-zero outputs are
    held to an absolute bound instead of a relative one."""
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    if y_ref.size == 0:
        return 0.0
    floor = 0.1 * float(np.sqrt(np.mean(y_ref * y_ref)))
    den = np.maximum(np.max(np.abs(y_ref), axis=-1), floor)
    den = np.where(den > 0, den, 1.0)
    return float(np.max(np.max(np.abs(y - y_ref), axis=-1) / den))


def elementwise_rel_err(y, y_ref):
    """max |y - y_ref| / |y_ref| over the elements with |y_ref| >= 0.1 rms(y_ref) (a report, not a bound:
    near zero crossings bf16 output rounding alone makes this ratio large)."""
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    if y_ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(y_ref * y_ref)))
    sel = np.abs(y_ref) >= 0.1 * rms
    if not np.any(sel) or rms == 0:
        return 0.0
    return float(np.max(np.abs(y[sel] - y_ref[sel]) / np.abs(y_ref[sel])))


def assert_y_close(y, y_ref, report=None):
    """Both bounds on float64 arrays: the global max-norm one and the per-row one; returns the global."""
    err = S.max_rel_err(y, y_ref)
    assert err <= Y_TOL, err
    rerr = row_rel_err(y, y_ref)
    assert rerr <= ROW_TOL, rerr
    if report is not None:
        report.update(global_rel=err, row_rel=rerr, elementwise_rel=elementwise_rel_err(y, y_ref))
    return err


def check_y(case, Y, ref_act, epilogue=svdq.EPI_NONE, rows=None, report=None):
    """Y against the oracle: the global bound and the per-row bound, both asserted; the
    element-wise ratio is added to `report` (a dict) when one is given."""
    y = y_to_f64(Y)
    if rows is not None:
        y = y[rows]
    return assert_y_close(y, S.linear(case.ref, ref_act, epilogue), report)
