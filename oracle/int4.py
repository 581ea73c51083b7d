"""The INT4 variant of the SVDQuant W4A4 layer, step by step.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The Diffusers/Nunchaku page names two variants of the 4-bit kernel family
(svdq_w4a4): NVFP4 for Blackwell and INT4 for the generations before it, with
``--precision int4|nvfp4`` choosing between them when a model is quantized.
Everything but the 4-bit format is the layer of ``oracle.svdquant``: the same
smoothing, the same 16-bit low-rank branch (L1, L2 in bfloat16), the same
residual R.  Only the quantizer Q changes.

The SVDQuant summary page gives the quantizer (section 3, "Quantization
preliminary"): Q_X = round(X / s_X) with s_X = max|X| / q_max, and the product
of two quantized tensors is the scales times the integer product.  For INT4 the
pages fix neither q_max, the granularity nor the scale type.  Readings:

  * q_max = 7, the largest magnitude of a signed 4-bit integer used
    symmetrically (codes -7 .. 7; -8 is never produced).
  * One scale per group of 64 consecutive elements along K (per row of X_hat,
    per output row of R^T).
  * The scale is stored in bfloat16, the layer's compute dtype ("compute_dtype:
    bfloat16" in the page's quantization_config): s = bf16(f32(amax / 7)).
  * As for NVFP4, the division X / s is a multiplication by the correctly
    rounded float32 reciprocal: q = clamp(rne(f32(x * f32(1 / s))), -7, 7);
    a group whose scale is 0 gets q = 0.  (rne: round half to even.)
  * No per-tensor scale: a bfloat16 scale has float32's exponent range.
  * Output: act( sum_g s_a[m,g] s_w[n,g] sum_{k in g} q_a[m,k] q_w[n,k]
                 + (X_hat L1) L2 + b ),  act in {identity, tanh-GELU}.

Every quantization decision is taken in float32, like the kernels; products
and sums are in float64 here (exact for the integer products).
"""

from dataclasses import dataclass

import numpy as np

from .formats import bf16, bf16_from_bits, bf16_bits
from .svdquant import (
    EPI_GELU_TANH,
    bf16_from_f64,
    gelu_tanh,
    low_rank_factors,
    residual,
    smoothing_factors,
)

GROUP = 64  # elements per INT4 scale, along K
Q_MAX = 7  # largest code magnitude


def int4_quantize(t):
    """Quantize rows of a float32 [rows, K] matrix along K (K % 64 == 0).

    Per group of 64: amax = max|t|; s = bf16(f32(amax / 7)); rcp = 0 if s == 0
    else f32(1 / s); q = clamp(rne(f32(t * rcp)), -7, 7).

    Returns (codes int8 [rows, K], scale bits uint16 [rows, K / 64]).
    """
    t = np.asarray(t, dtype=np.float32)
    rows, k = t.shape
    assert k % GROUP == 0
    groups = t.reshape(rows, k // GROUP, GROUP)
    amax = np.max(np.abs(groups), axis=2)
    s_bits = bf16_bits((amax / np.float32(Q_MAX)).astype(np.float32))
    s = bf16_from_bits(s_bits)
    safe = np.where(s == 0, np.float32(1.0), s)
    rcp = np.where(s == 0, np.float32(0.0), (np.float32(1.0) / safe).astype(np.float32)).astype(np.float32)
    prod = (groups * rcp[..., None]).astype(np.float32)
    q = np.clip(np.rint(prod.astype(np.float64)), -Q_MAX, Q_MAX).astype(np.int8)
    return q.reshape(rows, k), s_bits


def int4_dequantize(codes, scale_bits):
    """q * s per group, float64 (exact: a 4-bit integer times a bfloat16 value)."""
    codes = np.asarray(codes, dtype=np.int8)
    rows, k = codes.shape
    s = bf16_from_bits(scale_bits).astype(np.float64)
    return (codes.astype(np.float64).reshape(rows, k // GROUP, GROUP) * s[..., None]).reshape(rows, k)


@dataclass
class Int4Layer:
    """A prepared INT4 layer in logical (unswizzled) layouts."""

    K: int
    N: int
    rank: int
    lam: np.ndarray  # f32 [K]
    inv_lam: np.ndarray  # f32 [K]
    L1: np.ndarray  # bf16 values (f64) [K, r]
    L2: np.ndarray  # bf16 values (f64) [r, N]
    R: np.ndarray  # f64 [K, N]
    w_codes: np.ndarray  # int8 [N, K], -7 .. 7
    w_scales: np.ndarray  # uint16 bf16 bits [N, K / 64]
    bias: np.ndarray = None  # bf16 values (f64) [N] or None

    @property
    def deq_w(self):
        if getattr(self, "_deq_w", None) is None:
            self._deq_w = int4_dequantize(self.w_codes, self.w_scales)
        return self._deq_w


def prepare(W, act_amax, rank, bias=None, factors=None):
    """Offline preparation, as ``oracle.svdquant.prepare`` up to the residual R, then
    the INT4 quantizer on R^T (rows = output features, groups of 64 along K)."""
    W = np.asarray(W, dtype=np.float64)
    n, k = W.shape
    w_amax = np.max(np.abs(W), axis=0).astype(np.float32)
    lam, inv_lam = smoothing_factors(act_amax, w_amax)
    w_hat_t = lam.astype(np.float64)[:, None] * W.T  # exact: f32 x bf16
    if factors is None:
        if rank > 0:
            l1, l2, _ = low_rank_factors(w_hat_t, rank)
            l1b, l2b = bf16_from_f64(l1), bf16_from_f64(l2)
        else:
            l1b, l2b = np.zeros((k, 0)), np.zeros((0, n))
    else:
        l1b = np.asarray(factors[0], dtype=np.float64)
        l2b = np.asarray(factors[1], dtype=np.float64)
        assert l1b.shape == (k, rank) and l2b.shape == (rank, n)
    r = residual(w_hat_t, l1b, l2b)
    w_codes, w_scales = int4_quantize(np.ascontiguousarray(r.T.astype(np.float32)))
    b = None if bias is None else np.asarray(bias, dtype=np.float64)
    return Int4Layer(k, n, rank, lam, inv_lam, l1b, l2b, r, w_codes, w_scales, b)


@dataclass
class Act:
    x_hat: np.ndarray  # bf16 values (f32) [M, K]
    codes: np.ndarray  # int8 [M, K]
    scales: np.ndarray  # uint16 bf16 bits [M, K / 64]
    lr: np.ndarray  # f64 [M, r] = X_hat L1


def quantize_act(layer, X):
    """Kernel-1 semantics: smoothing, INT4 of X_hat, down projection X_hat L1."""
    X = np.asarray(X, dtype=np.float32)
    x_hat = bf16((X * layer.inv_lam[None, :]).astype(np.float32))
    codes, scales = int4_quantize(x_hat)
    lr = x_hat.astype(np.float64) @ layer.L1
    return Act(x_hat, codes, scales, lr)


def linear(layer, act, epilogue=0, rows=None):
    """Kernel-2 semantics in float64: Q(X_hat) Q(R) + (X_hat L1) L2 + b."""
    codes, scales, lr = act.codes, act.scales, act.lr
    if rows is not None:
        codes, scales, lr = codes[rows], scales[rows], lr[rows]
    y = int4_dequantize(codes, scales) @ layer.deq_w.T + lr @ layer.L2
    if layer.bias is not None:
        y = y + layer.bias[None, :]
    if epilogue == EPI_GELU_TANH:
        y = gelu_tanh(y)
    return y


def forward(layer, X, epilogue=0):
    return linear(layer, quantize_act(layer, X), epilogue)
