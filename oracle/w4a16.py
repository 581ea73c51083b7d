"""W4A16 linear layer: 4-bit weights, 16-bit activations.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).  Plain NumPy, float64
except where a step is defined in float32.

Sources: the Diffusers/Nunchaku page names a second kernel family next to the
W4A4 one, awq_w4a16: 4-bit weights with 16-bit activations, for the adaptive
norm and modulation projections (FLUX adanorm_single / adanorm_zero), which
are memory bound and precision sensitive.  The SVDQuant summary page, section
2 "AWQ", describes AWQ as activation-aware weight quantization that protects
the weights that matter by shifting scale onto the activations; its section 3
notes that W4A16 upcasts the weights, so the gain is memory, not arithmetic.

Readings of what the pages leave open:
  * The 4-bit weights use the NVFP4 encoding of the W4A4 layer's residual:
    E2M1 codes, one E4M3 scale per 16 consecutive weights along K, a float32
    tensor scale g = amax / 2688 (1 when amax is 0).
  * The activation-aware scale is one positive float32 s_j per input channel
    (1 when absent): the quantized weight is W' = f32(W diag(s)), and the
    activations are divided by s at run time, so X W^T = X~ W'^T before
    quantization.  The pages give no rule for choosing s (AWQ searches for it
    offline), so s is an input of the layer.
  * The divided activation is rounded once to a 16-bit operand, as X_hat is in
    the W4A4 layer: x~_j = f16(f32(x_j * f32(1 / s_j))), to nearest, saturating
    at +-65504.  f16 rather than bf16: the dequantized weights (E2M1 times
    E4M3) are exact in f16, the two tensor-core operands share one type, and
    f16 keeps 3 more bits of x~; its range covers the modulation inputs.
  * Y = g * sum_j x~_j deq(W')_nj + b, act = identity, rounded to bf16 once.
"""

from dataclasses import dataclass

import numpy as np

from . import svdquant as S


@dataclass
class W4A16:
    codes: np.ndarray   # uint8 [N, K], one E2M1 code per weight (sign in bit 3)
    scales: np.ndarray  # uint8 [N, K / 16], E4M3
    g: np.float32       # tensor scale
    inv_s: np.ndarray   # float32 [K]
    bias: np.ndarray    # float64 [N] or None
    deq: np.ndarray     # float64 [N, K] = e2m1 * e4m3 (without g)


def prepare(W, s=None, bias=None, rows=None):
    """Quantize W [N, K] (float32 values of bf16 weights) as W' = f32(W diag(s)).

    ``rows`` keeps only those output rows (g still comes from all of W'), for
    large layers checked on sampled outputs.
    """
    W = np.asarray(W, np.float32)
    N, K = W.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    s32 = np.ones(K, np.float32) if s is None else np.asarray(s, np.float32)
    if np.any(~(s32 > 0)) or not np.all(np.isfinite(s32)):
        raise ValueError("s must be positive and finite")
    amax = np.float32(0)
    for r0 in range(0, N, 4096):  # max |W'| in blocks of rows
        blk = (W[r0:r0 + 4096] * s32[None, :]).astype(np.float32)
        amax = max(amax, np.max(np.abs(blk)))
    g = S.global_scale(amax)
    sel = slice(None) if rows is None else rows
    Wp = (W[sel] * s32[None, :]).astype(np.float32)
    codes, scales = S.nvfp4_quantize(Wp, g)
    inv_s = (np.float32(1.0) / s32).astype(np.float32)
    b = None if bias is None else np.asarray(bias, np.float64)[sel]
    return W4A16(codes, scales, np.float32(g), inv_s, b, S.nvfp4_dequantize(codes, scales))


def act_operand(X, inv_s):
    """x~ = f16(f32(x * inv_s)), round to nearest even, saturating at the f16 maximum."""
    t = (np.asarray(X, np.float32) * np.asarray(inv_s, np.float32)[None, :]).astype(np.float32)
    t = np.clip(t, np.float32(-65504.0), np.float32(65504.0))
    return t.astype(np.float16)


def linear(layer, X, rows=None):
    """Y = g * (X~ @ deq^T) + b in float64, X~ = act_operand(X, 1/s)."""
    X = np.asarray(X, np.float32)
    if rows is not None:
        X = X[rows]
    Xt = act_operand(X, layer.inv_s).astype(np.float64)
    y = np.float64(layer.g) * (Xt @ layer.deq.T)
    if layer.bias is not None:
        y = y + layer.bias[None, :]
    return y
