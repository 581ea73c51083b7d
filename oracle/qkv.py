"""Per-head RMSNorm of Q and K and the rotary embedding, after the fused QKV projection.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).  Plain NumPy in float64.

Source: the Diffusers/Nunchaku page, fused-QKV section.  FLUX's to_q, to_k and
to_v are concatenated along the output dimension, in that order, into one
quantized to_qkv layer, and Nunchaku hands that projection, the normalization
modules norm_q / norm_k and the image rotary embedding to a single fused
operator (fused_qkv_norm_rottary).  The page names the operator and its
operands, not its arithmetic.  The readings taken here:

  * The projection's result is rounded to bfloat16 first, exactly as the plain
    layer returns it; the fused operator then works on those values.
  * Its N columns split into Q, K and V of N / 3 columns each, and each of
    those into heads of ``head_dim`` consecutive columns (FLUX: 128).
  * RMSNorm per Q head and per K head over its ``head_dim`` values:
    z = y / sqrt(mean(y^2) + eps) * w, with w = norm_q for Q and norm_k for K
    (one weight vector of ``head_dim`` values shared by all heads), eps = 1e-6.
  * Rotary embedding of Q and K after the norm.  Row m of the angle table holds
    (cos, sin) for each adjacent pair (2i, 2i + 1) of a head; the pair turns by
    that angle: (z0 cos - z1 sin, z1 cos + z0 sin).
  * V passes through unchanged.
  * The fused kernel rounds each output to bfloat16 once, at the end; this
    oracle returns the float64 values before that rounding.
"""

import numpy as np

HEAD_DIM = 128
EPS = 1e-6


def split_heads(y, head_dim):
    """[M, C] -> [M, C / head_dim, head_dim] (a view)."""
    M, C = y.shape
    if C % head_dim:
        raise ValueError("columns must be whole heads")
    return y.reshape(M, C // head_dim, head_dim)


def rms_norm_heads(y, w, eps):
    """z = y / sqrt(mean(y^2) + eps) * w over the last axis of [M, H, D]."""
    ms = np.mean(y * y, axis=-1, keepdims=True)
    return y / np.sqrt(ms + eps) * np.asarray(w, np.float64)[None, None, :]


def rotate_pairs(z, rope):
    """Turn adjacent pairs (2i, 2i + 1) of [M, H, D] by the angles of rope [M, D/2, 2]."""
    c = rope[:, None, :, 0]
    s = rope[:, None, :, 1]
    z0 = z[..., 0::2]
    z1 = z[..., 1::2]
    out = np.empty_like(z)
    out[..., 0::2] = z0 * c - z1 * s
    out[..., 1::2] = z1 * c + z0 * s
    return out


def qkv_norm_rope(y, norm_q, norm_k, rope, eps=EPS, head_dim=HEAD_DIM):
    """Q/K RMSNorm + rotary embedding of the fused QKV output y [M, 3 C].

    y: the projection's output (bf16 values, as float), rope: float32
    [M, head_dim / 2, 2] (cos, sin), norm_q / norm_k: [head_dim].  Returns
    float64 [M, 3 C]: normalized and rotated Q and K, V unchanged.
    """
    y = np.asarray(y, np.float64)
    rope = np.asarray(rope, np.float64)
    M, N = y.shape
    if N % 3 or (N // 3) % head_dim or head_dim % 2:
        raise ValueError("N must be 3 x whole heads of an even head_dim")
    if rope.shape != (M, head_dim // 2, 2):
        raise ValueError("rope must be [M, head_dim / 2, 2]")
    C = N // 3
    out = y.copy()
    for part, w in ((0, norm_q), (1, norm_k)):
        cols = slice(part * C, (part + 1) * C)
        z = rms_norm_heads(split_heads(y[:, cols], head_dim), w, eps)
        out[:, cols] = rotate_pairs(z, rope).reshape(M, C)
    return out
