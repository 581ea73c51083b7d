"""The SVDQuant W4A4 linear layer with a 16-bit low-rank branch, step by step.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).  Plain NumPy, float64
unless a step is defined in float32 (every quantization decision is taken in
float32, the precision of the kernels).

Layout convention: W is given like ``nn.Linear`` weights, [N, K] (out x in).
The pages' W (m x n, input dim first) is therefore W^T here, and smoothing
scales input channel j of both X and W^T:

    X_hat   = X . diag(lambda)^-1                (section 4.2, "Migrate outliers")
    W_hat^T = diag(lambda) . W^T
    W_hat^T = L1 L2 + R,  L1 = U_r Sigma_r [K, r],  L2 = V_r^T [r, N]
                                                 (section 4.2, eq. W_hat = L1 L2 + R)
    Y       = Q(X_hat) Q(R) + (X_hat L1) L2 + b  (section 4.2, decomposition of XW)

Readings of what the pages leave open:
  * lambda_j = sqrt(max|X_:,j| / max|W_:,j|) (SmoothQuant migration strength
    1/2), 1 where either maximum is 0; every step correctly rounded float32.
  * Sigma goes wholly into L1 (L1 = U Sigma_r, as the page writes it); L1 and
    L2 are rounded to bfloat16 (the "16-bit branch") straight from float64.
  * R uses the bfloat16 factors, so W_hat = L1 L2 + R holds for the operands
    actually multiplied; R is formed in float64 as W_hat^T minus the rank-one
    terms L1[:, j] L2[j, :] subtracted in order j = 0 .. r-1.
  * Q is NVFP4: the page's quantizer (s = max|X| / q_max, q_max = 6) applied
    per 16 consecutive elements along K with an E4M3 block scale, under a
    float32 per-tensor scale g = amax / (6 * 448) (1 if amax is 0).  The
    element code is E2M1(t * rcp(d)) with d = E4M3(s_b) * g.
  * The activation tensor scale is static: set once from calibration maxima.
  * X_hat is rounded to bfloat16 and that one X_hat feeds both branches.
  * Output: act(alpha * sum_k deqA deqW + (X_hat L1) L2 + b), alpha = g_a g_w,
    act in {identity, tanh-GELU}.
"""

from dataclasses import dataclass, field

import numpy as np

from .formats import (
    bf16,
    e2m1_decode,
    e2m1_encode,
    e4m3_decode,
    e4m3_encode,
)

BLOCK = 16  # elements per E4M3 block scale, along K
Q_MAX = np.float32(6.0)  # largest E2M1 magnitude (page: q_max = 6 for FP4)
E4M3_MAX = np.float32(448.0)
GLOBAL_DIV = np.float32(6.0 * 448.0)  # 2688: block scales then fit E4M3

EPI_NONE = 0
EPI_GELU_TANH = 1


# --------------------------------------------------------------------------
# rounding helpers (float64 -> bfloat16 directly, no intermediate float32)
# --------------------------------------------------------------------------


def bf16_from_f64(x):
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    bfloat16 keeps 8 significant bits with binary32's exponent range; values
    below the smallest normal (2^-126) round on the subnormal grid 2^-133.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    tiny = np.abs(x) < 2.0**-126
    # normal range: round the 53-bit significand to 8 bits at bit 45
    u = x.view(np.uint64).copy()
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    u = (u + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    out[...] = u.view(np.float64)
    step = 2.0**-133
    out[tiny] = np.round(x[tiny] / step) * step  # np.round: half to even
    return out


# --------------------------------------------------------------------------
# NVFP4 quantizer (section 3 quantizer, applied per 16-element block)
# --------------------------------------------------------------------------


def global_scale(amax):
    """Per-tensor float32 scale g = f32(amax / 2688); 1 when amax is 0."""
    a = np.float32(amax)
    if a == 0:
        return np.float32(1.0)
    return np.float32(a / GLOBAL_DIV)


def nvfp4_quantize(t, g):
    """Quantize rows of a float32 [rows, K] matrix along K (K % 16 == 0).

    Per block of 16: amax_b = max|t|; s_b = E4M3(f32(amax_b * c)) with
    c = f32(1 / f32(6 g)); d = f32(value(s_b) * g); rcp = 0 if d == 0 else
    f32(1 / d); code = E2M1(f32(t * rcp)).

    Returns (codes uint8 [rows, K] one 4-bit code per element,
             scales uint8 [rows, K / 16] E4M3 codes).
    """
    t = np.asarray(t, dtype=np.float32)
    rows, k = t.shape
    assert k % BLOCK == 0
    g = np.float32(g)
    blocks = t.reshape(rows, k // BLOCK, BLOCK)
    amax = np.max(np.abs(blocks), axis=2)
    c = np.float32(np.float32(1.0) / np.float32(np.float32(6.0) * g))
    s_code = e4m3_encode((amax * c).astype(np.float32))
    d = (e4m3_decode(s_code).astype(np.float32) * g).astype(np.float32)
    safe_d = np.where(d == 0, np.float32(1.0), d)
    rcp = np.where(d == 0, np.float32(0.0), np.float32(1.0) / safe_d).astype(np.float32)
    codes = e2m1_encode((blocks * rcp[..., None]).astype(np.float32))
    return codes.reshape(rows, k), s_code


def nvfp4_dequantize(codes, scales):
    """Block values e2m1(code) * e4m3(scale) in float64 (exact), without g."""
    codes = np.asarray(codes)
    rows, k = codes.shape
    vals = e2m1_decode(codes).reshape(rows, k // BLOCK, BLOCK)
    return (vals * e4m3_decode(scales)[..., None]).reshape(rows, k)


# --------------------------------------------------------------------------
# smoothing (section 4.2, "Migrate outliers from activation to weight")
# --------------------------------------------------------------------------


def smoothing_factors(act_amax, w_amax):
    """lambda_j = f32(sqrt(f32(a_j / w_j))) (1 where a_j or w_j is 0), 1/lambda."""
    a = np.asarray(act_amax, dtype=np.float32)
    w = np.asarray(w_amax, dtype=np.float32)
    ok = (a > 0) & (w > 0)
    ratio = (a / np.where(ok, w, np.float32(1.0))).astype(np.float32)
    lam = np.where(ok, np.sqrt(ratio).astype(np.float32), np.float32(1.0)).astype(np.float32)
    inv_lam = (np.float32(1.0) / lam).astype(np.float32)
    return lam, inv_lam


# --------------------------------------------------------------------------
# low-rank branch (section 4.2, "Absorb magnified weight outliers")
# --------------------------------------------------------------------------


def low_rank_factors(w_hat_t, rank):
    """Top-``rank`` SVD factors of W_hat^T [K, N]: L1 = U_r Sigma_r, L2 = V_r^T."""
    u, s, vt = np.linalg.svd(np.asarray(w_hat_t, dtype=np.float64), full_matrices=False)
    l1 = u[:, :rank] * s[:rank]
    l2 = vt[:rank, :].copy()
    return l1, l2, s


def residual(w_hat_t, l1, l2):
    """R = W_hat^T - L1 L2, rank-one terms subtracted in order j = 0 .. r-1.

    (Done in blocks of rows so that no full-size temporary is made; every
    element sees the same subtractions in the same order.)
    """
    r = np.array(w_hat_t, dtype=np.float64, copy=True)
    for k0 in range(0, r.shape[0], 512):
        blk = r[k0:k0 + 512]
        for j in range(l1.shape[1]):
            blk -= np.outer(l1[k0:k0 + 512, j], l2[j, :])
    return r


# --------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------


@dataclass
class Layer:
    """Everything a prepared layer holds, in logical (unswizzled) layouts."""

    K: int
    N: int
    rank: int
    lam: np.ndarray  # f32 [K]
    inv_lam: np.ndarray  # f32 [K]
    L1_base: np.ndarray  # bf16 values (f64) [K, r]
    L2_base: np.ndarray  # bf16 values (f64) [r, N]
    R: np.ndarray  # f64 [K, N]
    w_codes: np.ndarray  # uint8 [N, K] E2M1 codes of R^T
    w_scales: np.ndarray  # uint8 [N, K/16] E4M3 codes
    g_w: np.float32
    g_a: np.float32
    bias: np.ndarray = None  # bf16 values (f64) [N] or None
    sigma: np.ndarray = None  # singular values of W_hat^T (when computed here)
    L1_lora: np.ndarray = field(default=None)  # [K, r_e] after attach
    L2_lora: np.ndarray = field(default=None)  # [r_e, N]

    @property
    def L1(self):
        if self.L1_lora is None:
            return self.L1_base
        return np.concatenate([self.L1_base, self.L1_lora], axis=1)

    @property
    def L2(self):
        if self.L2_lora is None:
            return self.L2_base
        return np.concatenate([self.L2_base, self.L2_lora], axis=0)

    @property
    def alpha(self):
        return np.float64(self.g_a) * np.float64(self.g_w)

    @property
    def deq_w(self):
        """Dequantized Q(R)^T block values [N, K] (computed once per layer)."""
        if getattr(self, "_deq_w", None) is None:
            self._deq_w = nvfp4_dequantize(self.w_codes, self.w_scales)
        return self._deq_w


def act_global_scale(act_amax, inv_lam):
    """Static g_a: max over j of bf16(f32(a_j / lambda_j)) over 2688.

    Rounding is monotone, so this equals max|X_hat| of the calibration rows.
    """
    xh = bf16((np.asarray(act_amax, np.float32) * inv_lam).astype(np.float32))
    return global_scale(np.max(xh) if xh.size else 0.0)


def prepare(W, act_amax, rank, bias=None, factors=None, out_rows=None):
    """Offline preparation of one layer.

    W: [N, K] bfloat16 values (any float dtype holding them).
    act_amax: float32 [K], max|X_:,j| over calibration rows.
    factors: optional (L1 [K, r], L2 [r, N]) bfloat16 values to use instead of
             this module's SVD (the weights of a checkpoint, say).
    out_rows: optional subset of the N output features to keep (for shapes too
             large to prepare whole here).  lambda comes from the whole weight
             and R's kept columns from the rank-one order above; g_w =
             max|R| / 2688 takes the maximum of W_hat^T - L1 L2 evaluated
             with one matrix product (it can differ from the rank-one order
             only in the last bits, and enters a test only through Y, which
             is compared within its tolerance).  Only the kept rows of R^T are
             quantized, and L2, the bias and N are restricted to them.
    """
    W = np.asarray(W, dtype=np.float64)
    n, k = W.shape
    w_amax = np.max(np.abs(W), axis=0).astype(np.float32)
    lam, inv_lam = smoothing_factors(act_amax, w_amax)
    w_hat_t = lam.astype(np.float64)[:, None] * W.T  # exact: f32 x bf16
    sigma = None
    if factors is None:
        if rank > 0:
            l1, l2, sigma = low_rank_factors(w_hat_t, rank)
            l1b, l2b = bf16_from_f64(l1), bf16_from_f64(l2)
        else:
            l1b, l2b = np.zeros((k, 0)), np.zeros((0, n))
    else:
        l1b = np.asarray(factors[0], dtype=np.float64)
        l2b = np.asarray(factors[1], dtype=np.float64)
        assert l1b.shape == (k, rank) and l2b.shape == (rank, n)
    cols = np.arange(n) if out_rows is None else np.asarray(out_rows)
    if out_rows is None:
        r = residual(w_hat_t, l1b, l2b)
        amax_r = np.max(np.abs(r)) if r.size else 0.0
    else:
        r = residual(w_hat_t[:, cols], l1b, l2b[:, cols])
        amax_r = np.max(np.abs(w_hat_t - l1b @ l2b)) if w_hat_t.size else 0.0
    del w_hat_t
    g_w = global_scale(np.float32(amax_r))  # max commutes with the (monotone) f32 rounding
    w_codes, w_scales = nvfp4_quantize(np.ascontiguousarray(r.T.astype(np.float32)), g_w)
    g_a = act_global_scale(act_amax, inv_lam)
    b = None if bias is None else np.asarray(bias, dtype=np.float64)[cols]
    return Layer(k, len(cols), rank, lam, inv_lam, l1b, l2b[:, cols], r, w_codes, w_scales, g_w, g_a, b, sigma)


def attach_lora(layer, A, B, scale=1.0):
    """Concatenate a LoRA adapter onto the low-rank branch; R is not touched.

    X A B = X_hat (diag(lambda) A) B, so A is smoothed like W^T:
    A'_{j,i} = bf16(f32(f32(lambda_j * A_{j,i}) * scale)).  L1' = [L1 | A'],
    L2' = [L2 ; B].  (Abstract of arXiv 2411.05007: LoRAs without
    re-quantization.)
    """
    A32 = np.asarray(A, dtype=np.float32)
    prod = (layer.lam[:, None] * A32).astype(np.float32)
    prod = (prod * np.float32(scale)).astype(np.float32)
    layer.L1_lora = bf16(prod).astype(np.float64)
    layer.L2_lora = np.asarray(B, dtype=np.float64)
    return layer


def detach_lora(layer):
    layer.L1_lora = None
    layer.L2_lora = None
    return layer


@dataclass
class Act:
    x_hat: np.ndarray  # bf16 values (f32) [M, K]
    codes: np.ndarray  # uint8 [M, K]
    scales: np.ndarray  # uint8 [M, K/16]
    lr: np.ndarray  # f64 [M, r_tot] = X_hat L1


def quantize_act(layer, X):
    """Kernel-1 semantics: smoothing, NVFP4 of X_hat, down projection X_hat L1."""
    X = np.asarray(X, dtype=np.float32)
    x_hat = bf16((X * layer.inv_lam[None, :]).astype(np.float32))
    codes, scales = nvfp4_quantize(x_hat, layer.g_a)
    lr = x_hat.astype(np.float64) @ layer.L1
    return Act(x_hat, codes, scales, lr)


def gelu_tanh(x):
    """Textbook tanh GELU: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x**3)))


def linear(layer, act, epilogue=EPI_NONE, rows=None):
    """Kernel-2 semantics in float64: alpha * Q(X_hat) Q(R) + (X_hat L1) L2 + b.

    ``rows`` restricts the output to a subset of rows (for large shapes).
    """
    codes, scales, lr = act.codes, act.scales, act.lr
    if rows is not None:
        codes, scales, lr = codes[rows], scales[rows], lr[rows]
    deq_a = nvfp4_dequantize(codes, scales)
    y = layer.alpha * (deq_a @ layer.deq_w.T) + lr @ layer.L2
    if layer.bias is not None:
        y = y + layer.bias[None, :]
    if epilogue == EPI_GELU_TANH:
        y = gelu_tanh(y)
    return y


def forward(layer, X, epilogue=EPI_NONE):
    return linear(layer, quantize_act(layer, X), epilogue)


def mlp_pair(layer1, layer2, X):
    """Two layers of a transformer MLP run as one fused pair (Diffusers/Nunchaku page, the
    fused GELU/MLP path of the 4-bit kernel family).  Fusion moves where fc2's activation
    quantization happens (into fc1's output tile), not what it computes, so the pair is the
    composition of the two layers:

        h    = bf16(GELU(fc1(X)))        fc1's output in its output type, rounded once
        act2 = quantize_act(fc2, h)      fc2's smoothing, NVFP4 codes and scales, h_hat L1
        Y    = linear(fc2, act2)

    Returns (h as float32 holding bf16 values, act2, Y in float64).
    """
    h = bf16_from_f64(forward(layer1, X, EPI_GELU_TANH)).astype(np.float32)
    act2 = quantize_act(layer2, h)
    return h, act2, linear(layer2, act2)


# --------------------------------------------------------------------------
# error measures (section 4.1, "Problem formulation")
# --------------------------------------------------------------------------


def quant_error(XW, Y):
    """E = || XW - Y ||_F."""
    return float(np.linalg.norm(np.asarray(XW, np.float64) - np.asarray(Y, np.float64)))


def error_bound(X, W, QX, QW):
    """||X|| ||W - QW|| + ||X - QX|| (||W|| + ||W - QW||) (Frobenius norms)."""
    n = np.linalg.norm
    dw = n(W - QW)
    return float(n(X) * dw + n(X - QX) * (n(W) + dw))


def max_rel_err(y, y_ref):
    """max|y - y_ref| / max|y_ref| (the tolerance metric of the parity tests)."""
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    den = np.max(np.abs(y_ref))
    return float(np.max(np.abs(y - y_ref)) / (den if den > 0 else 1.0))
