"""Seeded synthetic inputs for the W4A4 + low-rank linear layer.

This module only draws random numbers (NumPy ``default_rng([seed, stream])``)
and rounds them to bfloat16 inputs; it holds none of the method's arithmetic.
Both the CUDA path (through ``bench.py`` and the tests) and the CPU oracle are
fed from here.

The SVDQuant pages evaluate on FLUX.1 / PixArt / SDXL checkpoints that are
not available; these distributions stand in for their linear-layer inputs:
  * "outlier channels": a few input channels of X scaled up (activation
    outliers), a few input columns of W scaled up (weight outliers) -- the two
    kinds of outliers section 3 of the SVDQuant summary page describes;
  * shapes are the FLUX-like projection shapes of the benchmark workloads.
"""

from dataclasses import dataclass

import ml_dtypes
import numpy as np

BF16 = ml_dtypes.bfloat16

STREAM_X = 0
STREAM_W = 1
STREAM_BIAS = 2
STREAM_X_OUTLIER = 3
STREAM_W_OUTLIER = 4
STREAM_LORA_A = 5
STREAM_LORA_B = 6
STREAM_W2 = 7
STREAM_W2_OUTLIER = 8
STREAM_SAMPLE = 9
STREAM_NORM_Q = 10
STREAM_NORM_K = 11
STREAM_AWQ_S = 12


def rng(seed, stream):
    return np.random.default_rng([int(seed), int(stream)])


def to_bf16(a):
    """float array -> ml_dtypes.bfloat16 array (round to nearest even)."""
    return np.asarray(a, dtype=np.float32).astype(BF16)


def make_x(M, K, seed, dist="normal", n_outlier=4, outlier_scale=40.0, stream=STREAM_X,
           outlier_stream=STREAM_X_OUTLIER):
    """Activations [M, K] bf16: N(0,1) or Student-t(4), ``n_outlier`` channels scaled."""
    g = rng(seed, stream)
    if dist == "normal":
        x = g.standard_normal((M, K), dtype=np.float32)
    elif dist == "student_t4":
        x = g.standard_t(4.0, size=(M, K)).astype(np.float32)
    else:
        raise ValueError(dist)
    if n_outlier:
        idx = rng(seed, outlier_stream).choice(K, size=n_outlier, replace=False)
        x[:, idx] *= np.float32(outlier_scale)
    return to_bf16(x)


def make_w(N, K, seed, n_outlier=4, outlier_scale=20.0, std=0.02, stream=STREAM_W,
           outlier_stream=STREAM_W_OUTLIER):
    """Weights [N, K] bf16 (nn.Linear layout): N(0, std) with outlier input columns."""
    w = rng(seed, stream).standard_normal((N, K), dtype=np.float32) * np.float32(std)
    if n_outlier:
        idx = rng(seed, outlier_stream).choice(K, size=n_outlier, replace=False)
        w[:, idx] *= np.float32(outlier_scale)
    return to_bf16(w)


def make_bias(N, seed, std=0.01):
    return to_bf16(rng(seed, STREAM_BIAS).standard_normal(N, dtype=np.float32) * np.float32(std))


def make_lora(K, N, r_e, seed, std=0.01):
    a = rng(seed, STREAM_LORA_A).standard_normal((K, r_e), dtype=np.float32) * np.float32(std)
    b = rng(seed, STREAM_LORA_B).standard_normal((r_e, N), dtype=np.float32) * np.float32(std)
    return to_bf16(a), to_bf16(b)


def make_norm_weights(head_dim, seed, std=0.1):
    """RMSNorm weights of Q and K: bf16 [head_dim] each, 1 + N(0, std)."""
    q = 1.0 + rng(seed, STREAM_NORM_Q).standard_normal(head_dim) * std
    k = 1.0 + rng(seed, STREAM_NORM_K).standard_normal(head_dim) * std
    return to_bf16(q), to_bf16(k)


def make_rope(M, head_dim, base=10000.0):
    """Rotary angle table float32 [M, head_dim / 2, 2] = (cos, sin) of
    m * base^(-2 i / head_dim) for token m and pair i: one position per row,
    the usual frequency ladder.  A fixed table, no random draws."""
    m = np.arange(M, dtype=np.float64)[:, None]
    freq = base ** (-2.0 * np.arange(head_dim // 2, dtype=np.float64) / head_dim)
    ang = m * freq[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)


def make_awq_scales(K, seed, spread=0.5):
    """Positive per-input-channel scales exp(U(-spread, spread)) for the W4A16 layer (float32)."""
    return np.exp(rng(seed, STREAM_AWQ_S).uniform(-spread, spread, K)).astype(np.float32)


@dataclass(frozen=True)
class W4A16Spec:
    """A W4A16 modulation projection: M conditioning rows, K -> N."""

    name: str
    M: int
    K: int
    N: int
    seed: int

    def x(self):
        return make_x(self.M, self.K, self.seed, n_outlier=0)

    def w(self):
        return make_w(self.N, self.K, self.seed)

    def s(self):
        return make_awq_scales(self.K, self.seed)

    def b(self):
        return make_bias(self.N, self.seed)


def w4a16_spec(M, N=18432, K=3072):
    """FLUX-like modulation projection: 3072 -> 6 x 3072 (double blocks) or 3 x 3072 (single blocks)."""
    return W4A16Spec(f"w4a16_mod_M{M}_K{K}_N{N}", M, K, N, seed=5)


@dataclass(frozen=True)
class LayerSpec:
    """One linear layer of a workload."""

    name: str
    M: int
    K: int
    N: int
    rank: int
    seed: int
    x_dist: str = "normal"
    x_outliers: int = 4
    x_outlier_scale: float = 40.0
    w_outliers: int = 4
    w_outlier_scale: float = 20.0
    bias: bool = False
    gelu: bool = False
    lora_rank: int = 0
    w_stream: int = STREAM_W
    w_outlier_stream: int = STREAM_W_OUTLIER

    @property
    def flops_fp4(self):
        return 2 * self.M * self.N * self.K

    def x(self, M=None):
        return make_x(self.M if M is None else M, self.K, self.seed, self.x_dist,
                      self.x_outliers, self.x_outlier_scale)

    def w(self):
        return make_w(self.N, self.K, self.seed, self.w_outliers, self.w_outlier_scale,
                      stream=self.w_stream, outlier_stream=self.w_outlier_stream)

    def b(self):
        return make_bias(self.N, self.seed) if self.bias else None

    def lora(self):
        return make_lora(self.K, self.N, self.lora_rank, self.seed) if self.lora_rank else None


# The five benchmark configurations (seed = configuration number - 1).
CFG1 = LayerSpec("single_layer_M64_K256_N256_r16", 64, 256, 256, 16, seed=0)
CFG2 = LayerSpec("attn_proj_M4096_K3072_N3072_r32", 4096, 3072, 3072, 32, seed=1,
                 x_dist="student_t4", x_outliers=round(0.01 * 3072), x_outlier_scale=50.0,
                 w_outliers=round(0.005 * 3072), w_outlier_scale=20.0, bias=True)
CFG3_FC1 = LayerSpec("mlp_fc1_M4608_K3072_N12288_r32_gelu", 4608, 3072, 12288, 32, seed=2,
                     gelu=True)
CFG3_FC2 = LayerSpec("mlp_fc2_M4608_K12288_N3072_r32", 4608, 12288, 3072, 32, seed=2,
                     w_stream=STREAM_W2, w_outlier_stream=STREAM_W2_OUTLIER)
CFG4 = LayerSpec("qkv_M4608_K3072_N9216_r32_lora16", 4608, 3072, 9216, 32, seed=3, lora_rank=16)

SWEEP_M = (256, 1024, 4096, 16384)
SWEEP_KN = (3072, 12288)
SWEEP_R = (0, 16, 32, 64)


def sweep_spec(M, KN, r):
    return LayerSpec(f"sweep_M{M}_K{KN}_N{KN}_r{r}", M, KN, KN, r, seed=4)


def sweep():
    return [sweep_spec(m, kn, r) for kn in SWEEP_KN for m in SWEEP_M for r in SWEEP_R]


CONFIGS = {1: [CFG1], 2: [CFG2], 3: [CFG3_FC1, CFG3_FC2], 4: [CFG4], 5: sweep()}
