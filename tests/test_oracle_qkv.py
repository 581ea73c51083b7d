"""Pins for oracle.qkv (Q/K RMSNorm + rotary embedding after the fused QKV
projection, Diffusers/Nunchaku page, fused-QKV section): closed forms of the
norm, a quarter turn that fixes the pairing and the sign of the rotation,
invariants of a rotation, and a pure-Python brute force.  The mutation tests
at the end plant mistakes in the oracle and check that a pin catches each."""

import math

import numpy as np
import pytest

import bruteforce as BF
from bit_w4a4_quantized_b200 import workloads as WL
from oracle import qkv as Q


def _case(M=5, heads=2, D=8, seed=0, scale=3.0):
    g = np.random.default_rng(seed)
    y = g.standard_normal((M, 3 * heads * D)) * scale
    ang = g.uniform(-np.pi, np.pi, (M, D // 2))
    rope = np.stack([np.cos(ang), np.sin(ang)], -1)
    wq = 1.0 + 0.1 * g.standard_normal(D)
    wk = 1.0 + 0.1 * g.standard_normal(D)
    return y, wq, wk, rope, ang


def _identity_rope(M, D):
    rope = np.zeros((M, D // 2, 2))
    rope[..., 0] = 1.0
    return rope


def test_unit_weights_and_zero_angle_give_unit_rms_heads():
    y, _, _, _, _ = _case(M=7, heads=3, D=16)
    D = 16
    eps = 1e-3
    out = Q.qkv_norm_rope(y, np.ones(D), np.ones(D), _identity_rope(7, D), eps=eps, head_dim=D)
    C = y.shape[1] // 3
    for h0 in range(0, 2 * C, D):
        ms_in = np.mean(y[:, h0:h0 + D] ** 2, axis=1)
        ms_out = np.mean(out[:, h0:h0 + D] ** 2, axis=1)
        np.testing.assert_allclose(ms_out, ms_in / (ms_in + eps), rtol=1e-13)
        # direction kept: out is a positive multiple of y
        np.testing.assert_allclose(out[:, h0:h0 + D], y[:, h0:h0 + D] / np.sqrt(ms_in + eps)[:, None],
                                   rtol=1e-13)
    np.testing.assert_array_equal(out[:, 2 * C:], y[:, 2 * C:])


def test_quarter_turn_fixes_pairing_and_sign():
    # one nonzero value v per Q/K head, eps = 0: the normalized value is
    # sign(v) sqrt(D) w_d; a quarter turn (cos 0, sin 1) takes a pair (z0, z1)
    # to (-z1, z0)
    D, M = 8, 2
    y = np.zeros((M, 3 * D))
    y[0, 0] = 2.5          # Q, element 0 = first of pair 0
    y[0, D + 5] = 1.0      # K, element 5 = second of pair 2
    y[1, 6] = -3.0         # Q, element 6 = first of pair 3
    y[1, D + 3] = -4.0     # K, element 3 = second of pair 1
    wq = np.arange(1, D + 1, dtype=np.float64)
    wk = np.arange(1, D + 1, dtype=np.float64) * 0.5
    rope = np.zeros((M, D // 2, 2))
    rope[..., 1] = 1.0
    out = Q.qkv_norm_rope(y, wq, wk, rope, eps=0.0, head_dim=D)
    r = math.sqrt(D)
    want = np.zeros_like(y)
    want[0, 1] = r * wq[0]          # (z0, 0) -> (0, z0)
    want[0, D + 4] = -r * wk[5]     # (0, z1) -> (-z1, 0)
    want[1, 7] = -r * wq[6]         # z0 = -r wq[6] moves to the second slot
    want[1, D + 2] = r * wk[3]      # z1 = -r wk[3] -> -z1 in the first slot
    np.testing.assert_allclose(out, want, atol=1e-12)


def test_rotation_keeps_pair_norms_and_inverse_angle_undoes_it():
    y, wq, wk, rope, ang = _case(M=6, heads=2, D=16)
    D = 16
    out = Q.qkv_norm_rope(y, wq, wk, rope, head_dim=D)
    ref = Q.qkv_norm_rope(y, wq, wk, _identity_rope(6, D), head_dim=D)
    C = y.shape[1] // 3
    qk = slice(0, 2 * C)
    n_out = np.hypot(out[:, qk][:, 0::2], out[:, qk][:, 1::2])
    n_ref = np.hypot(ref[:, qk][:, 0::2], ref[:, qk][:, 1::2])
    np.testing.assert_allclose(n_out, n_ref, rtol=1e-13)
    # turning back by -angle (eps = 0, unit weights: the norm is then idempotent)
    fwd = Q.qkv_norm_rope(y, np.ones(D), np.ones(D), rope, eps=0.0, head_dim=D)
    back = np.stack([np.cos(-ang), np.sin(-ang)], -1)
    undone = Q.qkv_norm_rope(fwd, np.ones(D), np.ones(D), back, eps=0.0, head_dim=D)
    plain = Q.qkv_norm_rope(y, np.ones(D), np.ones(D), _identity_rope(6, D), eps=0.0, head_dim=D)
    np.testing.assert_allclose(undone, plain, atol=1e-12)


def test_two_turns_compose_into_the_sum_of_angles():
    y, _, _, _, a = _case(M=4, heads=1, D=8, seed=3)
    b = np.random.default_rng(4).uniform(-np.pi, np.pi, a.shape)
    cs = lambda t: np.stack([np.cos(t), np.sin(t)], -1)
    one = np.ones(8)
    twice = Q.qkv_norm_rope(Q.qkv_norm_rope(y, one, one, cs(a), eps=0.0, head_dim=8), one, one, cs(b),
                            eps=0.0, head_dim=8)
    once = Q.qkv_norm_rope(y, one, one, cs(a + b), eps=0.0, head_dim=8)
    np.testing.assert_allclose(twice, once, atol=1e-12)


def test_norm_ignores_the_scale_of_a_head_when_eps_is_zero():
    y, wq, wk, rope, _ = _case(M=3, heads=2, D=8, seed=5)
    C = y.shape[1] // 3
    y2 = y.copy()
    y2[:, :2 * C] *= 37.0
    a = Q.qkv_norm_rope(y, wq, wk, rope, eps=0.0, head_dim=8)
    b = Q.qkv_norm_rope(y2, wq, wk, rope, eps=0.0, head_dim=8)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_brute_force(seed):
    y, wq, wk, rope, _ = _case(M=4, heads=2, D=8, seed=seed)
    want = BF.qkv_norm_rope(y.tolist(), wq.tolist(), wk.tolist(), rope.tolist(), 1e-6, 8)
    got = Q.qkv_norm_rope(y, wq, wk, rope, eps=1e-6, head_dim=8)
    np.testing.assert_allclose(got, np.array(want), rtol=1e-12, atol=1e-12)


def test_workload_tables_have_the_documented_form():
    rope = WL.make_rope(40, 128)
    assert rope.shape == (40, 64, 2) and rope.dtype == np.float32
    np.testing.assert_array_equal(rope[0, :, 0], 1.0)   # position 0: no turn
    np.testing.assert_array_equal(rope[0, :, 1], 0.0)
    np.testing.assert_allclose(rope[..., 0] ** 2 + rope[..., 1] ** 2, 1.0, rtol=1e-6)
    wq, wk = WL.make_norm_weights(128, seed=3)
    assert wq.shape == wk.shape == (128,) and not np.array_equal(wq, wk)


def test_rejects_shapes_that_are_not_whole_heads():
    with pytest.raises(ValueError):
        Q.qkv_norm_rope(np.zeros((2, 3 * 12)), np.ones(8), np.ones(8), np.zeros((2, 4, 2)), head_dim=8)
    with pytest.raises(ValueError):
        Q.qkv_norm_rope(np.zeros((2, 3 * 8)), np.ones(8), np.ones(8), np.zeros((3, 4, 2)), head_dim=8)


# ------------------------------------------------------------------ mutations


def _pins_fail():
    failed = 0
    for t in (test_quarter_turn_fixes_pairing_and_sign, test_unit_weights_and_zero_angle_give_unit_rms_heads,
              lambda: test_matches_brute_force(0)):
        try:
            t()
        except AssertionError:
            failed += 1
    return failed


def _rot_wrong_sign(z, rope):
    c, s = rope[:, None, :, 0], rope[:, None, :, 1]
    out = np.empty_like(z)
    out[..., 0::2] = z[..., 0::2] * c + z[..., 1::2] * s
    out[..., 1::2] = z[..., 1::2] * c - z[..., 0::2] * s
    return out


def _rot_half_pairs(z, rope):
    D = z.shape[-1]
    c, s = rope[:, None, :, 0], rope[:, None, :, 1]
    out = np.empty_like(z)
    out[..., :D // 2] = z[..., :D // 2] * c - z[..., D // 2:] * s
    out[..., D // 2:] = z[..., D // 2:] * c + z[..., :D // 2] * s
    return out


def _norm_no_eps(y, w, eps):
    return y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True)) * np.asarray(w)[None, None, :]


def _norm_no_weight(y, w, eps):
    return y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)


@pytest.mark.parametrize("name,fn", [("rotate_pairs", _rot_wrong_sign), ("rotate_pairs", _rot_half_pairs),
                                     ("rms_norm_heads", _norm_no_eps), ("rms_norm_heads", _norm_no_weight)])
def test_planted_mistakes_are_caught(monkeypatch, name, fn):
    monkeypatch.setattr(Q, name, fn)
    assert _pins_fail() >= 1


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=30, deadline=None)
@given(M=st.integers(1, 4), heads=st.integers(1, 3), half=st.sampled_from([1, 2, 4]), seed=st.integers(0, 10_000),
       eps=st.sampled_from([0.0, 1e-6, 0.5]), scale=st.sampled_from([1e-3, 1.0, 300.0]))
def test_matches_brute_force_on_random_heads(M, heads, half, seed, eps, scale):
    D = 2 * half
    y, wq, wk, rope, _ = _case(M=M, heads=heads, D=D, seed=seed, scale=scale)
    want = BF.qkv_norm_rope(y.tolist(), wq.tolist(), wk.tolist(), rope.tolist(), eps, D)
    got = Q.qkv_norm_rope(y, wq, wk, rope, eps=eps, head_dim=D)
    np.testing.assert_allclose(got, np.array(want), rtol=1e-11, atol=1e-11)
