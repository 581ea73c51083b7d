"""The output bounds the GPU parity tests apply, checked on the CPU with planted mistakes.

The global bound (max|Y - Y_ref| / max|Y_ref|) is set by the largest rows, so a wrong tile of
small outputs can hide under it; the per-row bound must catch that tile, and both must pass
outputs that differ from the reference only by bf16 rounding."""

import numpy as np
import pytest

from gpu_cases import ROW_TOL, Y_TOL, assert_y_close, elementwise_rel_err, row_rel_err
from oracle import formats as F
from oracle import svdquant as S


def _outputs(seed=0):
    g = np.random.default_rng(seed)
    y = g.standard_normal((256, 512))
    y[:4] *= 200.0  # a few outlier rows set the tensor's max
    return y


def test_bf16_rounding_alone_passes_both_bounds():
    y_ref = _outputs()
    y = F.bf16(y_ref.astype(np.float32)).astype(np.float64)
    report = {}
    assert_y_close(y, y_ref, report)
    assert report["row_rel"] <= 2.0**-8 and report["global_rel"] <= 2.0**-8
    assert report["elementwise_rel"] <= 2.0**-8


def test_a_wrong_small_tile_passes_the_global_bound_but_not_the_row_bound():
    y_ref = _outputs()
    y = y_ref.copy()
    y[128:256, 256:384] *= 1.05  # 5 % off, on rows whose scale is 1/200 of the max
    assert S.max_rel_err(y, y_ref) <= Y_TOL
    assert row_rel_err(y, y_ref) > ROW_TOL
    with pytest.raises(AssertionError):
        assert_y_close(y, y_ref)


def test_rows_of_zeros_are_held_to_a_tenth_of_the_rms():
    y_ref = _outputs()
    y_ref[10] = 0.0
    y = y_ref.copy()
    rms = np.sqrt(np.mean(y_ref**2))
    y[10, 3] = 0.5 * ROW_TOL * 0.1 * rms  # inside the absolute floor
    assert row_rel_err(y, y_ref) <= ROW_TOL
    y[10, 3] = 2.0 * ROW_TOL * 0.1 * rms  # beyond it
    assert row_rel_err(y, y_ref) > ROW_TOL


def test_all_zero_reference_and_empty_arrays():
    z = np.zeros((3, 4))
    assert row_rel_err(z, z) == 0.0 and elementwise_rel_err(z, z) == 0.0
    e = np.zeros((0, 4))
    assert row_rel_err(e, e) == 0.0
