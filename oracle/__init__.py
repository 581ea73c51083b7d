"""Plain, slow, fp64 CPU oracle for the SVDQuant W4A4 + low-rank linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code,
tables or helpers with the CUDA/C++ library under ``bit_w4a4_quantized_b200``.

Sources (the SVDQuant summary page, hoonably.github.io/blog/svdquant):
  * section 3 "Quantization preliminary": the quantizer Q_X = round(X / s_X),
    s_X = max|X| / q_max, and q_max = 6 for 4-bit floating point;
    XW ~ s_X s_W Q_X Q_W.
  * section 4.1 "Problem formulation": the error E(X, W) and its bound.
  * section 4.2 "SVDQuant: absorbing outliers via low-rank branch": smoothing
    (migrate outliers from X to W), W_hat = L1 L2 + R with L1 = U Sigma_r,
    L2 = V_r^T, and XW = X_hat L1 L2 + X_hat R ~ X_hat L1 L2 + Q(X_hat) Q(R).
  * section 4.3 "Nunchaku": the down projection shares the activation read of
    the quantizer, the up projection is added into the 4-bit GEMM output.
The abstract record of arXiv 2411.05007 adds: LoRA adapters attach to the
low-rank branch without re-quantizing R.  The Diffusers/Nunchaku page adds:
NVFP4 (Blackwell), compute dtype bfloat16, QKV fusion along the output dim,
and (fused-QKV section) one fused operator for the QKV projection, the Q/K
normalization and the rotary embedding: ``qkv`` restates that operator.  The
same page's second kernel family, awq_w4a16 (4-bit weights, 16-bit
activations, for the modulation projections), is restated in ``w4a16``; the
INT4 variant of the 4-bit family (``--precision int4``) in ``int4``.

Every reading the pages leave open (NVFP4 two-level scales, rounding, sign of
zero, static activation scale, ...) is stated in the
docstrings of ``formats`` and ``svdquant``.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, independent library casts (ml_dtypes, torch, LAPACK
drivers) and brute force; none is "parity unpinned".
"""

from . import formats, svdquant  # noqa: F401
