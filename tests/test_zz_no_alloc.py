"""The fused MLP pair through the entry point that allocates nothing (svdq_w4a4_linear_mlp_static).

Callers that cannot allocate device memory use this entry point instead of svdq_w4a4_linear_mlp:
the library's static scratch area stands in for the workspace.  Its results must be those of
the workspace entry point, call after call (the area keeps the previous call's partials, which
must not leak into the next).  This file is collected last, so that a run stopping at the first
failure has run every other test first; it also passes on its own in a fresh process, where its
first call is the one that looks the area up."""

import ctypes

import numpy as np
import pytest
import torch

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL
from gpu_cases import LR_TOL, assert_y_close, y_to_f64
from oracle import formats as F

pytestmark = pytest.mark.gpu


def _layers(M, K1, N1, N2, r1, r2, seed):
    X = WL.make_x(M, K1, seed=seed)
    W1 = WL.make_w(N1, K1, seed=seed)
    W2 = WL.make_w(N2, N1, seed=seed + 1, n_outlier=0)
    fc1 = svdq.Layer(W1, svdq.calibrate_amax(X), r1, bias=WL.make_bias(N1, seed), device="cuda")
    Xd = torch.from_numpy(X.view(np.uint16).astype(np.int16)).view(torch.bfloat16).cuda()
    act1 = fc1.quantize_act(Xd)
    h = fc1.linear(act1, M, epilogue=svdq.EPI_GELU_TANH)  # calibration of fc2 on the hidden state
    amax2 = svdq.calibrate_amax(h.view(torch.int16).cpu().numpy().view(np.uint16).view(WL.BF16))
    fc2 = svdq.Layer(W2, amax2, r2, device="cuda")
    return fc1, fc2, act1


def _static(fc1, act1, M, fc2, act2):
    return svdq.lib().svdq_w4a4_linear_mlp_static(fc1._h, act1.data_ptr(), act1.numel(), M, fc2._h,
                                                  act2.data_ptr(), act2.numel(), svdq.EPI_GELU_TANH,
                                                  torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,K1,N1,N2,r1,r2", [(300, 256, 640, 256, 16, 32), (1000, 512, 1024, 512, 32, 16)])
def test_static_scratch_gives_the_workspace_entry_points_results(M, K1, N1, N2, r1, r2):
    fc1, fc2, act1 = _layers(M, K1, N1, N2, r1, r2, seed=M + N1)
    ref2 = fc1.linear_mlp(act1, M, fc2)  # the entry point with a workspace
    Yref = fc2.linear(ref2, M)
    torch.cuda.synchronize()
    c_r, s_r, lr_r = fc2.act_unpack(ref2.cpu().numpy(), M)
    yref = y_to_f64(Yref)
    for call in range(2):  # the second call finds the first call's partials in the area
        act2 = fc2.new_act_buffer(M)
        assert _static(fc1, act1, M, fc2, act2) == svdq.OK, svdq.last_error()
        Y = fc2.linear(act2, M)
        torch.cuda.synchronize()
        c, sc, lr = fc2.act_unpack(act2.cpu().numpy(), M)
        np.testing.assert_array_equal(c, c_r)
        np.testing.assert_array_equal(sc, s_r)
        a = F.bf16_from_bits(lr).astype(np.float64)
        b = F.bf16_from_bits(lr_r).astype(np.float64)
        assert np.max(np.abs(a - b)) <= LR_TOL * max(np.max(np.abs(b)), 1e-30), call
        assert_y_close(y_to_f64(Y), yref)
    fc1.poll_status()
    fc2.poll_status()


def test_a_pair_larger_than_the_area_is_refused():
    """48 of fc1's weight tiles x 4096 rows x 64 ranks of float partials need 48 MiB > 32 MiB:
    refused before any launch (the activation buffers are not even looked at)."""
    M, N1 = 4096, 12288
    fc1 = svdq.Layer(WL.make_w(N1, 64, seed=3), np.ones(64, np.float32), 0, device="cuda")
    fc2 = svdq.Layer(WL.make_w(64, N1, seed=4), np.ones(N1, np.float32), 64, device="cuda")
    lib = svdq.lib()
    need = ctypes.c_size_t()
    assert lib.svdq_mlp_workspace_bytes(fc1._h, fc2._h, M, ctypes.byref(need)) == svdq.OK
    assert need.value > (32 << 20)
    st = lib.svdq_w4a4_linear_mlp_static(fc1._h, None, 0, M, fc2._h, None, 0, svdq.EPI_GELU_TANH, None)
    assert st == svdq.ERR_UNSUPPORTED_SHAPE
    assert "static area" in svdq.last_error()
