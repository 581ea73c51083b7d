"""The C ABI without a GPU: the library loads, exports exactly what
include/svdq.h declares, validates arguments, and its host-only entry points
work (no CUDA call is made by these tests)."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "svdq.h")).read()
    return sorted(set(re.findall(r"^SVDQ_API\s+[\w\s\*]+?\b(svdq_\w+)\(", text, flags=re.M)))


def test_library_loads_and_reports_version():
    assert svdq.lib().svdq_abi_version() == 1


def test_exports_match_header():
    decl = declared_symbols()
    assert len(decl) >= 18
    assert sorted(svdq.EXPORTED_SYMBOLS) == decl
    L = svdq.lib()
    for name in decl:
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", svdq.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted(l.split()[-1] for l in out.splitlines() if " T " in l and "svdq_" in l)
    assert exported == decl


def _desc(K=256, N=256, rank=16, cap=16):
    W = WL.make_w(N, K, seed=0).view(np.uint16)
    amax = np.ones(K, np.float32)
    d = svdq.PrepareDesc()
    d.K, d.N, d.rank, d.rank_capacity, d.format = K, N, rank, cap, svdq.FMT_NVFP4
    d.W, d.act_amax = W.ctypes.data, amax.ctypes.data
    return d, (W, amax)


@pytest.mark.parametrize("field,value,status", [
    ("K", 100, svdq.ERR_UNSUPPORTED_SHAPE),
    ("N", 0, svdq.ERR_UNSUPPORTED_SHAPE),
    ("rank", 8, svdq.ERR_UNSUPPORTED_SHAPE),
    ("rank_capacity", 8, svdq.ERR_UNSUPPORTED_SHAPE),
    ("rank_capacity", 512, svdq.ERR_UNSUPPORTED_SHAPE),
    ("format", 7, svdq.ERR_INVALID_ARGUMENT),
    ("W", None, svdq.ERR_INVALID_ARGUMENT),
])
def test_prepare_rejects_bad_descriptors(field, value, status):
    d, keep = _desc()
    setattr(d, field, value)
    h = ctypes.c_void_p()
    st = svdq.lib().svdq_prepare_host(ctypes.byref(d), ctypes.byref(h))
    assert st == status
    assert svdq.last_error()
    assert svdq.lib().svdq_layer_device_bytes(ctypes.byref(d)) == 0
    del keep


@pytest.mark.parametrize("bad", [-1.0, float("nan"), float("inf")])
def test_prepare_rejects_bad_calibration_maxima(bad):
    d, (W, amax) = _desc()
    amax[17] = bad
    h = ctypes.c_void_p()
    assert svdq.lib().svdq_prepare_host(ctypes.byref(d), ctypes.byref(h)) == svdq.ERR_INVALID_ARGUMENT
    assert "act_amax[17]" in svdq.last_error()
    assert svdq.lib().svdq_layer_device_bytes(ctypes.byref(d)) == 0


def test_lora_swap_checks_its_arguments_before_the_device():
    """Shape, capacity, missing and misaligned adapters and the scale are
    refused from the arguments alone (no pointer is read), before the layer's
    device state is looked at."""
    spec = WL.CFG1
    layer = svdq.Layer(spec.w(), svdq.calibrate_amax(spec.x()), 16, rank_capacity=48)
    lib = svdq.lib()
    h = layer._h
    assert lib.svdq_lora_swap(h, 64, 128, 8, 1.0, None) == svdq.ERR_UNSUPPORTED_SHAPE  # not a multiple of 16
    assert lib.svdq_lora_swap(h, 64, 128, 48, 1.0, None) == svdq.ERR_UNSUPPORTED_SHAPE  # 16 + 48 > 48
    # a rank whose sum with the base rank overflows int32 is still over capacity
    assert lib.svdq_lora_swap(h, 64, 128, 2147483632, 1.0, None) == svdq.ERR_UNSUPPORTED_SHAPE
    assert lib.svdq_lora_swap(h, None, 128, 16, 1.0, None) == svdq.ERR_INVALID_ARGUMENT
    assert lib.svdq_lora_swap(h, 65, 128, 16, 1.0, None) == svdq.ERR_INVALID_ARGUMENT
    assert "aligned" in svdq.last_error()
    assert lib.svdq_lora_swap(h, 64, 129, 16, 1.0, None) == svdq.ERR_INVALID_ARGUMENT
    assert lib.svdq_lora_swap(h, 64, 128, 16, float("inf"), None) == svdq.ERR_INVALID_ARGUMENT
    assert lib.svdq_lora_swap(h, 64, 128, 16, 1.0, None) == svdq.ERR_INVALID_ARGUMENT  # valid, but not uploaded
    assert "uploaded" in svdq.last_error()


def test_null_arguments_are_errors_not_crashes():
    L = svdq.lib()
    assert L.svdq_prepare_host(None, None) == svdq.ERR_INVALID_ARGUMENT
    assert L.svdq_act_buffer_bytes(None, 4, None) == svdq.ERR_INVALID_ARGUMENT
    assert L.svdq_layer_export(None, 1, None, 0) == svdq.ERR_INVALID_ARGUMENT
    assert L.svdq_act_unpack(None, 1, None, 0, None, None, None) == svdq.ERR_INVALID_ARGUMENT
    assert L.svdq_quantize_act(None, None, 1, None, 0, None) == svdq.ERR_INVALID_ARGUMENT
    assert L.svdq_w4a4_linear(None, None, 0, 1, None, 0, None) == svdq.ERR_INVALID_ARGUMENT
    assert L.svdq_lora_swap(None, None, None, 0, 1.0, None) == svdq.ERR_INVALID_ARGUMENT
    assert L.svdq_poll_status(None, None) == svdq.ERR_INVALID_ARGUMENT
    L.svdq_layer_destroy(None)


def test_host_only_layer_cannot_launch():
    spec = WL.CFG1
    X = spec.x()
    layer = svdq.Layer(spec.w(), np.max(np.abs(X.astype(np.float32)), 0), spec.rank)
    st = svdq.lib().svdq_quantize_act(layer._h, 16, 64, 256, 1 << 20, None)
    assert st == svdq.ERR_INVALID_ARGUMENT
    assert "uploaded" in svdq.last_error()
    buf = np.zeros(16, np.uint8)
    assert svdq.lib().svdq_layer_export(layer._h, 99, buf.ctypes.data, 16) == svdq.ERR_INVALID_ARGUMENT
    assert svdq.lib().svdq_layer_export(layer._h, svdq.EXPORT_LAMBDA, buf.ctypes.data, 16) == \
        svdq.ERR_BUFFER_TOO_SMALL
    with pytest.raises(svdq.SvdqError):
        layer.export(svdq.EXPORT_R)  # not kept


def test_rope_packed_bytes_follow_the_row_tiles():
    n = ctypes.c_size_t()
    L = svdq.lib()
    assert L.svdq_rope_packed_bytes(1, 128, ctypes.byref(n)) == svdq.OK and n.value == 2 * 32 * 128 * 16
    assert svdq.rope_packed_bytes(256) == 2 * 65536 and svdq.rope_packed_bytes(257) == 4 * 65536
    assert L.svdq_rope_packed_bytes(0, 128, ctypes.byref(n)) == svdq.ERR_INVALID_ARGUMENT
    assert L.svdq_rope_packed_bytes(16, 64, ctypes.byref(n)) == svdq.ERR_UNSUPPORTED_SHAPE
    assert L.svdq_rope_pack(None, 16, 128, None, 0, None) == svdq.ERR_INVALID_ARGUMENT


def test_calibrate_amax_is_running_max():
    x1 = WL.make_x(17, 64, seed=1)
    x2 = WL.make_x(9, 64, seed=2)
    amax = svdq.calibrate_amax(x1)
    amax = svdq.calibrate_amax(x2, amax)
    ref = np.maximum(np.abs(x1.astype(np.float32)).max(0), np.abs(x2.astype(np.float32)).max(0))
    np.testing.assert_array_equal(amax, ref)


def test_buffer_sizes_follow_tiling():
    spec = WL.CFG1
    X = spec.x()
    layer = svdq.Layer(spec.w(), np.max(np.abs(X.astype(np.float32)), 0), 16, rank_capacity=48)
    # activation tiles of 128 rows, an even number of them: (256 K -> 16 KB codes
    # + 2 KB scales) + 1 chunk of 64 ranks (16 KB) per tile
    assert layer.act_buffer_bytes(1) == 2 * (16384 + 2048 + 16384)
    assert layer.act_buffer_bytes(256) == 2 * (16384 + 2048 + 16384)
    assert layer.act_buffer_bytes(257) == 4 * (16384 + 2048 + 16384)
    info = layer.info()
    assert (info.K, info.N, info.rank, info.rank_total, info.rank_capacity) == (256, 256, 16, 16, 48)
    assert info.dev_buf is None and info.device == -1
    assert info.device_bytes == layer.device_bytes > 0


def test_clone_copies_the_prepared_layer_and_outlives_it():
    spec = WL.CFG1
    X = spec.x()
    layer = svdq.Layer(spec.w(), svdq.calibrate_amax(X), spec.rank)
    twin = layer.clone()
    want = {e: layer.export(e) for e in (svdq.EXPORT_LAMBDA, svdq.EXPORT_L1, svdq.EXPORT_L2, svdq.EXPORT_W_CODES,
                                         svdq.EXPORT_W_SCALES, svdq.EXPORT_SCALARS)}
    layer.close()
    for e, v in want.items():
        np.testing.assert_array_equal(twin.export(e), v)
    assert twin.info().rank_total == spec.rank
    # not bound to a device buffer: launching must be refused, not crash
    st = svdq.lib().svdq_quantize_act(twin._h, 1, 1, 1, 1, None)
    assert st == svdq.ERR_INVALID_ARGUMENT


def test_binding_refuses_tensors_the_abi_cannot_check():
    """The C ABI sees only pointers, so the binding refuses, before any library
    call, a host tensor, another device, a wrong dtype or shape, a
    non-contiguous view and a short norm weight.  A meta tensor stands in for
    the layer's device buffer: nothing here touches a GPU."""
    import torch

    spec = WL.CFG1
    K, N = spec.K, spec.N
    layer = svdq.Layer(spec.w(), svdq.calibrate_amax(spec.x()), spec.rank)
    with pytest.raises(svdq.SvdqError) as e:
        layer.quantize_act(torch.zeros((4, K), dtype=torch.bfloat16))
    assert e.value.status == svdq.ERR_INVALID_ARGUMENT and "uploaded" in str(e.value)
    layer.dev_buf = torch.empty(0, dtype=torch.uint8, device="meta")

    def meta(shape, dt=torch.bfloat16):
        return torch.empty(shape, dtype=dt, device="meta")

    act = meta((1 << 16,), torch.uint8)
    refused = [
        lambda: layer.quantize_act(torch.zeros((4, K), dtype=torch.bfloat16)),  # host memory
        lambda: layer.quantize_act(meta((4, K), torch.float32)),
        lambda: layer.quantize_act(meta((4, K + 64))),
        lambda: layer.quantize_act(meta((K,))),
        lambda: layer.quantize_act(meta((K, 4)).t()),  # a transposed view
        lambda: layer.quantize_act(meta((4, K)), act=torch.zeros(1 << 16, dtype=torch.uint8)),
        lambda: layer.linear(torch.zeros(1 << 16, dtype=torch.uint8), 4),
        lambda: layer.linear(act, 4, out=meta((4, N + 1))),
        lambda: layer.linear(act, 4, out=meta((4, N), torch.float16)),
        lambda: layer.linear(act, 4, out=meta((N, 4)).t()),
        lambda: layer.forward(meta((4, K), torch.float16)),
        lambda: layer.lora_swap(meta((K, 16)), None),
        lambda: layer.lora_swap(meta((K, 16)), meta((32, N))),
        lambda: layer.lora_swap(meta((K + 64, 16)), meta((16, N))),
        lambda: layer.lora_swap(torch.zeros((K, 16), dtype=torch.bfloat16), meta((16, N))),
        lambda: layer.linear_qkv_norm_rope(act, 4, meta((64,)), meta((128,)), meta((64,), torch.uint8)),
        lambda: layer.linear_qkv_norm_rope(act, 4, meta((128,)), meta((128,), torch.float32), meta((64,), torch.uint8)),
        lambda: layer.linear_qkv_norm_rope(act, 4, meta((128,)), meta((128,)), torch.zeros(64, dtype=torch.uint8)),
    ]
    for i, f in enumerate(refused):
        with pytest.raises((ValueError, TypeError)):
            f()
            pytest.fail(f"case {i} was not refused")

    w = svdq.W4A16Layer(WL.make_w(16, 64, seed=3))
    with pytest.raises(svdq.SvdqError):
        w.linear(torch.zeros((1, 64), dtype=torch.bfloat16))
    w.dev_buf = torch.empty(0, dtype=torch.uint8, device="meta")
    for f in (lambda: w.linear(torch.zeros((1, 64), dtype=torch.bfloat16)),
              lambda: w.linear(meta((1, 128))),
              lambda: w.linear(meta((1, 64), torch.float32)),
              lambda: w.linear(meta((1, 64)), out=meta((1, 17)))):
        with pytest.raises((ValueError, TypeError)):
            f()
    with pytest.raises(ValueError):
        svdq.rope_pack(torch.zeros((4, 64, 2), dtype=torch.float32))  # host memory


C_CALLER = r"""
#include <stdio.h>
#include "svdq.h"

int main(void) {
  svdq_prepare_desc d = {0};
  size_t bytes = 1;
  if (svdq_abi_version() != SVDQ_ABI_VERSION) return 1;
  if (svdq_layer_device_bytes(&d) != 0) return 2;             /* W missing: refused, size 0 */
  if (svdq_rope_packed_bytes(128, 128, &bytes) != SVDQ_OK || bytes == 0) return 3;
  if (svdq_quantize_act(NULL, NULL, 1, NULL, 0, NULL) != SVDQ_ERR_INVALID_ARGUMENT) return 4;
  printf("%s\n", svdq_last_error());
  return 0;
}
"""


@pytest.mark.skipif(subprocess.run(["which", "gcc"], capture_output=True).returncode != 0, reason="needs gcc")
def test_header_is_plain_c_and_links_from_c(tmp_path):
    """include/svdq.h compiles as strict C99 and a C program links against
    libsvdq.so and calls it (host-only entry points; no CUDA call)."""
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    lib_dir = os.path.dirname(svdq.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I" + os.path.join(ROOT, "include"),
                    str(src), "-L" + lib_dir, "-lsvdq", "-Wl,-rpath," + lib_dir, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.strip()  # the refusal left its message in svdq_last_error()
