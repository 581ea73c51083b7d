"""The prepared layer as a flat, versioned blob (svdq_layer_serialize / svdq_layer_import), on the CPU.

A layer imported from a blob must be the layer that wrote it: every export equal byte for byte,
and its own blob identical.  Truncated, corrupted, foreign and future-version blobs are refused
with a status, not read."""

import struct

import numpy as np
import pytest

from bit_w4a4_quantized_b200 import svdq
from bit_w4a4_quantized_b200 import workloads as WL

EXPORTS = (svdq.EXPORT_LAMBDA, svdq.EXPORT_INV_LAMBDA, svdq.EXPORT_L1, svdq.EXPORT_L2, svdq.EXPORT_W_CODES,
           svdq.EXPORT_W_SCALES, svdq.EXPORT_SCALARS, svdq.EXPORT_RESID_NORM)


def _layer(rank=16, bias=True, rank_capacity=None):
    spec = WL.CFG1
    return svdq.Layer(spec.w(), svdq.calibrate_amax(spec.x()), rank, rank_capacity=rank_capacity,
                      bias=WL.make_bias(spec.N, 0) if bias else None)


@pytest.mark.parametrize("rank,bias,cap", [(16, True, None), (0, False, None), (32, False, 64)])
def test_round_trip_is_the_same_layer(rank, bias, cap):
    a = _layer(rank, bias, cap)
    blob = a.serialize()
    b = svdq.Layer.from_blob(blob)
    for what in EXPORTS:
        np.testing.assert_array_equal(a.export(what), b.export(what), err_msg=str(what))
    if rank:
        np.testing.assert_array_equal(a.export(svdq.EXPORT_SIGMA), b.export(svdq.EXPORT_SIGMA))
    ia, ib = a.info(), b.info()
    for f in ("K", "N", "rank", "rank_total", "rank_capacity", "format", "g_a", "g_w", "alpha", "device_bytes"):
        assert getattr(ia, f) == getattr(ib, f), f
    assert b.serialize() == blob


def test_header_fields():
    a = _layer(16)
    blob = a.serialize()
    assert blob[:8] == b"SVDQLAYR"
    version, header_bytes = struct.unpack_from("<II", blob, 8)
    assert (version, header_bytes) == (1, 128)
    K, N = struct.unpack_from("<qq", blob, 16)
    assert (K, N) == (a.K, a.N)


def _import_status(blob):
    import ctypes

    h = ctypes.c_void_p()
    st = svdq.lib().svdq_layer_import(blob, len(blob), ctypes.byref(h))
    if st == svdq.OK:
        svdq.lib().svdq_layer_destroy(h)
    return st


def test_damaged_blobs_are_refused():
    blob = bytearray(_layer(16).serialize())
    assert _import_status(bytes(blob)) == svdq.OK
    assert _import_status(bytes(blob[:-8])) == svdq.ERR_INVALID_ARGUMENT  # truncated
    assert "truncated" in svdq.last_error()
    assert _import_status(bytes(blob[:100])) == svdq.ERR_INVALID_ARGUMENT  # shorter than the header
    for pos in (128, len(blob) // 2, len(blob) - 1):  # one flipped bit anywhere after the header
        bad = bytearray(blob)
        bad[pos] ^= 0x10
        assert _import_status(bytes(bad)) == svdq.ERR_INVALID_ARGUMENT
        assert "checksum" in svdq.last_error()
    bad = bytearray(blob)
    bad[0:8] = b"NOTALAYR"
    assert _import_status(bytes(bad)) == svdq.ERR_INVALID_ARGUMENT
    bad = bytearray(blob)
    struct.pack_into("<I", bad, 8, 2)  # a future version
    assert _import_status(bytes(bad)) == svdq.ERR_INVALID_ARGUMENT
    assert "version" in svdq.last_error()
    bad = bytearray(blob)
    struct.pack_into("<q", bad, 16, 100)  # K not a multiple of 64
    assert _import_status(bytes(bad)) == svdq.ERR_UNSUPPORTED_SHAPE


def test_serialize_arguments():
    import ctypes

    a = _layer(16)
    n = ctypes.c_size_t()
    lib = svdq.lib()
    assert lib.svdq_layer_serialize(a._h, None, 0, ctypes.byref(n)) == svdq.OK and n.value > 128
    small = ctypes.create_string_buffer(n.value - 1)
    assert lib.svdq_layer_serialize(a._h, small, n.value - 1, None) == svdq.ERR_BUFFER_TOO_SMALL
    assert lib.svdq_layer_serialize(None, None, 0, ctypes.byref(n)) == svdq.ERR_INVALID_ARGUMENT
    assert lib.svdq_layer_serialize(a._h, None, 0, None) == svdq.ERR_INVALID_ARGUMENT
    assert lib.svdq_layer_import(None, 0, None) == svdq.ERR_INVALID_ARGUMENT
