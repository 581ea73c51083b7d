"""ctypes binding of libsvdq.so (the C ABI in include/svdq.h).

Argument marshalling only: every step of the layer runs in the library (host
preparation in C++, the forward pass in the CUDA kernels).  PyTorch supplies
device memory and streams.  There is no fallback: if the library is missing
or a call fails, an exception is raised.
"""

import ctypes
import os

import numpy as np

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libsvdq.so")

OK = 0
ERR_INVALID_ARGUMENT = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_UNSUPPORTED_DEVICE = 3
ERR_BUFFER_TOO_SMALL = 4
ERR_CUDA = 5
ERR_TIMEOUT = 6
ERR_INTERNAL = 7
ERR_HOST_ALLOC = 8

FMT_NVFP4 = 1
FMT_INT4 = 2
PREPARE_KEEP_R = 1
EPI_NONE = 0
EPI_GELU_TANH = 1

EXPORT_LAMBDA = 1
EXPORT_INV_LAMBDA = 2
EXPORT_L1 = 3
EXPORT_L2 = 4
EXPORT_R = 5
EXPORT_W_CODES = 6
EXPORT_W_SCALES = 7
EXPORT_SIGMA = 8
EXPORT_SCALARS = 9
EXPORT_RESID_NORM = 10

# every symbol include/svdq.h declares
EXPORTED_SYMBOLS = (
    "svdq_abi_version", "svdq_last_error", "svdq_calibrate_amax", "svdq_layer_device_bytes",
    "svdq_prepare_host", "svdq_layer_upload", "svdq_prepare_weights", "svdq_act_buffer_bytes",
    "svdq_quantize_act", "svdq_w4a4_linear", "svdq_lora_swap", "svdq_layer_export", "svdq_act_unpack",
    "svdq_get_layer_info", "svdq_poll_status", "svdq_layer_destroy", "svdq_test_override_device_arch",
    "svdq_test_bounded_wait", "svdq_layer_clone", "svdq_w4a4_linear_qkv_norm_rope",
    "svdq_rope_packed_bytes", "svdq_rope_pack", "svdq_w4a16_device_bytes", "svdq_w4a16_prepare_host",
    "svdq_w4a16_upload", "svdq_w4a16_linear", "svdq_w4a16_export", "svdq_w4a16_poll_status",
    "svdq_w4a16_destroy",
    "svdq_layer_serialize", "svdq_layer_import", "svdq_mlp_workspace_bytes", "svdq_w4a4_linear_mlp",
    "svdq_w4a4_linear_mlp_static",
)


class SvdqError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"svdq status {status}: {message}")
        self.status = status


class PrepareDesc(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int64), ("N", ctypes.c_int64),
        ("rank", ctypes.c_int32), ("rank_capacity", ctypes.c_int32),
        ("format", ctypes.c_int32), ("num_threads", ctypes.c_int32), ("flags", ctypes.c_int32),
        ("W", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("act_amax", ctypes.c_void_p),
        ("L1", ctypes.c_void_p), ("L2", ctypes.c_void_p),
        ("svd_seed", ctypes.c_uint64), ("svd_power_iters", ctypes.c_int32), ("svd_oversample", ctypes.c_int32),
    ]


class W4A16Desc(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int64), ("N", ctypes.c_int64), ("W", ctypes.c_void_p), ("s", ctypes.c_void_p),
        ("bias", ctypes.c_void_p),
    ]


class LayerInfo(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int64), ("N", ctypes.c_int64),
        ("rank", ctypes.c_int32), ("rank_total", ctypes.c_int32), ("rank_capacity", ctypes.c_int32),
        ("format", ctypes.c_int32),
        ("g_a", ctypes.c_float), ("g_w", ctypes.c_float), ("alpha", ctypes.c_float),
        ("device_bytes", ctypes.c_size_t), ("dev_buf", ctypes.c_void_p), ("device", ctypes.c_int32),
    ]


_lib = None


def lib():
    """Load libsvdq.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m bit_w4a4_quantized_b200.build` "
                           "(or __graft_entry__.build()); there is no fallback implementation")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    st = ctypes.c_int
    sig = {
        "svdq_abi_version": ([], ctypes.c_int),
        "svdq_last_error": ([], ctypes.c_char_p),
        "svdq_calibrate_amax": ([vp, i64, i64, vp], st),
        "svdq_layer_device_bytes": ([ctypes.POINTER(PrepareDesc)], sz),
        "svdq_prepare_host": ([ctypes.POINTER(PrepareDesc), ctypes.POINTER(vp)], st),
        "svdq_layer_upload": ([vp, vp, sz, vp], st),
        "svdq_prepare_weights": ([ctypes.POINTER(PrepareDesc), vp, sz, ctypes.POINTER(vp), vp], st),
        "svdq_act_buffer_bytes": ([vp, i64, ctypes.POINTER(sz)], st),
        "svdq_quantize_act": ([vp, vp, i64, vp, sz, vp], st),
        "svdq_w4a4_linear": ([vp, vp, sz, i64, vp, ctypes.c_int, vp], st),
        "svdq_w4a4_linear_qkv_norm_rope": ([vp, vp, sz, i64, vp, vp, vp, vp, sz, i32, ctypes.c_float, vp], st),
        "svdq_rope_packed_bytes": ([i64, i32, ctypes.POINTER(sz)], st),
        "svdq_rope_pack": ([vp, i64, i32, vp, sz, vp], st),
        "svdq_lora_swap": ([vp, vp, vp, i32, ctypes.c_float, vp], st),
        "svdq_layer_export": ([vp, ctypes.c_int, vp, sz], st),
        "svdq_act_unpack": ([vp, i64, vp, sz, vp, vp, vp], st),
        "svdq_get_layer_info": ([vp, ctypes.POINTER(LayerInfo)], st),
        "svdq_poll_status": ([vp, vp], st),
        "svdq_layer_destroy": ([vp], None),
        "svdq_layer_clone": ([vp, ctypes.POINTER(vp)], st),
        "svdq_layer_serialize": ([vp, vp, sz, ctypes.POINTER(sz)], st),
        "svdq_mlp_workspace_bytes": ([vp, vp, i64, ctypes.POINTER(sz)], st),
        "svdq_w4a4_linear_mlp": ([vp, vp, sz, i64, vp, vp, sz, vp, sz, ctypes.c_int, vp], st),
        "svdq_w4a4_linear_mlp_static": ([vp, vp, sz, i64, vp, vp, sz, ctypes.c_int, vp], st),
        "svdq_layer_import": ([vp, sz, ctypes.POINTER(vp)], st),
        "svdq_w4a16_device_bytes": ([ctypes.POINTER(W4A16Desc)], sz),
        "svdq_w4a16_prepare_host": ([ctypes.POINTER(W4A16Desc), ctypes.POINTER(vp)], st),
        "svdq_w4a16_upload": ([vp, vp, sz, vp], st),
        "svdq_w4a16_linear": ([vp, vp, i64, vp, vp], st),
        "svdq_w4a16_export": ([vp, ctypes.c_int, vp, sz], st),
        "svdq_w4a16_poll_status": ([vp, vp], st),
        "svdq_w4a16_destroy": ([vp], None),
        "svdq_test_override_device_arch": ([ctypes.c_int], None),
        "svdq_test_bounded_wait": ([ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint32), vp], st),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def last_error():
    return lib().svdq_last_error().decode()


def check(status):
    if status != OK:
        raise SvdqError(status, last_error())


def rope_packed_bytes(M, head_dim=128):
    n = ctypes.c_size_t()
    check(lib().svdq_rope_packed_bytes(int(M), int(head_dim), ctypes.byref(n)))
    return n.value


def rope_pack(rope, head_dim=128, out=None, stream=None):
    """Device float32 [M, head_dim / 2, 2] (cos, sin) -> the packed table the
    fused QKV epilogue reads (a uint8 device tensor)."""
    import torch

    M = rope.shape[0]
    if not rope.is_cuda:
        raise ValueError("rope must be a device tensor")
    _need(rope, "rope", rope.device, torch.float32, min_numel=M * int(head_dim))
    if out is None:
        out = torch.empty(rope_packed_bytes(M, head_dim), dtype=torch.uint8, device=rope.device)
    _need(out, "out", rope.device)
    check(lib().svdq_rope_pack(rope.data_ptr(), M, int(head_dim), out.data_ptr(), _nbytes(out), _stream(stream)))
    return out


def _nbytes(t):
    return t.numel() * t.element_size()


def _need(t, name, device, dtype=None, shape=None, min_numel=None):
    """Refuse, before any library call, a tensor that the C ABI cannot check
    itself (it sees only a pointer): one on another device or on the host, a
    non-contiguous view, or one of the wrong dtype or shape.  None passes
    through, so that the library reports a missing argument."""
    import torch

    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the layer on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, fewer than {min_numel}")


def _ptr(a):
    """Data pointer of a numpy array or torch tensor (None -> NULL)."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return a.data_ptr()  # torch.Tensor


def _bf16_bits(a):
    """Host bf16 data as a contiguous uint16 numpy array."""
    if a is None:
        return None
    if not isinstance(a, np.ndarray):  # torch tensor
        import torch

        a = a.detach().to("cpu").contiguous()
        if a.dtype == torch.bfloat16:
            return a.view(torch.int16).numpy().view(np.uint16).copy()
        a = a.numpy()
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a)
    if a.dtype.name == "bfloat16":
        return np.ascontiguousarray(a).view(np.uint16)
    raise TypeError(f"expected bfloat16 data, got {a.dtype}")


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def calibrate_amax(X, amax=None):
    """Running max_i |X_ij| over a host bf16 [M, K] batch (the library's calibration)."""
    x = _bf16_bits(X)
    M, K = x.shape
    if amax is None:
        amax = np.zeros(K, np.float32)
    check(lib().svdq_calibrate_amax(_ptr(x), M, K, _ptr(amax)))
    return amax


class Layer:
    """One prepared SVDQuant W4A4 + low-rank layer (host handle + device image)."""

    def __init__(self, W, act_amax, rank, *, rank_capacity=None, bias=None, factors=None, seed=0, threads=0,
                 keep_r=False, power_iters=0, oversample=0, device=None, stream=None, fmt=FMT_NVFP4):
        """fmt: FMT_NVFP4 (E2M1 codes, E4M3 scales per 16) or FMT_INT4 (codes -7..7, bf16 scales per 64)."""
        self._h = None
        w = _bf16_bits(W)
        self.N, self.K = w.shape
        amax = np.ascontiguousarray(np.asarray(act_amax, dtype=np.float32))
        b = _bf16_bits(bias)
        l1 = l2 = None
        if factors is not None:
            l1, l2 = _bf16_bits(factors[0]), _bf16_bits(factors[1])
        self._keep = (w, amax, b, l1, l2)  # alive during the call
        d = PrepareDesc()
        d.K, d.N, d.rank = self.K, self.N, rank
        d.rank_capacity = rank if rank_capacity is None else rank_capacity
        d.format = fmt
        d.num_threads = threads
        d.flags = PREPARE_KEEP_R if keep_r else 0
        d.W, d.bias, d.act_amax = _ptr(w), _ptr(b), _ptr(amax)
        d.L1, d.L2 = _ptr(l1), _ptr(l2)
        d.svd_seed, d.svd_power_iters, d.svd_oversample = seed, power_iters, oversample
        self.desc = d
        self.device_bytes = lib().svdq_layer_device_bytes(ctypes.byref(d))
        if self.device_bytes == 0:
            raise SvdqError(ERR_INVALID_ARGUMENT, last_error())
        h = ctypes.c_void_p()
        check(lib().svdq_prepare_host(ctypes.byref(d), ctypes.byref(h)))
        self._h = h
        self._keep = None
        self.rank = rank
        self.fmt = fmt
        self.dev_buf = None
        if device is not None:
            self.upload(device, stream)

    def clone(self, device=None, stream=None):
        """A second handle with the same prepared weights (base rank, no adapter), optionally uploaded."""
        h = ctypes.c_void_p()
        check(lib().svdq_layer_clone(self._h, ctypes.byref(h)))
        c = Layer.__new__(Layer)
        c._h, c._keep, c.desc = h, None, self.desc
        c.N, c.K, c.rank, c.device_bytes, c.dev_buf = self.N, self.K, self.rank, self.device_bytes, None
        c.fmt = self.fmt
        if device is not None:
            c.upload(device, stream)
        return c

    def serialize(self):
        """The prepared layer as one flat, versioned blob (bytes), for a checkpoint."""
        n = ctypes.c_size_t()
        check(lib().svdq_layer_serialize(self._h, None, 0, ctypes.byref(n)))
        buf = ctypes.create_string_buffer(n.value)
        check(lib().svdq_layer_serialize(self._h, buf, n.value, ctypes.byref(n)))
        return buf.raw[:n.value]

    @classmethod
    def from_blob(cls, blob, device=None, stream=None):
        """A layer from a blob that ``serialize`` wrote: no SVD and no quantization run."""
        h = ctypes.c_void_p()
        b = bytes(blob)
        check(lib().svdq_layer_import(b, len(b), ctypes.byref(h)))
        c = cls.__new__(cls)
        c._h, c._keep, c.desc, c.dev_buf = h, None, None, None
        i = LayerInfo()
        check(lib().svdq_get_layer_info(h, ctypes.byref(i)))
        c.N, c.K, c.rank, c.device_bytes = i.N, i.K, i.rank, i.device_bytes
        c.fmt = i.format
        if device is not None:
            c.upload(device, stream)
        return c

    # ------------------------------------------------------------- device side
    def upload(self, device="cuda", stream=None):
        import torch

        self.dev_buf = torch.empty(self.device_bytes, dtype=torch.uint8, device=device)
        with torch.cuda.device(self.dev_buf.device):
            check(lib().svdq_layer_upload(self._h, self.dev_buf.data_ptr(), self.device_bytes, _stream(stream)))
        return self

    def _device(self):
        if self.dev_buf is None:
            raise SvdqError(ERR_INVALID_ARGUMENT, "layer has not been uploaded")
        return self.dev_buf.device

    def act_buffer_bytes(self, M):
        n = ctypes.c_size_t()
        check(lib().svdq_act_buffer_bytes(self._h, M, ctypes.byref(n)))
        return n.value

    def new_act_buffer(self, M):
        import torch

        return torch.empty(self.act_buffer_bytes(M), dtype=torch.uint8, device=self._device())

    def quantize_act(self, X, act=None, stream=None):
        """Kernel 1 on a device bf16 [M, K] tensor; returns the activation buffer."""
        import torch

        dev = self._device()
        if X is None or X.dim() != 2:
            raise ValueError("X must be a 2-D tensor [M, K]")
        M = X.shape[0]
        _need(X, "X", dev, torch.bfloat16, (M, self.K))
        if act is None:
            act = self.new_act_buffer(M)
        _need(act, "act", dev)
        check(lib().svdq_quantize_act(self._h, X.data_ptr(), M, act.data_ptr(), _nbytes(act), _stream(stream)))
        return act

    def linear(self, act, M, out=None, epilogue=EPI_NONE, stream=None):
        """Kernel 2; returns Y bf16 [M, N]."""
        import torch

        dev = self._device()
        _need(act, "act", dev)
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.bfloat16, device=dev)
        _need(out, "out", dev, torch.bfloat16, (M, self.N))
        check(lib().svdq_w4a4_linear(self._h, _ptr(act), 0 if act is None else _nbytes(act), M, out.data_ptr(),
                                     epilogue, _stream(stream)))
        return out

    def linear_qkv_norm_rope(self, act, M, norm_q, norm_k, rope_packed, eps=1e-6, head_dim=128, out=None,
                             stream=None):
        """Kernel 2 on a fused Q | K | V layer with per-head RMSNorm of Q and K
        and their rotary turn (norm_q, norm_k: device bf16 [head_dim];
        rope_packed: from ``rope_pack``); returns bf16 [M, N]."""
        import torch

        dev = self._device()
        _need(act, "act", dev)
        _need(norm_q, "norm_q", dev, torch.bfloat16, min_numel=int(head_dim))
        _need(norm_k, "norm_k", dev, torch.bfloat16, min_numel=int(head_dim))
        _need(rope_packed, "rope_packed", dev)
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.bfloat16, device=dev)
        _need(out, "out", dev, torch.bfloat16, (M, self.N))
        check(lib().svdq_w4a4_linear_qkv_norm_rope(self._h, _ptr(act), 0 if act is None else _nbytes(act), M,
                                                   out.data_ptr(),
                                                   _ptr(norm_q), _ptr(norm_k), _ptr(rope_packed),
                                                   0 if rope_packed is None else _nbytes(rope_packed),
                                                   int(head_dim), float(eps), _stream(stream)))
        return out

    def mlp_workspace_bytes(self, fc2, M):
        n = ctypes.c_size_t()
        check(lib().svdq_mlp_workspace_bytes(self._h, fc2._h, M, ctypes.byref(n)))
        return n.value

    def linear_mlp(self, act, M, fc2, act2=None, workspace=None, epilogue=EPI_GELU_TANH, stream=None):
        """This layer as fc1 of a fused MLP pair: fc2's activation buffer from this layer's
        output tile, without writing the output; returns act2 (pass it to fc2.linear)."""
        import torch

        dev = self._device()
        _need(act, "act", dev)
        if act2 is None:
            act2 = fc2.new_act_buffer(M)
        _need(act2, "act2", dev)
        wb = self.mlp_workspace_bytes(fc2, M)
        if workspace is None and wb:
            workspace = torch.empty(wb, dtype=torch.uint8, device=dev)
        if workspace is not None:
            _need(workspace, "workspace", dev)
        check(lib().svdq_w4a4_linear_mlp(self._h, _ptr(act), _nbytes(act), M, fc2._h, _ptr(act2), _nbytes(act2),
                                         _ptr(workspace), 0 if workspace is None else _nbytes(workspace),
                                         epilogue, _stream(stream)))
        return act2

    def forward(self, X, out=None, epilogue=EPI_NONE, act=None, stream=None):
        act = self.quantize_act(X, act, stream)
        return self.linear(act, X.shape[0], out, epilogue, stream)

    def lora_swap(self, A=None, B=None, scale=1.0, stream=None):
        """Attach a LoRA (device bf16 A [K, r_e], B [r_e, N]); A=None detaches."""
        import torch

        dev = self._device()
        if A is None:
            B = None
            r_e = 0
        else:
            if A.dim() != 2 or B is None:
                raise ValueError("A must be [K, r_e] and B [r_e, N]")
            r_e = A.shape[1]
            _need(A, "A", dev, torch.bfloat16, (self.K, r_e))
            _need(B, "B", dev, torch.bfloat16, (r_e, self.N))
        check(lib().svdq_lora_swap(self._h, _ptr(A), _ptr(B), r_e, float(scale), _stream(stream)))

    def poll_status(self, stream=None):
        check(lib().svdq_poll_status(self._h, _stream(stream)))

    # --------------------------------------------------------------- host side
    def info(self):
        i = LayerInfo()
        check(lib().svdq_get_layer_info(self._h, ctypes.byref(i)))
        return i

    def export(self, what):
        K, N, r = self.K, self.N, self.rank
        shapes = {
            EXPORT_LAMBDA: ((K,), np.float32), EXPORT_INV_LAMBDA: ((K,), np.float32),
            EXPORT_L1: ((K, r), np.uint16), EXPORT_L2: ((r, N), np.uint16),
            EXPORT_R: ((K, N), np.float32), EXPORT_W_CODES: ((N, K // 2), np.uint8),
            EXPORT_W_SCALES: ((N, K // 16), np.uint8), EXPORT_SIGMA: ((r,), np.float64),
            EXPORT_SCALARS: ((4,), np.float32), EXPORT_RESID_NORM: ((2,), np.float64),
        }
        if self.fmt == FMT_INT4:  # bf16 bits of one scale per 64 inputs
            shapes[EXPORT_W_SCALES] = ((N, K // 64), np.uint16)
        shape, dt = shapes[what]
        out = np.empty(shape, dtype=dt)
        check(lib().svdq_layer_export(self._h, what, out.ctypes.data, out.nbytes))
        return out

    def act_unpack(self, act_host, M):
        """Logical codes [M, K/2], scales [M, K/16] (INT4: bf16 bits [M, K/64]), lr bf16 bits [M, r_tot]
        of a host copy."""
        a = np.ascontiguousarray(np.asarray(act_host, dtype=np.uint8))
        rt = self.info().rank_total
        codes = np.empty((M, self.K // 2), np.uint8)
        scales = np.empty((M, self.K // 64), np.uint16) if self.fmt == FMT_INT4 else np.empty((M, self.K // 16),
                                                                                               np.uint8)
        lr = np.empty((M, rt), np.uint16)
        check(lib().svdq_act_unpack(self._h, M, a.ctypes.data, a.nbytes, codes.ctypes.data, scales.ctypes.data,
                                    lr.ctypes.data if rt else None))
        return codes, scales, lr

    def close(self):
        if self._h is not None and _lib is not None:
            _lib.svdq_layer_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class W4A16Layer:
    """A W4A16 layer: 4-bit NVFP4 weights of W diag(s); bf16 activations divided by s and
    rounded once to f16 in the kernel; float32 sums, bf16 output."""

    def __init__(self, W, s=None, bias=None, *, device=None, stream=None):
        self._h = None
        w = _bf16_bits(W)
        self.N, self.K = w.shape
        sv = None if s is None else np.ascontiguousarray(np.asarray(s, dtype=np.float32))
        b = _bf16_bits(bias)
        d = W4A16Desc()
        d.K, d.N, d.W, d.s, d.bias = self.K, self.N, _ptr(w), _ptr(sv), _ptr(b)
        self.device_bytes = lib().svdq_w4a16_device_bytes(ctypes.byref(d))
        if self.device_bytes == 0:
            raise SvdqError(ERR_UNSUPPORTED_SHAPE, last_error())
        h = ctypes.c_void_p()
        check(lib().svdq_w4a16_prepare_host(ctypes.byref(d), ctypes.byref(h)))
        self._h = h
        self.dev_buf = None
        if device is not None:
            self.upload(device, stream)

    def upload(self, device="cuda", stream=None):
        import torch

        self.dev_buf = torch.empty(self.device_bytes, dtype=torch.uint8, device=device)
        with torch.cuda.device(self.dev_buf.device):
            check(lib().svdq_w4a16_upload(self._h, self.dev_buf.data_ptr(), self.device_bytes, _stream(stream)))

    def linear(self, X, out=None, stream=None):
        """Y bf16 [M, N] from a device bf16 [M, K] tensor."""
        import torch

        if self.dev_buf is None:
            raise SvdqError(ERR_INVALID_ARGUMENT, "layer has not been uploaded")
        dev = self.dev_buf.device
        if X is None or X.dim() != 2:
            raise ValueError("X must be a 2-D tensor [M, K]")
        M = X.shape[0]
        _need(X, "X", dev, torch.bfloat16, (M, self.K))
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.bfloat16, device=dev)
        _need(out, "out", dev, torch.bfloat16, (M, self.N))
        check(lib().svdq_w4a16_linear(self._h, X.data_ptr(), M, out.data_ptr(), _stream(stream)))
        return out

    def export(self, what):
        K, N = self.K, self.N
        shapes = {EXPORT_W_CODES: ((N, K // 2), np.uint8), EXPORT_W_SCALES: ((N, K // 16), np.uint8),
                  EXPORT_INV_LAMBDA: ((K,), np.float32), EXPORT_SCALARS: ((1,), np.float32)}
        shape, dt = shapes.get(what, ((1,), np.uint8))  # anything else: the library reports the error
        out = np.empty(shape, dtype=dt)
        check(lib().svdq_w4a16_export(self._h, what, out.ctypes.data, out.nbytes))
        return out

    def poll_status(self, stream=None):
        """Raise SvdqError if the kernel gave up a bounded wait since the last poll."""
        check(lib().svdq_w4a16_poll_status(self._h, _stream(stream)))

    def close(self):
        if self._h is not None and _lib is not None:
            _lib.svdq_w4a16_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def test_bounded_wait(timeout_ns, stream=None):
    """Run the library's bounded-wait test kernel; returns its status word."""
    out = ctypes.c_uint32(0)
    check(lib().svdq_test_bounded_wait(timeout_ns, ctypes.byref(out), _stream(stream)))
    return out.value


def override_device_arch(sm):
    lib().svdq_test_override_device_arch(int(sm))


class HostPipeline:
    """Forward passes of one layer over batches that live in host memory.

    Each batch's X is copied in, run through both kernels and its Y copied out.  Two slots
    (device X, activation buffer and Y each) and three streams let the host-to-device copy of
    batch i + 1 and the device-to-host copy of batch i - 1 run in both directions of the link
    while batch i computes.  Host tensors should be pinned, or the copies do not overlap.
    Stream and copy plumbing only: the layer's kernels do the work."""

    def __init__(self, layer, M, epilogue=EPI_NONE):
        import torch

        dev = layer._device()
        self.layer, self.M, self.epilogue = layer, M, epilogue
        self.X = [torch.empty((M, layer.K), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.act = [layer.new_act_buffer(M) for _ in range(2)]
        self.Y = [torch.empty((M, layer.N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.s_in, self.s_run, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.h2d_bytes = 2 * M * layer.K
        self.d2h_bytes = 2 * M * layer.N

    def run(self, xs_host, ys_host):
        """Y_i = layer(X_i) for host bf16 X_i [M, K] into host bf16 Y_i [M, N]; returns once
        every copy is queued (the last one is done when `done_event()` is)."""
        import torch

        n = len(xs_host)
        if len(ys_host) != n:
            raise ValueError("xs_host and ys_host differ in length")
        ran = [None] * n
        out = [None] * n
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(self.s_in):
                if i >= 2:
                    self.s_in.wait_event(ran[i - 2])  # slot j's X and act are free
                self.X[j].copy_(xs_host[i], non_blocking=True)
                copied = torch.cuda.Event()
                copied.record(self.s_in)
            with torch.cuda.stream(self.s_run):
                self.s_run.wait_event(copied)
                if i >= 2:
                    self.s_run.wait_event(out[i - 2])  # slot j's Y has been read out
                self.layer.forward(self.X[j], out=self.Y[j], epilogue=self.epilogue, act=self.act[j],
                                   stream=self.s_run)
                ran[i] = torch.cuda.Event()
                ran[i].record(self.s_run)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(ran[i])
                ys_host[i].copy_(self.Y[j], non_blocking=True)
                out[i] = torch.cuda.Event()
                out[i].record(self.s_out)
        self._last = out[n - 1] if n else None

    def done_event(self):
        return self._last
