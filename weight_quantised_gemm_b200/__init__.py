"""Python binding of libqgemm (the C ABI in include/qgemm.h).

Argument marshalling only: every step of the GEMM runs in the library's CUDA
kernels; torch provides device memory and streams. There is no CPU fallback:
the shared library is loaded on first use, and every entry point raises if
it is missing (the package itself imports without it, so that its build
module can run on a fresh checkout).

    import weight_quantised_gemm_b200 as wq
    pw = wq.qgemm_pack(W_fp32_numpy, bits=4)          # host, RTN, packed at rest
    dw = pw.to_device("cuda")                         # device-resident weights
    y = wq.qgemm(x_bf16_cuda, dw, bias=b_bf16_cuda)   # out = x . dequant(W)^T + b
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqgemm.so")

QGEMM_OK = 0
QGEMM_ERR_INVALID_ARG = 1
QGEMM_ERR_UNSUPPORTED = 2
QGEMM_ERR_ALIGNMENT = 3
QGEMM_ERR_NONFINITE = 4
QGEMM_ERR_CUDA = 5
QGEMM_ERR_DEVICE_TIMEOUT = 6

QGEMM_PATH_AUTO = 0
QGEMM_PATH_SMALL_M = 1
QGEMM_PATH_LARGE_M = 2
QGEMM_FLAG_OVERLAP_PREVIOUS = 0x100
QGEMM_FLAG_GROUPED_ONE_LAUNCH = 0x200

QGEMM_EPI_NONE = 0
QGEMM_EPI_GELU_TANH = 1
QGEMM_EPI_RESIDUAL_GATE = 2

GROUP_OF_BITS = {1: 128, 2: 128, 4: 64, 8: 64}


class QGemmError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {qgemm_status_str(status)} ({status}): {detail}")


class _Epilogue(ctypes.Structure):
    _fields_ = [("op", ctypes.c_int32), ("residual", ctypes.c_void_p), ("gate", ctypes.c_void_p)]


class _Weights(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("group", ctypes.c_int32), ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p)]


class _Problem(ctypes.Structure):
    _fields_ = [("X", ctypes.c_void_p), ("M", ctypes.c_int32), ("W", _Weights), ("out", ctypes.c_void_p),
                ("bias", ctypes.c_void_p)]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is not built; run `python -m weight_quantised_gemm_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_size_t
    W = ctypes.POINTER(_Weights)
    sig = {
        "qgemm_pack_sizes": (ctypes.c_int, [i32, i32, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(sz),
                                            ctypes.POINTER(sz)]),
        "qgemm_pack": (ctypes.c_int, [vp, i32, i32, i32, i32, vp, vp, vp]),
        "qgemm_pack_device": (ctypes.c_int, [vp, i32, i32, i32, i32, vp, vp, vp, vp]),
        "qgemm_save": (ctypes.c_int, [ctypes.c_char_p, i32, i32, i32, i32, vp, vp, vp]),
        "qgemm_load_header": (ctypes.c_int, [ctypes.c_char_p, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                             ctypes.POINTER(i32), ctypes.POINTER(i32)]),
        "qgemm_load": (ctypes.c_int, [ctypes.c_char_p, vp, vp, vp]),
        "qgemm": (ctypes.c_int, [vp, i32, W, vp, vp, vp]),
        "qgemm_ex": (ctypes.c_int, [vp, i32, W, vp, vp, i32, vp]),
        "qgemm_fused": (ctypes.c_int, [vp, i32, W, vp, vp, ctypes.POINTER(_Epilogue), i32, vp]),
        "qgemm_select_path": (ctypes.c_int, [i32, i32, i32, i32]),
        "qgemm_dequant_tile": (ctypes.c_int, [W, i32, i32, i32, i32, vp, vp]),
        "qgemm_debug_stream": (ctypes.c_int, [vp, i32, W, i32, vp]),
        "qgemm_grouped": (ctypes.c_int, [ctypes.POINTER(_Problem), i32, i32, vp]),
        "qgemm_get_device_status": (ctypes.c_int, [vp]),
        "qgemm_set_wait_limit_ns": (ctypes.c_int, [u64]),
        "qgemm_debug_wait_timeout": (ctypes.c_int, [u64, vp]),
        "qgemm_status_str": (ctypes.c_char_p, [ctypes.c_int]),
        "qgemm_last_error": (ctypes.c_char_p, []),
        "qgemm_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


class _LazyLib:
    """The loaded libqgemm.so, opened on first attribute access."""
    _handle = None

    def __getattr__(self, name):
        if _LazyLib._handle is None:
            _LazyLib._handle = _load()
        return getattr(_LazyLib._handle, name)


_lib = _LazyLib()
EXPORTED = ("qgemm_pack_sizes", "qgemm_pack", "qgemm_pack_device", "qgemm_save", "qgemm_load_header",
            "qgemm_load", "qgemm", "qgemm_ex", "qgemm_fused",
            "qgemm_select_path",
            "qgemm_dequant_tile", "qgemm_debug_stream", "qgemm_grouped",
            "qgemm_get_device_status", "qgemm_set_wait_limit_ns", "qgemm_debug_wait_timeout",
            "qgemm_status_str", "qgemm_last_error", "qgemm_version")


def library_path() -> str:
    return _LIB_PATH


def qgemm_status_str(status: int) -> str:
    return _lib.qgemm_status_str(int(status)).decode()


def qgemm_last_error() -> str:
    return _lib.qgemm_last_error().decode()


def qgemm_version() -> str:
    return _lib.qgemm_version().decode()


def _check(status: int, where: str) -> None:
    if status != QGEMM_OK:
        raise QGemmError(status, where, qgemm_last_error())


def qgemm_pack_sizes(N: int, K: int, bits: int, group: Optional[int] = None):
    group = GROUP_OF_BITS.get(bits, 0) if group is None else group
    p, s, b = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.qgemm_pack_sizes(N, K, bits, group, ctypes.byref(p), ctypes.byref(s), ctypes.byref(b)),
           "qgemm_pack_sizes")
    return p.value, s.value, b.value


@dataclasses.dataclass
class PackedWeights:
    """Host copy of a packed weight: codes, fp16 scales, fp16 biases (None for ternary)."""
    N: int
    K: int
    bits: int
    group: int
    packed: np.ndarray   # uint8 [N, K*bits/8]
    scales: np.ndarray   # float16 [K/group, N] (group-major)
    biases: Optional[np.ndarray]  # float16 [K/group, N]

    @property
    def nbytes(self) -> int:
        return self.packed.nbytes + self.scales.nbytes + (0 if self.biases is None else self.biases.nbytes)

    def save(self, path: str) -> None:
        """Writes the at-rest file (C ABI qgemm_save)."""
        _check(_lib.qgemm_save(os.fsencode(path), self.N, self.K, self.bits, self.group, self.packed.ctypes.data,
                               self.scales.ctypes.data, None if self.biases is None else self.biases.ctypes.data),
               "qgemm_save")

    def to_device(self, device="cuda") -> "DeviceWeights":
        import torch
        dev = torch.device(device)
        packed = torch.from_numpy(self.packed).to(dev)
        scales = torch.from_numpy(self.scales.view(np.int16)).to(dev)
        biases = None if self.biases is None else torch.from_numpy(self.biases.view(np.int16)).to(dev)
        return DeviceWeights(self.N, self.K, self.bits, self.group, packed, scales, biases)


@dataclasses.dataclass
class DeviceWeights:
    """Device-resident packed weight (torch tensors own the memory)."""
    N: int
    K: int
    bits: int
    group: int
    packed: "object"
    scales: "object"
    biases: "object"

    @property
    def nbytes(self) -> int:
        n = self.packed.numel() + 2 * self.scales.numel()
        return n + (0 if self.biases is None else 2 * self.biases.numel())

    def descriptor(self) -> _Weights:
        return _Weights(self.N, self.K, self.bits, self.group, self.packed.data_ptr(), self.scales.data_ptr(),
                        None if self.biases is None else self.biases.data_ptr())


def qgemm_pack(W, bits: int, group: Optional[int] = None) -> PackedWeights:
    """RTN-quantise host fp32 W [N, K] into the packed at-rest format (C ABI qgemm_pack)."""
    W = np.ascontiguousarray(np.asarray(W, dtype=np.float32))
    if W.ndim != 2:
        raise ValueError("W must be 2-D [N, K]")
    N, K = W.shape
    group = GROUP_OF_BITS.get(bits, 0) if group is None else group
    pb, sb, bb = qgemm_pack_sizes(N, K, bits, group)
    packed = np.empty(pb, dtype=np.uint8)
    scales = np.empty(sb // 2, dtype=np.float16)
    biases = np.empty(bb // 2, dtype=np.float16) if bb else None
    _check(_lib.qgemm_pack(W.ctypes.data, N, K, bits, group, packed.ctypes.data, scales.ctypes.data,
                           None if biases is None else biases.ctypes.data), "qgemm_pack")
    return PackedWeights(N, K, bits, group, packed.reshape(N, -1), scales.reshape(K // group, N),
                         None if biases is None else biases.reshape(K // group, N))


def qgemm_pack_device(W, bits: int, group: Optional[int] = None, stream=None) -> "DeviceWeights":
    """RTN-quantise a device fp32 W [N, K] on the GPU (C ABI qgemm_pack_device):
    the same bytes as qgemm_pack. Errors in the data surface through
    check_device_status."""
    import torch
    if W.dtype != torch.float32 or not W.is_cuda or W.dim() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D fp32 CUDA tensor")
    N, K = W.shape
    group = GROUP_OF_BITS.get(bits, 0) if group is None else group
    pb, sb, bb = qgemm_pack_sizes(N, K, bits, group)
    packed = torch.empty(pb, dtype=torch.uint8, device=W.device)
    scales = torch.empty(sb // 2, dtype=torch.int16, device=W.device)
    biases = torch.empty(bb // 2, dtype=torch.int16, device=W.device) if bb else None
    with torch.cuda.device(W.device):
        _check(_lib.qgemm_pack_device(W.data_ptr(), N, K, bits, group, packed.data_ptr(), scales.data_ptr(),
                                      None if biases is None else biases.data_ptr(),
                                      _stream_handle(stream, W.device)), "qgemm_pack_device")
    return DeviceWeights(N, K, bits, group, packed.view(N, -1), scales, biases)


def qgemm_load(path: str) -> PackedWeights:
    """Reads an at-rest file written by qgemm_save (C ABI qgemm_load_header + qgemm_load)."""
    N, K, bits, group = (ctypes.c_int32() for _ in range(4))
    p = os.fsencode(path)
    _check(_lib.qgemm_load_header(p, ctypes.byref(N), ctypes.byref(K), ctypes.byref(bits), ctypes.byref(group)),
           "qgemm_load_header")
    N, K, bits, group = N.value, K.value, bits.value, group.value
    pb, sb, bb = qgemm_pack_sizes(N, K, bits, group)
    packed = np.empty(pb, dtype=np.uint8)
    scales = np.empty(sb // 2, dtype=np.float16)
    biases = np.empty(bb // 2, dtype=np.float16) if bb else None
    _check(_lib.qgemm_load(p, packed.ctypes.data, scales.ctypes.data, None if biases is None else biases.ctypes.data),
           "qgemm_load")
    return PackedWeights(N, K, bits, group, packed.reshape(N, -1), scales.reshape(K // group, N),
                         None if biases is None else biases.reshape(K // group, N))


def _stream_handle(stream, device=None) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return stream.cuda_stream


def _same_device(device, W: "DeviceWeights", **tensors) -> None:
    """Every tensor argument on X's CUDA device: the library launches on the
    current device and takes raw pointers, so a host or other-device buffer
    must be refused here, before any launch."""
    arrays = {"W.packed": W.packed, "W.scales": W.scales, "W.biases": W.biases, **tensors}
    for name, t in arrays.items():
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, X on {device}")


def qgemm(X, W: DeviceWeights, bias=None, out=None, path: int = QGEMM_PATH_AUTO, stream=None,
          overlap_previous: bool = False):
    """out[M, N] = X[M, K] . dequant(W)^T (+ bias), bf16 in and out, on `stream`
    (default: torch's current stream). Enqueues only; see qgemm_get_device_status.
    overlap_previous sets QGEMM_FLAG_OVERLAP_PREVIOUS (weights must be static)."""
    import torch
    if X.dtype != torch.bfloat16 or not X.is_cuda or X.dim() != 2 or not X.is_contiguous():
        raise ValueError("X must be a contiguous 2-D bf16 CUDA tensor")
    M, K = X.shape
    if K != W.K:
        raise ValueError(f"X has K={K}, weights have K={W.K}")
    if out is None:
        out = torch.empty((M, W.N), dtype=torch.bfloat16, device=X.device)
    elif out.dtype != torch.bfloat16 or tuple(out.shape) != (M, W.N) or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 [M, N] tensor")
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != W.N or not bias.is_cuda):
        raise ValueError("bias must be a bf16 CUDA tensor of N elements")
    _same_device(X.device, W, out=out, bias=bias)
    desc = W.descriptor()
    flags = QGEMM_FLAG_OVERLAP_PREVIOUS if overlap_previous else 0
    with torch.cuda.device(X.device):
        _check(_lib.qgemm_ex(X.data_ptr(), M, ctypes.byref(desc), out.data_ptr(),
                             None if bias is None else bias.data_ptr(), int(path) | flags,
                             _stream_handle(stream, X.device)), "qgemm")
    return out


def qgemm_fused(X, W: DeviceWeights, op: int, bias=None, residual=None, gate=None, out=None,
                path: int = QGEMM_PATH_AUTO, stream=None, overlap_previous: bool = False):
    """qgemm with a fused epilogue (QGEMM_EPI_*): GELU, or out = residual + gate * y.
    `out` may be `residual` itself (in-place update of the residual stream)."""
    import torch
    if X.dtype != torch.bfloat16 or not X.is_cuda or X.dim() != 2 or not X.is_contiguous():
        raise ValueError("X must be a contiguous 2-D bf16 CUDA tensor")
    M, K = X.shape
    if K != W.K:
        raise ValueError(f"X has K={K}, weights have K={W.K}")
    if out is None:
        out = torch.empty((M, W.N), dtype=torch.bfloat16, device=X.device)
    elif out.dtype != torch.bfloat16 or tuple(out.shape) != (M, W.N) or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 [M, N] tensor")
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != W.N or not bias.is_cuda):
        raise ValueError("bias must be a bf16 CUDA tensor of N elements")
    if op == QGEMM_EPI_RESIDUAL_GATE:
        if residual is None or gate is None:
            raise ValueError("the residual update needs residual and gate")
        if residual.dtype != torch.bfloat16 or tuple(residual.shape) != (M, W.N) or not residual.is_contiguous():
            raise ValueError("residual must be a contiguous bf16 [M, N] tensor")
        if gate.dtype != torch.bfloat16 or gate.numel() != W.N or not gate.is_cuda:
            raise ValueError("gate must be a bf16 CUDA tensor of N elements")
    _same_device(X.device, W, out=out, bias=bias, residual=residual, gate=gate)
    epi = _Epilogue(int(op), None if residual is None else residual.data_ptr(),
                    None if gate is None else gate.data_ptr())
    desc = W.descriptor()
    flags = QGEMM_FLAG_OVERLAP_PREVIOUS if overlap_previous else 0
    with torch.cuda.device(X.device):
        _check(_lib.qgemm_fused(X.data_ptr(), M, ctypes.byref(desc), out.data_ptr(),
                                None if bias is None else bias.data_ptr(), ctypes.byref(epi), int(path) | flags,
                                _stream_handle(stream, X.device)), "qgemm_fused")
    return out


def qgemm_grouped(problems, outs=None, stream=None, overlap_previous: bool = False, one_launch: bool = False):
    """Several independent small-M GEMVs (C ABI qgemm_grouped): `problems` is
    a list of (X, W, bias) with X a bf16 [M, K] CUDA tensor (M <= 16), W
    DeviceWeights (one format for all) and bias a bf16 [N] tensor or None.
    Consecutive overlapped launches, or one persistent launch with
    `one_launch` (QGEMM_FLAG_GROUPED_ONE_LAUNCH). Returns the outputs (bf16
    [M, N] each), written into `outs` when given."""
    import torch
    if not problems:
        raise ValueError("no problems")
    dev = problems[0][0].device
    arr = (_Problem * len(problems))()
    result = []
    for i, (X, W, bias) in enumerate(problems):
        if X.dtype != torch.bfloat16 or not X.is_cuda or X.dim() != 2 or not X.is_contiguous():
            raise ValueError(f"problem {i}: X must be a contiguous 2-D bf16 CUDA tensor")
        M, K = X.shape
        if K != W.K:
            raise ValueError(f"problem {i}: X has K={K}, weights have K={W.K}")
        out = None if outs is None else outs[i]
        if out is None:
            out = torch.empty((M, W.N), dtype=torch.bfloat16, device=dev)
        elif out.dtype != torch.bfloat16 or tuple(out.shape) != (M, W.N) or not out.is_contiguous():
            raise ValueError(f"problem {i}: out must be a contiguous bf16 [M, N] tensor")
        if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != W.N or not bias.is_cuda):
            raise ValueError(f"problem {i}: bias must be a bf16 CUDA tensor of N elements")
        _same_device(dev, W, X=X, out=out, bias=bias)
        arr[i] = _Problem(X.data_ptr(), M, W.descriptor(), out.data_ptr(), None if bias is None else bias.data_ptr())
        result.append(out)
    flags = (QGEMM_FLAG_OVERLAP_PREVIOUS if overlap_previous else 0) | (QGEMM_FLAG_GROUPED_ONE_LAUNCH if one_launch else 0)
    with torch.cuda.device(dev):
        _check(_lib.qgemm_grouped(arr, len(problems), flags, _stream_handle(stream, dev)), "qgemm_grouped")
    return result


def qgemm_select_path(M: int, N: int, K: int, bits: int) -> int:
    r = _lib.qgemm_select_path(M, N, K, bits)
    if r < 0:
        raise QGemmError(-r, "qgemm_select_path", "")
    return r


def qgemm_dequant_tile(W: DeviceWeights, n0: int = 0, k0: int = 0, rows: Optional[int] = None,
                       cols: Optional[int] = None, out=None, stream=None):
    """Dequantised weights W[n0:n0+rows, k0:k0+cols] as a bf16 tensor (debug entry point)."""
    import torch
    rows = W.N - n0 if rows is None else rows
    cols = W.K - k0 if cols is None else cols
    dev = W.packed.device
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
    elif out.dtype != torch.bfloat16 or tuple(out.shape) != (rows, cols) or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 [rows, cols] tensor")
    _same_device(dev, W, out=out)
    desc = W.descriptor()
    with torch.cuda.device(dev):
        _check(_lib.qgemm_dequant_tile(ctypes.byref(desc), n0, k0, rows, cols, out.data_ptr(),
                                       _stream_handle(stream, dev)), "qgemm_dequant_tile")
    return out


def qgemm_debug_stream(X, W: DeviceWeights, stream=None, overlap_previous: bool = False) -> None:
    """The small-M kernel as qgemm would launch it for (X, W), streaming the
    packed weights through its ring and computing nothing (C ABI
    qgemm_debug_stream): the streaming floor of the shape."""
    import torch
    if X.dtype != torch.bfloat16 or not X.is_cuda or X.dim() != 2 or not X.is_contiguous():
        raise ValueError("X must be a contiguous 2-D bf16 CUDA tensor")
    if X.shape[1] != W.K:
        raise ValueError(f"X has K={X.shape[1]}, weights have K={W.K}")
    _same_device(X.device, W)
    desc = W.descriptor()
    with torch.cuda.device(X.device):
        _check(_lib.qgemm_debug_stream(X.data_ptr(), X.shape[0], ctypes.byref(desc),
                                       QGEMM_FLAG_OVERLAP_PREVIOUS if overlap_previous else 0,
                                       _stream_handle(stream, X.device)), "qgemm_debug_stream")


def qgemm_get_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status; raises nothing."""
    return _lib.qgemm_get_device_status(_stream_handle(stream))


def check_device_status(stream=None) -> None:
    _check(qgemm_get_device_status(stream), "device status")


def qgemm_set_wait_limit_ns(limit_ns: int) -> None:
    _check(_lib.qgemm_set_wait_limit_ns(int(limit_ns)), "qgemm_set_wait_limit_ns")


def qgemm_debug_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(_lib.qgemm_debug_wait_timeout(int(limit_ns), _stream_handle(stream)), "qgemm_debug_wait_timeout")
