"""Thin Python binding of the qlin C ABI (``include/qlin.h``).

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of the computation runs in ``libqlin.so``.  There is no
fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqlin.so")

QLIN_OK = 0
STATUS_NAMES = {0: "QLIN_OK", -1: "QLIN_ERR_INVALID_ARG", -2: "QLIN_ERR_UNSUPPORTED", -3: "QLIN_ERR_SHAPE",
                -4: "QLIN_ERR_ALIGNMENT", -5: "QLIN_ERR_CUDA", -6: "QLIN_ERR_WORKSPACE"}

EXPORTED = (
    "qlin_status_string", "qlin_last_cuda_error", "qlin_packed_bytes", "qlin_code_bytes", "qlin_pack",
    "qlin_unpack", "qlin_dequant", "qlin_rht", "qlin_gemv_workspace_bytes", "qlin_gemv",
    "qlin_gemm_workspace_bytes", "qlin_gemm", "qlin_device_error", "qlin_gemm_noalloc", "qlin_set_overlap",
    "qlin_quantize_rtn", "qlin_gemv_plan", "qlin_gptq_workspace_bytes", "qlin_quantize_gptq", "qlin_linear_host",
)


class QlinError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {status_string(status)}")


class _Desc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("block_bits", ctypes.c_void_p)]


class Desc:
    """qlin_desc plus the host copy of the block widths it points to."""

    def __init__(self, N: int, K: int, bits: int, block_bits: Optional[Sequence[int]] = None):
        self.N, self.K, self.bits = int(N), int(K), int(bits)
        self._bb = None
        ptr = None
        if self.bits == 0:
            if block_bits is None:
                raise ValueError("mixed widths (bits=0) need block_bits")
            bb = bytes(int(b) for b in (block_bits.tolist() if hasattr(block_bits, "tolist") else block_bits))
            self._bb = ctypes.create_string_buffer(bb, len(bb))
            ptr = ctypes.addressof(self._bb)
        self.block_bits = None if self._bb is None else list(self._bb.raw)
        self.c = _Desc(self.N, self.K, self.bits, ptr)
        self._byref = ctypes.byref(self.c)
        self._ws = {}  # (entry point, M) -> workspace bytes: a pure function of the descriptor and M

    @classmethod
    def of(cls, w) -> "Desc":
        """Descriptor of a ``workloads.QuantWeight``."""
        return cls(w.N, w.K, w.bits, w.block_bits)

    def ref(self):
        return self._byref


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqlin.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m dequant_gemv_packed_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i32, cp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_char_p
    L.qlin_status_string.argtypes, L.qlin_status_string.restype = [ctypes.c_int], cp
    L.qlin_last_cuda_error.argtypes, L.qlin_last_cuda_error.restype = [], ctypes.c_int
    L.qlin_set_overlap.argtypes, L.qlin_set_overlap.restype = [ctypes.c_int], ctypes.c_int
    L.qlin_packed_bytes.argtypes, L.qlin_packed_bytes.restype = [vp], sz
    L.qlin_code_bytes.argtypes, L.qlin_code_bytes.restype = [vp], sz
    L.qlin_pack.argtypes, L.qlin_pack.restype = [vp, vp, vp, vp], ctypes.c_int
    L.qlin_unpack.argtypes, L.qlin_unpack.restype = [vp, vp, vp, vp], ctypes.c_int
    L.qlin_dequant.argtypes, L.qlin_dequant.restype = [vp, vp, vp, vp, vp, vp], ctypes.c_int
    L.qlin_rht.argtypes, L.qlin_rht.restype = [vp, vp, vp, i32, i32, vp], ctypes.c_int
    L.qlin_quantize_rtn.argtypes, L.qlin_quantize_rtn.restype = [vp, vp, vp, vp, vp, vp, vp], ctypes.c_int
    L.qlin_gptq_workspace_bytes.argtypes, L.qlin_gptq_workspace_bytes.restype = [vp], sz
    L.qlin_quantize_gptq.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.qlin_quantize_gptq.restype = ctypes.c_int
    L.qlin_gemv_plan.argtypes, L.qlin_gemv_plan.restype = [vp, i32, vp], ctypes.c_int
    L.qlin_gemv_workspace_bytes.argtypes, L.qlin_gemv_workspace_bytes.restype = [vp, i32], sz
    L.qlin_gemm_workspace_bytes.argtypes, L.qlin_gemm_workspace_bytes.restype = [vp, i32], sz
    L.qlin_device_error.argtypes, L.qlin_device_error.restype = [ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int
    lin = [vp, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp]
    L.qlin_gemv.argtypes, L.qlin_gemv.restype = lin, ctypes.c_int
    L.qlin_gemm.argtypes, L.qlin_gemm.restype = lin, ctypes.c_int
    L.qlin_gemm_noalloc.argtypes, L.qlin_gemm_noalloc.restype = [vp, vp, vp, vp, vp, vp, vp, i32, vp], ctypes.c_int
    L.qlin_linear_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp]
    L.qlin_linear_host.restype = ctypes.c_int
    _lib = L
    return L


def status_string(status: int) -> str:
    try:
        return lib().qlin_status_string(status).decode()
    except RuntimeError:
        return STATUS_NAMES.get(status, str(status))


def _check(status: int, what: str) -> None:
    if status != QLIN_OK:
        raise QlinError(status, what)


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, like: torch.Tensor = None) -> int:
    if stream is None:
        if _raw_stream is not None and like is not None and like.is_cuda:
            return _raw_stream(like.device.index)  # the current stream's handle, without a Stream object
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _alloc(shape, dtype, like: torch.Tensor) -> torch.Tensor:
    return torch.empty(shape, dtype=dtype, device=like.device)


# ----------------------------------------------------------------- entry points

def qlin_set_overlap(enable: bool) -> bool:
    """Allow qlin_gemv to overlap the preceding kernel on its stream (see qlin.h);
    returns the previous setting."""
    return bool(lib().qlin_set_overlap(1 if enable else 0))


def qlin_packed_bytes(desc: Desc) -> int:
    return int(lib().qlin_packed_bytes(desc.ref()))


def qlin_code_bytes(desc: Desc) -> int:
    return int(lib().qlin_code_bytes(desc.ref()))


def qlin_gemv_workspace_bytes(desc: Desc, M: int) -> int:
    return int(lib().qlin_gemv_workspace_bytes(desc.ref(), M))


def qlin_gemm_workspace_bytes(desc: Desc, M: int) -> int:
    return int(lib().qlin_gemm_workspace_bytes(desc.ref(), M))


def qlin_device_error() -> int:
    """Read and clear the device-side error word (0: no bounded wait expired)."""
    v = ctypes.c_uint32(0)
    _check(lib().qlin_device_error(ctypes.byref(v)), "qlin_device_error")
    return int(v.value)


def qlin_pack(desc: Desc, codes: torch.Tensor, packed: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    nbytes = qlin_packed_bytes(desc)
    if nbytes == 0:
        raise QlinError(-1, "qlin_pack (descriptor)")
    if packed is None:
        packed = _alloc((nbytes,), torch.uint8, codes)
    if packed.numel() * packed.element_size() < nbytes:
        raise ValueError("packed buffer too small")
    _check(lib().qlin_pack(desc.ref(), _dev(codes, torch.uint8, "codes"), packed.data_ptr(), _stream(stream)),
           "qlin_pack")
    return packed


def qlin_unpack(desc: Desc, packed: torch.Tensor, codes: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if codes is None:
        codes = _alloc((desc.N, desc.K), torch.uint8, packed)
    _check(lib().qlin_unpack(desc.ref(), _dev(packed, torch.uint8, "packed"), _dev(codes, torch.uint8, "codes"),
                             _stream(stream)), "qlin_unpack")
    return codes


def qlin_dequant(desc: Desc, packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                 w: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if w is None:
        w = _alloc((desc.N, desc.K), torch.float16, packed)
    _check(lib().qlin_dequant(desc.ref(), _dev(packed, torch.uint8, "packed"), _dev(scales, torch.float16, "scales"),
                              _dev(zeros, torch.float16, "zeros"), _dev(w, torch.float16, "w"), _stream(stream)),
           "qlin_dequant")
    return w


class _GemvPlan(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "kernel", "grid", "threads", "smem_bytes", "consumer_warps", "units_per_warp", "rows_per_cta",
        "rows_per_chunk", "stages", "chunks_in_flight")] + [("workspace_bytes", ctypes.c_uint64)]


def qlin_gemv_plan(desc: Desc, M: int) -> dict:
    """The launch plan qlin_gemv uses for this weight and M (host only)."""
    info = _GemvPlan()
    _check(lib().qlin_gemv_plan(desc.ref(), M, ctypes.byref(info)), "qlin_gemv_plan")
    return {name: getattr(info, name) for name, _ in _GemvPlan._fields_}


def qlin_quantize_rtn(desc: Desc, w: torch.Tensor, sign_bits: torch.Tensor, codes: Optional[torch.Tensor] = None,
                      scales: Optional[torch.Tensor] = None, zeros: Optional[torch.Tensor] = None, stream=None):
    """Rotated round-to-nearest quantisation of fp16 weight rows: (codes, scales, zeros)."""
    G = desc.K // 128
    if codes is None:
        codes = _alloc((desc.N, desc.K), torch.uint8, w)
    if scales is None:
        scales = _alloc((desc.N, G), torch.float16, w)
    if zeros is None:
        zeros = _alloc((desc.N, G), torch.float16, w)
    _check(lib().qlin_quantize_rtn(desc.ref(), _dev(w, torch.float16, "w"), _dev(sign_bits, torch.int32, "sign_bits"),
                                   _dev(codes, torch.uint8, "codes"), _dev(scales, torch.float16, "scales"),
                                   _dev(zeros, torch.float16, "zeros"), _stream(stream)), "qlin_quantize_rtn")
    return codes, scales, zeros


def qlin_gptq_workspace_bytes(desc: Desc) -> int:
    return int(lib().qlin_gptq_workspace_bytes(desc.ref()))


def qlin_quantize_gptq(desc: Desc, w: torch.Tensor, sign_bits: torch.Tensor, hinv_factor: torch.Tensor,
                       codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                       zeros: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None):
    """Rotation and error-compensated (GPTQ) quantisation of fp16 weight rows
    against the fp32 upper factor of the damped inverse Hessian: (codes, scales, zeros)."""
    G = desc.K // 128
    if codes is None:
        codes = _alloc((desc.N, desc.K), torch.uint8, w)
    if scales is None:
        scales = _alloc((desc.N, G), torch.float16, w)
    if zeros is None:
        zeros = _alloc((desc.N, G), torch.float16, w)
    need = qlin_gptq_workspace_bytes(desc)
    if workspace is None:
        workspace = _alloc((max(need, 16),), torch.uint8, w)
    _check(lib().qlin_quantize_gptq(desc.ref(), _dev(w, torch.float16, "w"), _dev(sign_bits, torch.int32, "sign_bits"),
                                    _dev(hinv_factor, torch.float32, "hinv_factor"), _dev(codes, torch.uint8, "codes"),
                                    _dev(scales, torch.float16, "scales"), _dev(zeros, torch.float16, "zeros"),
                                    _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
           "qlin_quantize_gptq")
    return codes, scales, zeros


def qlin_rht(x: torch.Tensor, sign_bits: torch.Tensor, xr: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M, K = x.shape
    if xr is None:
        xr = torch.empty_like(x)
    _check(lib().qlin_rht(_dev(x, torch.float16, "x"), _dev(xr, torch.float16, "xr"),
                          _dev(sign_bits, torch.int32, "sign_bits"), M, K, _stream(stream)), "qlin_rht")
    return xr


def _linear(fn, what, ws_fn, desc, packed, scales, zeros, sign_bits, x, y, workspace, stream):
    M, K = x.shape
    if K != desc.K:
        raise ValueError("x.shape[1] != desc.K")
    if y is None:
        y = _alloc((M, desc.N), torch.float16, x)
    ws = desc._ws.get((what, M))
    if ws is None:
        ws = desc._ws[(what, M)] = ws_fn(desc, M)
    if workspace is None and ws:
        workspace = _alloc((ws,), torch.uint8, x)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(fn(desc.ref(), _dev(packed, torch.uint8, "packed"), _dev(scales, torch.float16, "scales"),
              _dev(zeros, torch.float16, "zeros"), _dev(sign_bits, torch.int32, "sign_bits"),
              _dev(x, torch.float16, "x"), _dev(y, torch.float16, "y"), M, ws_ptr, ws_len, _stream(stream, x)), what)
    return y


def qlin_gemv(desc: Desc, packed, scales, zeros, sign_bits, x, y=None, workspace=None, stream=None) -> torch.Tensor:
    return _linear(lib().qlin_gemv, "qlin_gemv", qlin_gemv_workspace_bytes, desc, packed, scales, zeros, sign_bits,
                   x, y, workspace, stream)


def qlin_gemm(desc: Desc, packed, scales, zeros, sign_bits, x, y=None, workspace=None, stream=None) -> torch.Tensor:
    return _linear(lib().qlin_gemm, "qlin_gemm", qlin_gemm_workspace_bytes, desc, packed, scales, zeros, sign_bits,
                   x, y, workspace, stream)


def qlin_linear(desc: Desc, packed, scales, zeros, sign_bits, x, y=None, workspace=None, stream=None) -> torch.Tensor:
    """qlin_gemv for M <= 16, qlin_gemm otherwise."""
    f = qlin_gemv if x.shape[0] <= 16 else qlin_gemm
    return f(desc, packed, scales, zeros, sign_bits, x, y, workspace, stream)


def _host(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError(f"{name} must be a host tensor")
    if t.dtype != torch.float16:
        raise TypeError(f"{name} must be torch.float16, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def qlin_linear_host(desc: Desc, packed, scales, zeros, sign_bits, x_host, y_host, x_dev, y_dev,
                     workspace=None, stream=None) -> torch.Tensor:
    """The layer on host activations in one call (x_host [M, K] and y_host [M, N]
    fp16 host tensors, pinned for asynchronous copies; x_dev / y_dev device
    staging tensors of the same shapes); returns y_host, valid once the stream
    has passed the call."""
    M, K = x_host.shape
    if K != desc.K or tuple(y_host.shape) != (M, desc.N) or tuple(x_dev.shape) != (M, K) \
            or tuple(y_dev.shape) != (M, desc.N):
        raise ValueError("shapes: x_host/x_dev [M, K], y_host/y_dev [M, N]")
    what = "qlin_gemv" if M <= 16 else "qlin_gemm"
    ws = desc._ws.get((what, M))
    if ws is None:
        ws = desc._ws[(what, M)] = (qlin_gemv_workspace_bytes if M <= 16 else qlin_gemm_workspace_bytes)(desc, M)
    if workspace is None and ws:
        workspace = _alloc((ws,), torch.uint8, x_dev)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().qlin_linear_host(desc.ref(), _dev(packed, torch.uint8, "packed"), _dev(scales, torch.float16, "scales"),
                                  _dev(zeros, torch.float16, "zeros"), _dev(sign_bits, torch.int32, "sign_bits"),
                                  _host(x_host, "x_host"), _host(y_host, "y_host"), _dev(x_dev, torch.float16, "x_dev"),
                                  _dev(y_dev, torch.float16, "y_dev"), M, ws_ptr, ws_len, _stream(stream, x_dev)),
           "qlin_linear_host")
    return y_host


def algorithmic_bytes(desc: Desc) -> int:
    """Bytes one pass over the weight must read: packed codes, the fp16 scale and
    zero of every group, and (mixed widths) one selector byte per 64-row block."""
    sel = desc.N // 64 if desc.bits == 0 else 0
    return qlin_code_bytes(desc) + 4 * desc.N * (desc.K // 128) + sel


def kernel_launches_per_call(kind: str, desc: Desc, M: int) -> int:
    """Kernels one call enqueues: the layer kernel, plus the stand-alone rotation
    kernel whenever the call needs a workspace for the rotated activations."""
    if kind == "gemm":
        return 2
    return 2 if qlin_gemv_workspace_bytes(desc, M) else 1
