"""libiq8r: the IQ8R rotated W8A8 linear layer on B200 (sm_100a).

This module is the Python binding of the C ABI in ``include/iq8r.h``:
argument marshalling only. Every step of the layer runs in the library's
CUDA kernels (or, for ``iq8r_pack``, its host C++ packer); nothing here
computes. PyTorch supplies device memory and streams.

The library is built in-tree by ``quantised_fwht128_act_b200.build`` (or the
repository's ``__graft_entry__.build()``). If ``libiq8r.so`` is missing, every
call raises ``ImportError``: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

__all__ = [
    "IQ8R_OK", "IQ8R_ERR_INVALID_ARG", "IQ8R_ERR_UNSUPPORTED", "IQ8R_ERR_CUDA", "IQ8R_ERR_DEVICE_TIMEOUT",
    "IQ8R_FMT_G256_U8_BF16", "IQ8R_FMT_G128_BF16", "IQ8R_PATH_AUTO", "IQ8R_PATH_GEMV", "IQ8R_PATH_TC",
    "IQ8R_PATH_FLAG_WEIGHTS_WRITTEN",
    "IQ8R_RULE_RTN", "IQ8R_RULE_SEARCH", "IQ8R_FMT_CB4_G128",
    "IQ8RError", "IQ8RWeight", "lib", "lib_path",
    "iq8r_version", "iq8r_last_error", "iq8r_packed_sizes", "iq8r_pack", "iq8r_rotate_quant_act",
    "iq8r_linear", "iq8r_linear_bf16", "iq8r_linear_bf16_host", "iq8r_linear_ex", "iq8r_linear_noalloc", "iq8r_linear_partials", "iq8r_rescore",
    "iq8r_get_device_error",
    "iq8r_selftest_wait_timeout",
]

IQ8R_RULE_RTN = 0
IQ8R_RULE_SEARCH = 1
IQ8R_OK = 0
IQ8R_ERR_INVALID_ARG = 1
IQ8R_ERR_UNSUPPORTED = 2
IQ8R_ERR_CUDA = 3
IQ8R_ERR_DEVICE_TIMEOUT = 4

IQ8R_FMT_G256_U8_BF16 = 0
IQ8R_FMT_G128_BF16 = 1
IQ8R_FMT_CB4_G128 = 2

IQ8R_PATH_AUTO = 0
IQ8R_PATH_GEMV = 1
IQ8R_PATH_TC = 2
# OR into a path: the weights were written by the previous kernel on the stream
IQ8R_PATH_FLAG_WEIGHTS_WRITTEN = 0x100

_FMT_NAMES = {"g256": IQ8R_FMT_G256_U8_BF16, "g128": IQ8R_FMT_G128_BF16, "cb4": IQ8R_FMT_CB4_G128}

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libiq8r.so")


class IQ8RError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libiq8r status {status}: {message}")
        self.status = status


class _Weight(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32),
        ("rotated", ctypes.c_int32),
        ("n", ctypes.c_int64),
        ("k", ctypes.c_int64),
        ("codes", ctypes.c_void_p),
        ("sub_scale", ctypes.c_void_p),
        ("scale", ctypes.c_void_p),
    ]


_lib = None


def lib():
    """The loaded libiq8r (loads it on first use; raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(lib_path):
        raise ImportError(
            f"libiq8r is not built ({lib_path} is missing); run "
            "`python -m quantised_fwht128_act_b200.build` first")
    L = ctypes.CDLL(lib_path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    L.iq8r_version.restype = i32
    L.iq8r_version.argtypes = []
    L.iq8r_last_error.restype = ctypes.c_char_p
    L.iq8r_last_error.argtypes = []
    L.iq8r_packed_sizes.restype = i32
    L.iq8r_packed_sizes.argtypes = [i32, i64, i64, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.iq8r_pack.restype = i32
    L.iq8r_pack.argtypes = [i32, i32, vp, i64, i64, vp, vp, vp, i32]
    L.iq8r_pack_ex.restype = i32
    L.iq8r_pack_ex.argtypes = [i32, i32, i32, vp, i64, i64, vp, vp, vp, i32]
    L.iq8r_rotate_quant_act.restype = i32
    L.iq8r_rotate_quant_act.argtypes = [vp, i64, i64, i32, vp, vp, vp]
    L.iq8r_linear.restype = i32
    L.iq8r_linear.argtypes = [vp, vp, i64, ctypes.POINTER(_Weight), vp, vp]
    L.iq8r_linear_bf16.restype = i32
    L.iq8r_linear_bf16.argtypes = [vp, i64, ctypes.POINTER(_Weight), vp, vp, vp, vp]
    L.iq8r_linear_bf16_host.restype = i32
    L.iq8r_linear_bf16_host.argtypes = [vp, i64, ctypes.POINTER(_Weight), vp, vp, vp, vp, vp, vp]
    L.iq8r_rescore.restype = i32
    L.iq8r_rescore.argtypes = [vp, vp, i64, ctypes.POINTER(_Weight), vp, i64, vp, vp]
    L.iq8r_linear_noalloc.restype = i32
    L.iq8r_linear_noalloc.argtypes = [vp, vp, i64, ctypes.POINTER(_Weight), vp, vp]
    L.iq8r_linear_ex.restype = i32
    L.iq8r_linear_ex.argtypes = [vp, vp, i64, ctypes.POINTER(_Weight), vp, i32, vp]
    L.iq8r_linear_partials.restype = i32
    L.iq8r_linear_partials.argtypes = [vp, i64, ctypes.POINTER(_Weight), i64, i64, vp, i32, vp]
    L.iq8r_get_device_error.restype = i32
    L.iq8r_get_device_error.argtypes = [vp]
    L.iq8r_selftest_wait_timeout.restype = i32
    L.iq8r_selftest_wait_timeout.argtypes = [i64, vp]
    _lib = L
    return L


def _check(status: int):
    if status != IQ8R_OK:
        raise IQ8RError(status, lib().iq8r_last_error().decode(errors="replace"))


def _fmt(fmt) -> int:
    if isinstance(fmt, str):
        return _FMT_NAMES[fmt]
    return int(fmt)


def _stream(stream) -> Optional[int]:
    """A cudaStream_t handle: a torch.cuda.Stream, an int, or None for the
    current torch stream."""
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def iq8r_version() -> int:
    return lib().iq8r_version()


def iq8r_last_error() -> str:
    return lib().iq8r_last_error().decode(errors="replace")


def iq8r_packed_sizes(fmt, n: int, k: int):
    c, s, sc = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().iq8r_packed_sizes(_fmt(fmt), n, k, ctypes.byref(c), ctypes.byref(s), ctypes.byref(sc)))
    return c.value, s.value, sc.value


def iq8r_pack(w_bf16, fmt="g256", rotate: bool = True, n_threads: int = 0, rule: str = "rtn"):
    """Pack a host bf16 weight [N, K] (numpy uint16 bit patterns, or a CPU
    torch tensor of bf16 / int16 / uint16). Returns numpy arrays
    (codes int8 [N, K] -- uint8 [N, K/2] packed indices for "cb4" --,
    sub uint8 [N, K/256] or None, scale uint16 bits).
    rule: "rtn" (round to nearest) or "search" (least-error scales, see
    include/iq8r.h)."""
    f = _fmt(fmt)
    if not isinstance(w_bf16, np.ndarray):
        import torch
        w_bf16 = w_bf16.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    if w.ndim != 2:
        raise ValueError("w must be [N, K]")
    n, k = w.shape
    codes = np.empty((n, k // 2), np.uint8) if f == IQ8R_FMT_CB4_G128 else np.empty((n, k), np.int8)
    if f == IQ8R_FMT_G256_U8_BF16:
        sub = np.empty((n, k // 256), np.uint8)
        scale = np.empty((n,), np.uint16)
    else:
        sub = None
        scale = np.empty((n, k // 128), np.uint16)
    rl = {"rtn": IQ8R_RULE_RTN, "search": IQ8R_RULE_SEARCH}[rule]
    _check(lib().iq8r_pack_ex(f, int(bool(rotate)), rl, _ptr(w), n, k, _ptr(codes), _ptr(sub), _ptr(scale),
                              n_threads))
    return codes, sub, scale


@dataclass
class IQ8RWeight:
    """A packed weight resident on the device (torch tensors own the memory)."""

    fmt: int
    rotated: int
    n: int
    k: int
    codes: "object"
    sub_scale: "object"
    scale: "object"

    @classmethod
    def from_packed(cls, codes, sub, scale, fmt="g256", rotated: bool = True, device="cuda"):
        import torch

        def dev(a):
            if a is None:
                return None
            t = torch.from_numpy(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
            return t.to(device).contiguous()

        c = dev(codes)
        f = _fmt(fmt)
        k = c.shape[1] * 2 if f == IQ8R_FMT_CB4_G128 else c.shape[1]  # two indices a byte
        return cls(f, int(bool(rotated)), c.shape[0], k, c, dev(sub), dev(scale))

    def _struct(self) -> _Weight:
        # built once per set of buffers: a step's call then costs one
        # comparison instead of three pointer queries and a new structure
        key = (self.fmt, self.rotated, self.n, self.k, id(self.codes), id(self.sub_scale), id(self.scale))
        cached = self.__dict__.get("_cached")
        if cached is None or cached[0] != key:
            cached = (key, _Weight(self.fmt, self.rotated, self.n, self.k, _ptr(self.codes), _ptr(self.sub_scale),
                                   _ptr(self.scale)))
            self.__dict__["_cached"] = cached
        return cached[1]


def iq8r_rotate_quant_act(x, rotate: bool = True, xq=None, x_scale=None, stream=None):
    """x: CUDA bf16 [M, K] contiguous. Returns (xq int8 [M, K], x_scale fp32 [M])."""
    import torch
    if x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous [M, K] tensor")
    m, k = x.shape
    if xq is None:
        xq = torch.empty((m, k), dtype=torch.int8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty((m,), dtype=torch.float32, device=x.device)
    _check(lib().iq8r_rotate_quant_act(_ptr(x), m, k, int(bool(rotate)), _ptr(xq), _ptr(x_scale), _stream(stream)))
    return xq, x_scale


def iq8r_linear_ex(xq, x_scale, weight: IQ8RWeight, y=None, path: int = IQ8R_PATH_AUTO, stream=None):
    import torch
    m = xq.shape[0]
    if y is None:
        y = torch.empty((m, weight.n), dtype=torch.bfloat16, device=xq.device)
    w = weight._struct()
    _check(lib().iq8r_linear_ex(_ptr(xq), _ptr(x_scale), m, ctypes.byref(w), _ptr(y), path, _stream(stream)))
    return y


def iq8r_rescore(xq, x_scale, weight: IQ8RWeight, cand, out=None, stream=None):
    """out[t][j] = y[t][cand[t][j]] (int32 candidate rows [M, C]; bf16 [M, C])."""
    import torch
    m, c = cand.shape
    if out is None:
        out = torch.empty((m, c), dtype=torch.bfloat16, device=xq.device)
    w = weight._struct()
    _check(lib().iq8r_rescore(_ptr(xq), _ptr(x_scale), m, ctypes.byref(w), _ptr(cand), c, _ptr(out),
                              _stream(stream)))
    return out


def iq8r_linear_noalloc(xq, x_scale, weight: IQ8RWeight, y=None, stream=None):
    """iq8r_linear with its split-K scratch in the library's fixed device
    array (no allocation; see include/iq8r.h)."""
    import torch
    m = xq.shape[0]
    if y is None:
        y = torch.empty((m, weight.n), dtype=torch.bfloat16, device=xq.device)
    w = weight._struct()
    _check(lib().iq8r_linear_noalloc(_ptr(xq), _ptr(x_scale), m, ctypes.byref(w), _ptr(y), _stream(stream)))
    return y


def iq8r_linear(xq, x_scale, weight: IQ8RWeight, y=None, stream=None):
    """y = x W^T (bf16 [M, N]) from int8 activations and a packed weight."""
    import torch
    m = xq.shape[0]
    if y is None:
        y = torch.empty((m, weight.n), dtype=torch.bfloat16, device=xq.device)
    w = weight._struct()
    _check(lib().iq8r_linear(_ptr(xq), _ptr(x_scale), m, ctypes.byref(w), _ptr(y), _stream(stream)))
    return y


def iq8r_linear_bf16(x, weight: IQ8RWeight, y=None, xq_out=None, x_scale_out=None, stream=None):
    """y = x W^T from bf16 activations [M, K] (rotated and quantised inside;
    one launch for M <= 2, and for M <= 8 with M * K <= 16384). xq_out /
    x_scale_out receive
    the activation codes and scales; staging buffers are made here when the
    call is not a one-launch decode step and none are given."""
    import torch
    if x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous [M, K] tensor")
    m = x.shape[0]
    if y is None:
        y = torch.empty((m, weight.n), dtype=torch.bfloat16, device=x.device)
    if m > 8 or (m > 2 and m * weight.k > 16384):
        if xq_out is None:
            xq_out = torch.empty((m, weight.k), dtype=torch.int8, device=x.device)
        if x_scale_out is None:
            x_scale_out = torch.empty((m,), dtype=torch.float32, device=x.device)
    w = weight._struct()
    _check(lib().iq8r_linear_bf16(_ptr(x), m, ctypes.byref(w), _ptr(y), _ptr(xq_out), _ptr(x_scale_out),
                                  _stream(stream)))
    return y


def iq8r_linear_bf16_host(x_host, weight: IQ8RWeight, x_dev, y_dev, y_host, xq_out=None, x_scale_out=None,
                          stream=None):
    """One call a step from host memory: x_host (pinned bf16 [M, K]) is copied
    to x_dev, the layer runs into y_dev, and y is copied to y_host (pinned bf16
    [M, N]), all queued on the stream (synchronise before reading y_host).
    xq_out / x_scale_out as for iq8r_linear_bf16 (required where the call is
    not one launch)."""
    m = x_host.shape[0]
    _check(lib().iq8r_linear_bf16_host(_ptr(x_host), m, ctypes.byref(weight._struct()), _ptr(x_dev), _ptr(y_dev),
                                       _ptr(y_host), _ptr(xq_out), _ptr(x_scale_out), _stream(stream)))
    return y_host


def iq8r_linear_partials(xq, weight: IQ8RWeight, n0: int = 0, n1: Optional[int] = None, p=None,
                         path: int = IQ8R_PATH_AUTO, stream=None):
    """Exact per-block int32 partial sums [M, n1 - n0, K / block]."""
    import torch
    m = xq.shape[0]
    n1 = weight.n if n1 is None else n1
    g = 256 if weight.fmt == IQ8R_FMT_G256_U8_BF16 else 128
    if p is None:
        p = torch.empty((m, n1 - n0, weight.k // g), dtype=torch.int32, device=xq.device)
    w = weight._struct()
    _check(lib().iq8r_linear_partials(_ptr(xq), m, ctypes.byref(w), n0, n1, _ptr(p), path, _stream(stream)))
    return p


def iq8r_get_device_error(stream=None):
    """Synchronise the stream and raise if a kernel reported a timeout."""
    _check(lib().iq8r_get_device_error(_stream(stream)))


def iq8r_selftest_wait_timeout(limit_ns: int = 2_000_000, stream=None):
    """Launch the bounded-wait self-test kernel (see include/iq8r.h)."""
    _check(lib().iq8r_selftest_wait_timeout(int(limit_ns), _stream(stream)))
