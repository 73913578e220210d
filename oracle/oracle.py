"""ctypes marshalling for the C oracle in ``bconv_oracle.c`` (test infrastructure only).

Functions take numpy arrays in the library's logical layouts (NHWC fp32 input, unpacked
0/1 weight bits ``[No][kh][kw][Ni]``) and return float64 arrays.  No arithmetic of the
method happens here: defaults for missing scale terms are expanded, arrays are made
contiguous, and the C routine is called.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

ORACLE_BINARY_WEIGHTS = 0
ORACLE_XNOR = 1
ORACLE_AND = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bconv_oracle.c")
SOURCE_PATH = _SRC
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


class _ConvDesc(ctypes.Structure):
    _fields_ = [
        (name, ctypes.c_int32)
        for name in (
            "batch", "in_h", "in_w", "in_channels", "out_channels",
            "kernel_h", "kernel_w", "stride_y", "stride_x",
            "type", "use_beta", "relu",
        )
    ]


def build(force: bool = False) -> str:
    """Compile ``bconv_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP, no FP contraction)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
            "-shared", "-fPIC", "-Wall", "-Werror", _SRC, "-o", tmp, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.oracle_bconv.restype = ctypes.c_int
    lib.oracle_bconv.argtypes = [ctypes.POINTER(_ConvDesc)] + [P] * 7 + [ctypes.c_int64] + [P] * 3
    lib.oracle_bfc.restype = ctypes.c_int
    lib.oracle_bfc.argtypes = [ctypes.c_int32] * 8 + [P] * 7 + [ctypes.c_int64] + [P] * 3
    lib.oracle_binarize.restype = ctypes.c_int
    lib.oracle_binarize.argtypes = [P, ctypes.c_int64, ctypes.c_int32] + [P] * 5
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def num_threads() -> int:
    """Threads an OpenMP region of the oracle uses (honours OMP_NUM_THREADS)."""
    return int(_load().oracle_num_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


class Variant:
    """The same entry points bound to another build of the oracle source (used by the
    tests that plant a mistake in a copy of the oracle and check that a pin catches it)."""

    def __init__(self, path: str):
        self._lib = _bind(path)

    def conv(self, *args, **kw):
        return conv(*args, _lib_override=self._lib, **kw)

    def fc(self, *args, **kw):
        return fc(*args, _lib_override=self._lib, **kw)

    def binarize(self, *args, **kw):
        return binarize(*args, _lib_override=self._lib, **kw)


def compile_source(src: str, out_path: str) -> str:
    """Compile C source text with the oracle's flags into a shared library at out_path."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src)
    subprocess.check_call([
        "gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
        "-shared", "-fPIC", c_path, "-o", out_path, "-lm",
    ])
    return out_path


def conv_out_dims(h: int, w: int, stride_y: int, stride_x: int) -> tuple[int, int]:
    """Output extent ceil(H/s) x ceil(W/s) (one output per input centre o*s)."""
    return (h + stride_y - 1) // stride_y, (w + stride_x - 1) // stride_x


def _scale_vector(scale, scale_value, n):
    if scale is not None:
        return _f32(scale)
    return np.full(n, scale_value, dtype=np.float32)


def conv(x, wbits, *, type: int, _lib_override=None, stride=(1, 1), scale=None, scale_value: float = 1.0, bias=None,
         in_scale=None, in_bias=None, use_beta: bool = False, relu: bool = False, pixels=None):
    """Oracle binary convolution.

    x      float32 [N, H, W, Ni];  wbits uint8 {0,1} [No, kh, kw, Ni]
    pixels optional int64 flattened output-pixel indices (n*Ho*Wo + oy*Wo + ox)
    Returns (S, beta, y): S and y float64 [P, No] (P = len(pixels) or N*Ho*Wo),
    beta float64 [P].
    """
    x = _f32(x)
    wbits = np.ascontiguousarray(wbits, dtype=np.uint8)
    n, h, w, ni = x.shape
    no, kh, kw, ni_w = wbits.shape
    if ni_w != ni:
        raise ValueError("weight channel count differs from the input's")
    sy, sx = stride
    ho, wo = conv_out_dims(h, w, sy, sx)
    scale = _scale_vector(scale, scale_value, no)
    bias = np.zeros(no, np.float32) if bias is None else _f32(bias)
    in_scale, in_bias = _f32(in_scale), _f32(in_bias)
    if pixels is None:
        npix = n * ho * wo
        pix = None
    else:
        pix = np.ascontiguousarray(pixels, dtype=np.int64)
        npix = pix.shape[0]
    S = np.empty((npix, no), np.float64)
    beta = np.empty(npix, np.float64)
    y = np.empty((npix, no), np.float64)
    d = _ConvDesc(n, h, w, ni, no, kh, kw, sy, sx, int(type), int(bool(use_beta)), int(bool(relu)))
    rc = (_lib_override or _load()).oracle_bconv(ctypes.byref(d), _ptr(x), _ptr(wbits), _ptr(scale), _ptr(bias),
                              _ptr(in_scale), _ptr(in_bias), _ptr(pix), npix, _ptr(S), _ptr(beta), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_bconv rejected its arguments")
    return S, beta, y


def fc(x, wbits, *, type: int, _lib_override=None, scale=None, scale_value: float = 1.0, bias=None, in_scale=None,
       in_bias=None, use_beta: bool = False, relu: bool = False, rows=None):
    """Oracle binary fully-connected layer (kernel = source size).

    x float32 [N, H, W, Ni];  wbits uint8 {0,1} [No, H, W, Ni];  rows optional image indices.
    Returns (S, beta, y) as for :func:`conv`, with one row per image.
    """
    x = _f32(x)
    wbits = np.ascontiguousarray(wbits, dtype=np.uint8)
    n, h, w, ni = x.shape
    no = wbits.shape[0]
    if wbits.shape[1:] != (h, w, ni):
        raise ValueError("fully-connected weights must match the source size")
    scale = _scale_vector(scale, scale_value, no)
    bias = np.zeros(no, np.float32) if bias is None else _f32(bias)
    in_scale, in_bias = _f32(in_scale), _f32(in_bias)
    if rows is None:
        nrows, r = n, None
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        nrows = r.shape[0]
    S = np.empty((nrows, no), np.float64)
    beta = np.empty(nrows, np.float64)
    y = np.empty((nrows, no), np.float64)
    rc = (_lib_override or _load()).oracle_bfc(n, h, w, ni, no, int(type), int(bool(use_beta)), int(bool(relu)),
                            _ptr(x), _ptr(wbits), _ptr(scale), _ptr(bias), _ptr(in_scale),
                            _ptr(in_bias), _ptr(r), nrows, _ptr(S), _ptr(beta), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_bfc rejected its arguments")
    return S, beta, y


def binarize(x, *, _lib_override=None, in_scale=None, in_bias=None):
    """Oracle binarization of an fp32 image as the next binary layer sees it.

    x float32 [..., C] (any leading shape).  Returns (bits, A, xt): bits uint8 {0,1} with
    x's shape, A float64 with the leading shape, xt float64 (the transformed values).
    """
    x = _f32(x)
    lead, c = x.shape[:-1], x.shape[-1]
    npix = int(np.prod(lead)) if lead else 1
    bits = np.empty(x.shape, np.uint8)
    A = np.empty(lead, np.float64)
    xt = np.empty(x.shape, np.float64)
    rc = (_lib_override or _load()).oracle_binarize(_ptr(x), npix, c, _ptr(_f32(in_scale)), _ptr(_f32(in_bias)),
                                                    _ptr(bits), _ptr(A), _ptr(xt))
    if rc != 0:
        raise ValueError("oracle_binarize rejected its arguments")
    return bits, A, xt
