"""A vectorised CPU binary convolution: the stated CPU baseline the benchmark times beside the
oracle (bit-packed XOR / AND + population count on AVX-512 or AVX2 registers, fp32 dot products
for binaryWeights).  It is not part of the CUDA library and no forward of the library uses it.

``bconv_simd.cpp`` holds the arithmetic; this module compiles it with g++ on first use and
marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

BINARY_WEIGHTS, XNOR, AND = 0, 1, 2
ISA_NAMES = {0: "scalar POPCNT", 1: "AVX2 (nibble-lookup popcount)", 2: "AVX-512 VPOPCNTQ"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bconv_simd.cpp")
_LIB = os.path.join(_HERE, "libbconv_simd.so")
_lock = threading.Lock()
_lib = None


class _Desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("batch", "in_h", "in_w", "in_channels", "out_channels", "kernel_h",
                                              "kernel_w", "stride_y", "stride_x", "type", "use_beta", "relu", "fc")]


def build(force: bool = False) -> str:
    """Compile bconv_simd.cpp into libbconv_simd.so (g++ -O3, OpenMP; the vector paths carry
    their own target attributes and are chosen at run time)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O3", "-std=c++17", "-fopenmp", "-shared", "-fPIC", "-Wall", "-Werror",
                               "-mpopcnt", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            lib.simd_bconv.restype = ctypes.c_int
            lib.simd_bconv.argtypes = [ctypes.POINTER(_Desc)] + [P] * 7 + [ctypes.c_int64, P, P, ctypes.c_int]
            lib.simd_best_isa.restype = ctypes.c_int
            lib.simd_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def best_isa() -> int:
    """The vector path this CPU supports (see ISA_NAMES)."""
    return int(_load().simd_best_isa())


def num_threads() -> int:
    return int(_load().simd_num_threads())


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _run(x, wpacked, *, type, kernel, stride, fc, scale, scale_value, bias, in_scale, in_bias, use_beta, relu,
         rows, isa):
    x = _f32(x)
    n, h, w, ni = x.shape
    no = wpacked.shape[0]
    wpacked = np.ascontiguousarray(wpacked, dtype=np.uint32)
    scale = _f32(scale) if scale is not None else np.full(no, scale_value, np.float32)
    bias = _f32(bias) if bias is not None else np.zeros(no, np.float32)
    kh, kw = kernel
    sy, sx = stride
    ho, wo = (1, 1) if fc else (-(-h // sy), -(-w // sx))
    pix = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    npix = n * ho * wo if pix is None else pix.shape[0]
    S = np.empty((npix, no), np.int32)
    y = np.empty((npix, no), np.float32)
    d = _Desc(n, h, w, ni, no, kh, kw, sy, sx, int(type), int(bool(use_beta)), int(bool(relu)), int(bool(fc)))
    rc = _load().simd_bconv(ctypes.byref(d), _p(x), _p(wpacked), _p(scale), _p(bias), _p(_f32(in_scale)),
                            _p(_f32(in_bias)), _p(pix), npix, _p(S), _p(y), -1 if isa is None else int(isa))
    if rc != 0:
        raise ValueError("simd_bconv rejected its arguments")
    if type == BINARY_WEIGHTS:
        S = S.view(np.float32)
    return S, y


def conv(x, wpacked, *, type: int, stride=(1, 1), scale=None, scale_value: float = 1.0, bias=None, in_scale=None,
         in_bias=None, use_beta: bool = False, relu: bool = False, pixels=None, isa: int | None = None):
    """x float32 [N, H, W, Ni]; wpacked uint32 [No, kh, kw, ceil(Ni/32)] (LSB-first).  Returns
    (S, y): S int32 (float32 for binaryWeights) and y float32, [P, No]."""
    no, kh, kw, _ = wpacked.shape
    return _run(x, wpacked, type=type, kernel=(kh, kw), stride=stride, fc=False, scale=scale,
                scale_value=scale_value, bias=bias, in_scale=in_scale, in_bias=in_bias, use_beta=use_beta,
                relu=relu, rows=pixels, isa=isa)


def fc(x, wpacked, *, type: int, scale=None, scale_value: float = 1.0, bias=None, in_scale=None, in_bias=None,
       use_beta: bool = False, relu: bool = False, rows=None, isa: int | None = None):
    """Fully-connected: wpacked uint32 [No, H, W, ceil(Ni/32)]; one output row per image."""
    _, h, w, _ = x.shape
    return _run(x, wpacked, type=type, kernel=(h, w), stride=(1, 1), fc=True, scale=scale, scale_value=scale_value,
                bias=bias, in_scale=in_scale, in_bias=in_bias, use_beta=use_beta, relu=relu, rows=rows, isa=isa)
