"""ctypes declarations of the C ABI in include/bconv.h (argument marshalling only).

Every function here has the name and argument order of its C counterpart.  Arrays passed
as "host" arguments are numpy arrays (made contiguous with the C type); "device"
arguments are integer addresses (e.g. ``tensor.data_ptr()``) and streams are integer
``cudaStream_t`` values (e.g. ``torch.cuda.current_stream().cuda_stream``).  A non-OK
status raises :class:`BconvError`.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_PKG)
_LIB_PATH = os.path.join(_PKG, "libbconv.so")
_HEADER = os.path.join(_ROOT, "include", "bconv.h")

TYPE_BINARY_WEIGHTS, TYPE_XNOR, TYPE_AND = 0, 1, 2
FLAG_NONE, FLAG_USE_BETA_SCALING = 0, 1
NEURON_NONE, NEURON_RELU = 0, 1
ALGO_AUTO, ALGO_POPC, ALGO_SIMT_F32, ALGO_TCGEN05 = 0, 1, 2, 3
CTA_AUTO, CTA_SINGLE, CTA_PAIR = 0, 1, 2
CODES_AUTO, CODES_INT8, CODES_FP4, CODES_BF16X3 = 0, 1, 2, 3
STAGING_AUTO, STAGING_PER_TAP, STAGING_ROWS, STAGING_INPUT = 0, 1, 2, 3

_STATUS = {0: "BCONV_OK", 1: "BCONV_ERR_INVALID_ARG", 2: "BCONV_ERR_UNSUPPORTED", 3: "BCONV_ERR_CUDA",
           4: "BCONV_ERR_OOM", 5: "BCONV_ERR_TIMEOUT", 6: "BCONV_ERR_NO_DEVICE"}


class BconvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {_STATUS.get(self.status, self.status)} ({_status_text(self.status)})")


class bconv_desc_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("batch", "in_h", "in_w", "in_channels", "out_channels", "kernel_h",
                                              "kernel_w", "stride_y", "stride_x", "groups", "neuron")] + [
        ("scale_value", ctypes.c_float)]


class bfc_desc_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("batch", "in_h", "in_w", "in_channels", "out_channels", "stride_y",
                                              "stride_x", "groups", "neuron")] + [("scale_value", ctypes.c_float)]


class bconv_io_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("in_", "in_bits", "in_a", "out", "out_bits", "out_a")]


_lock = threading.Lock()
_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_SIGS = {
    "bconv_create": (_I32, [ctypes.POINTER(bconv_desc_t), _P, _P, _P, _P, _P, _I32, ctypes.c_uint32, ctypes.POINTER(_P)]),
    "bconv_forward": (_I32, [_P, _P, _P, _P]),
    "bconv_forward_host": (_I32, [_P, _P, _P, _P]),
    "bconv_get_output_dims": (_I32, [_P] + [ctypes.POINTER(_I32)] * 4),
    "bconv_input_feature_channels": (_I32, [_P]),
    "bconv_output_feature_channels": (_I32, [_P]),
    "bconv_set_algo": (_I32, [_P, _I32]),
    "bconv_launches_per_forward": (_I32, [_P]),
    "bconv_effective_algo": (_I32, [_P]),
    "bconv_sync_status": (_I32, [_P, _P]),
    "bconv_profile_begin": (_I32, [_P, _I32]),
    "bconv_profile_end": (_I32, [_P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_I32)]),
    "bconv_destroy": (_I32, [_P]),
    "bfc_create": (_I32, [ctypes.POINTER(bfc_desc_t), _P, _P, _P, _P, _P, _I32, ctypes.c_uint32, ctypes.POINTER(_P)]),
    "bfc_forward": (_I32, [_P, _P, _P, _P]),
    "bfc_forward_host": (_I32, [_P, _P, _P, _P]),
    "bfc_input_feature_channels": (_I32, [_P]),
    "bfc_output_feature_channels": (_I32, [_P]),
    "bfc_set_algo": (_I32, [_P, _I32]),
    "bfc_launches_per_forward": (_I32, [_P]),
    "bfc_effective_algo": (_I32, [_P]),
    "bfc_sync_status": (_I32, [_P, _P]),
    "bfc_profile_begin": (_I32, [_P, _I32]),
    "bfc_profile_stride": (_I32, [_P, _I32]),
    "bconv_profile_stride": (_I32, [_P, _I32]),
    "bfc_profile_end": (_I32, [_P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_I32)]),
    "bfc_destroy": (_I32, [_P]),
    "bconv_status_string": (ctypes.c_char_p, [_I32]),
    "bconv_pack_bits": (_I32, [_P, ctypes.c_int64, _I32, _P]),
    "bconv_version": (_I32, []),
    "bconv_measure_peak": (_I32, [_I32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
    "bconv_forward_noalloc": (_I32, [ctypes.POINTER(bconv_desc_t), _I32, ctypes.c_uint32] + [_P] * 8),
    "bconv_set_output_terms": (_I32, [_P, _P, _P]),
    "bconv_check_wait_timeout": (_I32, [ctypes.c_double]),
    "bconv_forward_io": (_I32, [_P, ctypes.POINTER(bconv_io_t), _P]),
    "bfc_set_output_terms": (_I32, [_P, _P, _P]),
    "bfc_forward_io": (_I32, [_P, ctypes.POINTER(bconv_io_t), _P]),
    "bconv_set_cta_mode": (_I32, [_I32]),
    "bconv_cta_mode": (_I32, [_P]),
    "bfc_cta_mode": (_I32, [_P]),
    "bconv_set_tc_codes": (_I32, [_I32]),
    "bconv_tc_codes": (_I32, [_P]),
    "bconv_set_staging": (_I32, [_I32]),
    "bconv_staging": (_I32, [_P]),
    "bfc_tc_codes": (_I32, [_P]),
}
NOALLOC_SCRATCH_BYTES = 16 << 20


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libbconv.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m binarized_convolution_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def exported_symbols() -> list[str]:
    """Names of the functions include/bconv.h declares."""
    with open(_HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:bconv|bfc)_[a-z_]+)\s*\(", text)))


def _status_text(st: int) -> str:
    try:
        return load_library().bconv_status_string(st).decode()
    except Exception:  # noqa: BLE001 -- the message is best effort
        return "?"


def _check(st: int, where: str):
    if st != 0:
        raise BconvError(st, where)


def _host_f32(a, n, what):
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=np.float32)
    if a.size != n:
        raise ValueError(f"{what} must hold {n} values, got {a.size}")
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_P)


def _create(fn, desc, packed_weights, scale, bias, in_scale, in_bias, type, flags, ni, no, nwords):
    lib = load_library()
    w = np.ascontiguousarray(packed_weights, dtype=np.uint32)
    if w.size != nwords:
        raise ValueError(f"packed_weights must hold {nwords} words, got {w.size}")
    args = [_host_f32(scale, no, "scale"), _host_f32(bias, no, "bias"), _host_f32(in_scale, ni, "in_scale"),
            _host_f32(in_bias, ni, "in_bias")]
    h = _P()
    _check(getattr(lib, fn)(ctypes.byref(desc), _ptr(w), *[_ptr(a) for a in args], int(type), int(flags),
                            ctypes.byref(h)), fn)
    return h


def bconv_create(desc: bconv_desc_t, packed_weights, scale=None, bias=None, in_scale=None, in_bias=None,
                 type: int = TYPE_XNOR, flags: int = FLAG_NONE):
    nw = (desc.in_channels + 31) // 32
    nwords = desc.out_channels * desc.kernel_h * desc.kernel_w * nw
    return _create("bconv_create", desc, packed_weights, scale, bias, in_scale, in_bias, type, flags,
                   desc.in_channels, desc.out_channels, nwords)


def bfc_create(desc: bfc_desc_t, packed_weights, scale=None, bias=None, in_scale=None, in_bias=None,
               type: int = TYPE_XNOR, flags: int = FLAG_NONE):
    nw = (desc.in_channels + 31) // 32
    nwords = desc.out_channels * desc.in_h * desc.in_w * nw
    return _create("bfc_create", desc, packed_weights, scale, bias, in_scale, in_bias, type, flags,
                   desc.in_channels, desc.out_channels, nwords)


def bconv_forward(h, in_ptr: int, out_ptr: int, stream: int = 0):
    _check(load_library().bconv_forward(h, in_ptr, out_ptr, stream), "bconv_forward")


def bconv_set_output_terms(h, next_in_scale=None, next_in_bias=None):
    """Host arrays of out_channels floats (None: 1 / 0) for the layer that reads the bits."""
    no = bconv_output_feature_channels(h)
    s, b = _host_f32(next_in_scale, no, "next_in_scale"), _host_f32(next_in_bias, no, "next_in_bias")
    _check(load_library().bconv_set_output_terms(h, _ptr(s), _ptr(b)), "bconv_set_output_terms")


def bconv_forward_io(h, in_ptr: int | None = None, in_bits_ptr: int | None = None, in_a_ptr: int | None = None,
                     out_ptr: int | None = None, out_bits_ptr: int | None = None, out_a_ptr: int | None = None,
                     stream: int = 0):
    """Forward with fp32 or bit-packed input and output (device addresses; see bconv_io_t)."""
    io = bconv_io_t(in_ptr, in_bits_ptr, in_a_ptr, out_ptr, out_bits_ptr, out_a_ptr)
    _check(load_library().bconv_forward_io(h, ctypes.byref(io), stream), "bconv_forward_io")


def bfc_set_output_terms(h, next_in_scale=None, next_in_bias=None):
    no = bfc_output_feature_channels(h)
    s, b = _host_f32(next_in_scale, no, "next_in_scale"), _host_f32(next_in_bias, no, "next_in_bias")
    _check(load_library().bfc_set_output_terms(h, _ptr(s), _ptr(b)), "bfc_set_output_terms")


def bfc_forward_io(h, in_ptr: int | None = None, in_bits_ptr: int | None = None, in_a_ptr: int | None = None,
                   out_ptr: int | None = None, out_bits_ptr: int | None = None, out_a_ptr: int | None = None,
                   stream: int = 0):
    io = bconv_io_t(in_ptr, in_bits_ptr, in_a_ptr, out_ptr, out_bits_ptr, out_a_ptr)
    _check(load_library().bfc_forward_io(h, ctypes.byref(io), stream), "bfc_forward_io")


def bfc_forward(h, in_ptr: int, out_ptr: int, stream: int = 0):
    _check(load_library().bfc_forward(h, in_ptr, out_ptr, stream), "bfc_forward")


def bconv_forward_host(h, host_in_ptr: int, host_out_ptr: int, stream: int = 0):
    _check(load_library().bconv_forward_host(h, host_in_ptr, host_out_ptr, stream), "bconv_forward_host")


def bfc_forward_host(h, host_in_ptr: int, host_out_ptr: int, stream: int = 0):
    _check(load_library().bfc_forward_host(h, host_in_ptr, host_out_ptr, stream), "bfc_forward_host")


def bconv_get_output_dims(h):
    v = [_I32() for _ in range(4)]
    _check(load_library().bconv_get_output_dims(h, *[ctypes.byref(x) for x in v]), "bconv_get_output_dims")
    return tuple(x.value for x in v)


def bconv_input_feature_channels(h) -> int:
    return load_library().bconv_input_feature_channels(h)


def bconv_output_feature_channels(h) -> int:
    return load_library().bconv_output_feature_channels(h)


def bfc_input_feature_channels(h) -> int:
    return load_library().bfc_input_feature_channels(h)


def bfc_output_feature_channels(h) -> int:
    return load_library().bfc_output_feature_channels(h)


def bconv_set_algo(h, algo: int):
    _check(load_library().bconv_set_algo(h, int(algo)), "bconv_set_algo")


def bfc_set_algo(h, algo: int):
    _check(load_library().bfc_set_algo(h, int(algo)), "bfc_set_algo")


def bconv_launches_per_forward(h) -> int:
    return load_library().bconv_launches_per_forward(h)


def bfc_launches_per_forward(h) -> int:
    return load_library().bfc_launches_per_forward(h)


def bconv_effective_algo(h) -> int:
    return load_library().bconv_effective_algo(h)


def bfc_effective_algo(h) -> int:
    return load_library().bfc_effective_algo(h)


def bconv_set_cta_mode(mode: int):
    """Spread of the tensor-core contraction for layers created from now on (CTA_*)."""
    _check(load_library().bconv_set_cta_mode(int(mode)), "bconv_set_cta_mode")


def bconv_set_tc_codes(codes: int):
    """Operand codes of the XNOR/AND tensor-core path for layers created from now on (CODES_*)."""
    _check(load_library().bconv_set_tc_codes(int(codes)), "bconv_set_tc_codes")


def bconv_tc_codes(h) -> int:
    return load_library().bconv_tc_codes(h)


def bconv_set_staging(staging: int):
    """Activation staging of the tensor-core contraction for layers created from now on (STAGING_*)."""
    _check(load_library().bconv_set_staging(int(staging)), "bconv_set_staging")


def bconv_staging(h) -> int:
    return load_library().bconv_staging(h)


def bfc_tc_codes(h) -> int:
    return load_library().bfc_tc_codes(h)


def bconv_cta_mode(h) -> int:
    return load_library().bconv_cta_mode(h)


def bfc_cta_mode(h) -> int:
    return load_library().bfc_cta_mode(h)


def bconv_sync_status(h, stream: int = 0):
    _check(load_library().bconv_sync_status(h, stream), "bconv_sync_status")


def bfc_sync_status(h, stream: int = 0):
    _check(load_library().bfc_sync_status(h, stream), "bfc_sync_status")


def bconv_profile_begin(h, max_launches: int):
    _check(load_library().bconv_profile_begin(h, int(max_launches)), "bconv_profile_begin")


def bfc_profile_begin(h, max_launches: int):
    _check(load_library().bfc_profile_begin(h, int(max_launches)), "bfc_profile_begin")


def bconv_profile_stride(h, every: int):
    _check(load_library().bconv_profile_stride(h, int(every)), "bconv_profile_stride")


def bfc_profile_stride(h, every: int):
    _check(load_library().bfc_profile_stride(h, int(every)), "bfc_profile_stride")


def _profile_end(fn, h):
    ms, n = ctypes.c_float(), _I32()
    _check(getattr(load_library(), fn)(h, ctypes.byref(ms), ctypes.byref(n)), fn)
    return ms.value, n.value


def bconv_profile_end(h):
    """Returns (total milliseconds of the timed contraction launches, number of launches)."""
    return _profile_end("bconv_profile_end", h)


def bfc_profile_end(h):
    return _profile_end("bfc_profile_end", h)


def bconv_destroy(h):
    if h is not None:
        _check(load_library().bconv_destroy(h), "bconv_destroy")


def bfc_destroy(h):
    if h is not None:
        _check(load_library().bfc_destroy(h), "bfc_destroy")


def bconv_status_string(status: int) -> str:
    return load_library().bconv_status_string(int(status)).decode()


def bconv_pack_bits(bits) -> np.ndarray:
    """Pack 0/1 bytes of shape [..., nbits] into LSB-first uint32 words [..., ceil(nbits/32)]."""
    b = np.ascontiguousarray(bits, dtype=np.uint8)
    nbits = b.shape[-1]
    rows = b.size // nbits if nbits else 0
    out = np.empty(b.shape[:-1] + ((nbits + 31) // 32,), np.uint32)
    _check(load_library().bconv_pack_bits(_ptr(b), rows, nbits, _ptr(out)), "bconv_pack_bits")
    return out


def bconv_version() -> int:
    return load_library().bconv_version()


def bconv_check_wait_timeout(limit_ms: float = 20.0) -> int:
    """Status of the bounded-wait check (BCONV_ERR_TIMEOUT = 5 is the expected outcome)."""
    return int(load_library().bconv_check_wait_timeout(float(limit_ms)))


def bconv_measure_peak(kind: int):
    """Returns (ops per second, SM MHz) for probe kind 0 (POPC), 1 (LOP3), 2 (b1 mma.sync),
    3 (tcgen05 kind::i8 M128 N256) or 4 (tcgen05 kind::f16 bf16 M128 N256) on zero operands,
    5 or 6 (kinds 3 and 4 on pseudo-random +-1 operands)."""
    ops, mhz = ctypes.c_double(), ctypes.c_double()
    _check(load_library().bconv_measure_peak(int(kind), ctypes.byref(ops), ctypes.byref(mhz)), "bconv_measure_peak")
    return ops.value, mhz.value


def bconv_forward_noalloc(desc: bconv_desc_t, type: int, flags: int, weights_ptr: int, scale_ptr: int | None,
                          bias_ptr: int | None, in_scale_ptr: int | None, in_bias_ptr: int | None, in_ptr: int,
                          out_ptr: int, stream: int = 0):
    """XNOR/AND forward that allocates nothing; every pointer is a device address (or None)."""
    _check(load_library().bconv_forward_noalloc(ctypes.byref(desc), int(type), int(flags), weights_ptr, scale_ptr,
                                                bias_ptr, in_scale_ptr, in_bias_ptr, in_ptr, out_ptr, stream),
           "bconv_forward_noalloc")
