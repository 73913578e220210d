"""Layer objects over the C ABI: own a handle, take torch CUDA tensors, use the current stream.

These classes only marshal: they pack the weight bits with the library's own packer,
allocate the output tensor with torch, and call ``bconv_forward`` / ``bfc_forward`` on
``torch.cuda.current_stream()``.
"""
from __future__ import annotations

import numpy as np

from . import _native as nat

_TYPES = {"xnor": nat.TYPE_XNOR, "and": nat.TYPE_AND, "binary_weights": nat.TYPE_BINARY_WEIGHTS}


def _type_code(op) -> int:
    return _TYPES[op] if isinstance(op, str) else int(op)


def _require_cuda(x):
    import torch

    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise TypeError("expected a CUDA tensor")
    if x.dtype != torch.float32:
        raise TypeError("expected float32")
    return x.contiguous()


class _Layer:
    _destroy = None

    def close(self):
        if getattr(self, "handle", None) is not None:
            type(self)._destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 -- interpreter shutdown
            pass

    # ---- chained binary layers (bit-packed activations; see bconv_forward_io) ----
    def set_output_terms(self, next_in_scale=None, next_in_bias=None):
        """The input terms of the layer that will read this layer's bit-packed output."""
        type(self)._set_output_terms(self.handle, next_in_scale, next_in_bias)

    def bits_shape(self):
        """Shapes of this layer's bit-packed output: (32-bit words, A)."""
        *lead, c = self.out_dims
        return (*lead, (c + 31) // 32), tuple(lead)

    def forward_io(self, x=None, x_bits=None, x_a=None, out=None, out_bits=None, out_a=None):
        """Device tensors in either form: fp32 ``x`` or ``x_bits`` (+ ``x_a``); fp32 ``out`` or
        ``out_bits`` + ``out_a``.  Bit tensors hold the uint32 words (any 32-bit dtype)."""
        import torch

        def p(t):
            return None if t is None else t.data_ptr()

        type(self)._forward_io(self.handle, p(x), p(x_bits), p(x_a), p(out), p(out_bits), p(out_a),
                               torch.cuda.current_stream().cuda_stream)

    def forward_to_bits(self, x=None, x_bits=None, x_a=None):
        """Run the layer and return its output as (bits, A) device tensors (bits as int32)."""
        import torch

        src = x if x is not None else x_bits
        bshape, ashape = self.bits_shape()
        bits = torch.empty(bshape, dtype=torch.int32, device=src.device)
        a = torch.empty(ashape, dtype=torch.float32, device=src.device)
        self.forward_io(x=x, x_bits=x_bits, x_a=x_a, out_bits=bits, out_a=a)
        return bits, a

    def forward_from_bits(self, x_bits, x_a=None):
        """Run the layer on bit-packed input; returns the fp32 output tensor."""
        import torch

        out = torch.empty(self.out_dims, dtype=torch.float32, device=x_bits.device)
        self.forward_io(x_bits=x_bits, x_a=x_a, out=out)
        return out

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


class BinaryConv2d(_Layer):
    """A binary convolution (MPSCNNBinaryConvolution) on the current CUDA device.

    wbits: uint8 0/1 array [out_channels, kernel_h, kernel_w, in_channels] (or pass
    ``packed`` uint32 words [out_channels, kernel_h, kernel_w, ceil(in_channels/32)]).
    """

    _destroy = staticmethod(nat.bconv_destroy)
    _set_output_terms = staticmethod(nat.bconv_set_output_terms)
    _forward_io = staticmethod(nat.bconv_forward_io)

    def __init__(self, batch, in_h, in_w, in_channels, out_channels, kernel=(3, 3), stride=(1, 1), *,
                 wbits=None, packed=None, op="xnor", scale=None, scale_value=1.0, bias=None, in_scale=None,
                 in_bias=None, use_beta=False, relu=False, groups=1):
        kh, kw = (kernel, kernel) if isinstance(kernel, int) else kernel
        sy, sx = (stride, stride) if isinstance(stride, int) else stride
        if packed is None:
            if wbits is None:
                raise ValueError("give wbits or packed")
            packed = nat.bconv_pack_bits(np.asarray(wbits).reshape(out_channels, kh, kw, in_channels))
        self.desc = nat.bconv_desc_t(batch, in_h, in_w, in_channels, out_channels, kh, kw, sy, sx, groups,
                                     nat.NEURON_RELU if relu else nat.NEURON_NONE, scale_value)
        flags = nat.FLAG_USE_BETA_SCALING if use_beta else nat.FLAG_NONE
        self.handle = None
        self.handle = nat.bconv_create(self.desc, packed, scale, bias, in_scale, in_bias, _type_code(op), flags)
        self.out_dims = nat.bconv_get_output_dims(self.handle)

    @property
    def input_feature_channels(self) -> int:
        return nat.bconv_input_feature_channels(self.handle)

    @property
    def output_feature_channels(self) -> int:
        return nat.bconv_output_feature_channels(self.handle)

    def set_algo(self, algo: int):
        nat.bconv_set_algo(self.handle, algo)

    def launches_per_forward(self) -> int:
        return nat.bconv_launches_per_forward(self.handle)

    def effective_algo(self) -> int:
        return nat.bconv_effective_algo(self.handle)

    def cta_mode(self) -> int:
        return nat.bconv_cta_mode(self.handle)

    def tc_codes(self) -> int:
        return nat.bconv_tc_codes(self.handle)

    def staging(self) -> int:
        """How the tensor-core contraction brings in its activations: STAGING_PER_TAP, STAGING_ROWS
        (XNOR/AND, stride 1) or STAGING_INPUT (binaryWeights from the fp32 input, no pack
        kernel); 0 without a tensor-core path."""
        return nat.bconv_staging(self.handle)

    def forward_into(self, x, out):
        import torch

        nat.bconv_forward(self.handle, x.data_ptr(), out.data_ptr(), torch.cuda.current_stream().cuda_stream)
        return out

    def __call__(self, x):
        import torch

        x = _require_cuda(x)
        out = torch.empty(self.out_dims, dtype=torch.float32, device=x.device)
        return self.forward_into(x, out)

    def forward_host(self, x_host: np.ndarray, out_host: np.ndarray | None = None, stream: int = 0):
        if out_host is None:
            out_host = np.empty(self.out_dims, np.float32)
        x_host = np.ascontiguousarray(x_host, dtype=np.float32)
        nat.bconv_forward_host(self.handle, x_host.ctypes.data, out_host.ctypes.data, stream)
        return out_host

    def sync_status(self, stream: int = 0):
        nat.bconv_sync_status(self.handle, stream)


class BinaryFC(_Layer):
    """A binary fully-connected layer (kernel = source size, MPSCNNFullyConnected).

    wbits: uint8 0/1 array [out_channels, in_h, in_w, in_channels] (or ``packed`` words).
    """

    _destroy = staticmethod(nat.bfc_destroy)
    _set_output_terms = staticmethod(nat.bfc_set_output_terms)
    _forward_io = staticmethod(nat.bfc_forward_io)

    def __init__(self, batch, in_h, in_w, in_channels, out_channels, *, wbits=None, packed=None, op="xnor",
                 scale=None, scale_value=1.0, bias=None, in_scale=None, in_bias=None, use_beta=False, relu=False,
                 stride=(1, 1), groups=1):
        sy, sx = (stride, stride) if isinstance(stride, int) else stride
        if packed is None:
            if wbits is None:
                raise ValueError("give wbits or packed")
            packed = nat.bconv_pack_bits(np.asarray(wbits).reshape(out_channels, in_h, in_w, in_channels))
        self.desc = nat.bfc_desc_t(batch, in_h, in_w, in_channels, out_channels, sy, sx, groups,
                                   nat.NEURON_RELU if relu else nat.NEURON_NONE, scale_value)
        flags = nat.FLAG_USE_BETA_SCALING if use_beta else nat.FLAG_NONE
        self.handle = None
        self.handle = nat.bfc_create(self.desc, packed, scale, bias, in_scale, in_bias, _type_code(op), flags)
        self.out_dims = (batch, out_channels)

    @property
    def input_feature_channels(self) -> int:
        return nat.bfc_input_feature_channels(self.handle)

    @property
    def output_feature_channels(self) -> int:
        return nat.bfc_output_feature_channels(self.handle)

    def set_algo(self, algo: int):
        nat.bfc_set_algo(self.handle, algo)

    def launches_per_forward(self) -> int:
        return nat.bfc_launches_per_forward(self.handle)

    def effective_algo(self) -> int:
        return nat.bfc_effective_algo(self.handle)

    def cta_mode(self) -> int:
        return nat.bfc_cta_mode(self.handle)

    def tc_codes(self) -> int:
        return nat.bfc_tc_codes(self.handle)

    def forward_into(self, x, out):
        import torch

        nat.bfc_forward(self.handle, x.data_ptr(), out.data_ptr(), torch.cuda.current_stream().cuda_stream)
        return out

    def __call__(self, x):
        import torch

        x = _require_cuda(x)
        out = torch.empty(self.out_dims, dtype=torch.float32, device=x.device)
        return self.forward_into(x, out)

    def forward_host(self, x_host: np.ndarray, out_host: np.ndarray | None = None, stream: int = 0):
        if out_host is None:
            out_host = np.empty(self.out_dims, np.float32)
        x_host = np.ascontiguousarray(x_host, dtype=np.float32)
        nat.bfc_forward_host(self.handle, x_host.ctypes.data, out_host.ctypes.data, stream)
        return out_host

    def sync_status(self, stream: int = 0):
        nat.bfc_sync_status(self.handle, stream)
