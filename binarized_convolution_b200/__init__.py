"""B200-native binary convolution (XNOR / AND / binaryWeights) behind a C-ABI library.

This package is a thin ctypes binding over ``libbconv.so`` (built in-tree by
``python -m binarized_convolution_b200.build``).  The functions named like the C entry
points (``bconv_create``, ``bconv_forward``, ``bfc_create``, ...) only marshal arguments;
every step of the computation runs in the library's CUDA kernels.  PyTorch supplies device
memory and the current CUDA stream in the convenience classes :class:`BinaryConv2d` and
:class:`BinaryFC`.

There is no CPU fallback: if the library is missing or no CUDA device is visible, the calls
raise.
"""
from __future__ import annotations

from ._native import (  # noqa: F401
    ALGO_AUTO,
    ALGO_POPC,
    ALGO_SIMT_F32,
    ALGO_TCGEN05,
    CODES_AUTO,
    CODES_BF16X3,
    CODES_FP4,
    CODES_INT8,
    CTA_AUTO,
    CTA_PAIR,
    CTA_SINGLE,
    FLAG_NONE,
    FLAG_USE_BETA_SCALING,
    NEURON_NONE,
    NEURON_RELU,
    TYPE_AND,
    TYPE_BINARY_WEIGHTS,
    TYPE_XNOR,
    BconvError,
    bconv_create,
    bconv_cta_mode,
    bconv_set_cta_mode,
    bconv_set_tc_codes,
    bconv_tc_codes,
    bconv_desc_t,
    bconv_destroy,
    bconv_effective_algo,
    bconv_forward,
    bconv_forward_host,
    bconv_forward_noalloc,
    bconv_forward_io,
    bconv_check_wait_timeout,
    bconv_set_output_terms,
    bconv_io_t,
    bfc_forward_io,
    bfc_set_output_terms,
    NOALLOC_SCRATCH_BYTES,
    bconv_get_output_dims,
    bconv_input_feature_channels,
    bconv_launches_per_forward,
    bconv_measure_peak,
    bconv_output_feature_channels,
    bconv_pack_bits,
    bconv_profile_begin,
    bconv_profile_end,
    bconv_profile_stride,
    bconv_set_algo,
    bconv_status_string,
    bconv_sync_status,
    bconv_version,
    bfc_create,
    bfc_cta_mode,
    bfc_tc_codes,
    bfc_desc_t,
    bfc_destroy,
    bfc_effective_algo,
    bfc_forward,
    bfc_forward_host,
    bfc_input_feature_channels,
    bfc_launches_per_forward,
    bfc_output_feature_channels,
    bfc_profile_begin,
    bfc_profile_end,
    bfc_profile_stride,
    bfc_set_algo,
    bfc_sync_status,
    exported_symbols,
    library_path,
    load_library,
)
from .layers import BinaryConv2d, BinaryFC  # noqa: F401
