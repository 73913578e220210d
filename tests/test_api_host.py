"""The C-ABI library on the host (no GPU needed): it loads, exports every symbol the header
declares, packs bits as documented, and rejects bad arguments with a status instead of
crashing."""
import ctypes

import numpy as np
import pytest

import binarized_convolution_b200 as bc
from binarized_convolution_b200 import _native as nat


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(bc.library_path())
    names = bc.exported_symbols()
    assert set(names) == set(nat._SIGS), set(names) ^ set(nat._SIGS)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_symbol():
    for n in bc.exported_symbols():
        assert hasattr(bc, n), n


def test_pack_bits_lsb_first():
    rng = np.random.default_rng(0)
    for nbits in (1, 5, 31, 32, 33, 64, 100):
        bits = (rng.random((7, nbits)) < 0.5).astype(np.uint8)
        words = bc.bconv_pack_bits(bits)
        assert words.shape == (7, (nbits + 31) // 32)
        padded = np.zeros((7, words.shape[1] * 32), np.uint8)
        padded[:, :nbits] = bits
        ref = np.packbits(padded, axis=1, bitorder="little").view("<u4")
        np.testing.assert_array_equal(words, ref)
        for r in range(7):
            for f in range(nbits):
                assert ((int(words[r, f // 32]) >> (f % 32)) & 1) == bits[r, f]


def test_pack_bits_nonzero_bytes_are_ones():
    words = bc.bconv_pack_bits(np.array([[0, 2, 255, 0, 1]], np.uint8))
    assert int(words[0, 0]) == 0b10110


def test_status_strings_and_version():
    for s in range(7):
        assert bc.bconv_status_string(s)
    assert bc.bconv_status_string(99) == "unknown status"
    assert bc.bconv_version() >= 100


def _desc(**kw):
    d = dict(batch=1, in_h=4, in_w=4, in_channels=8, out_channels=2, kernel_h=3, kernel_w=3, stride_y=1, stride_x=1,
             groups=1, neuron=0, scale_value=1.0)
    d.update(kw)
    return nat.bconv_desc_t(**d)


def _create_status(desc, weights=True, type=1, flags=0):
    lib = bc.load_library()
    n = desc.out_channels * desc.kernel_h * desc.kernel_w * ((desc.in_channels + 31) // 32)
    w = np.zeros(max(n, 0) + 1, np.uint32)
    h = ctypes.c_void_p()
    st = lib.bconv_create(ctypes.byref(desc), w.ctypes.data_as(ctypes.c_void_p) if weights else None, None, None,
                          None, None, type, flags, ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("kw,expect", [
    (dict(groups=2), 2),
    (dict(groups=0), 1),
    (dict(in_channels=0), 1),
    (dict(out_channels=-1), 1),
    (dict(kernel_h=0), 1),
    (dict(stride_x=0), 1),
    (dict(batch=-1), 1),
    (dict(neuron=7), 1),
])
def test_create_rejects_bad_descriptors(kw, expect):
    st, h = _create_status(_desc(**kw))
    assert st == expect
    assert h.value is None


def test_create_rejects_bad_type_flags_and_pointers():
    assert _create_status(_desc(), type=3)[0] == 1
    assert _create_status(_desc(), flags=2)[0] == 1
    assert _create_status(_desc(), weights=False)[0] == 1
    lib = bc.load_library()
    h = ctypes.c_void_p()
    assert lib.bconv_create(None, None, None, None, None, None, 1, 0, ctypes.byref(h)) == 1
    assert lib.bconv_create(ctypes.byref(_desc()), None, None, None, None, None, 1, 0, None) == 1


def test_fc_create_validates_stride_and_groups():
    lib = bc.load_library()
    w = np.zeros(2 * 4 * 4 * 1, np.uint32)
    for stride, groups, expect in ((2, 1, 1), (1, 3, 2)):
        d = nat.bfc_desc_t(1, 4, 4, 8, 2, stride, 1, groups, 0, 1.0)
        h = ctypes.c_void_p()
        assert lib.bfc_create(ctypes.byref(d), w.ctypes.data_as(ctypes.c_void_p), None, None, None, None, 1, 0,
                              ctypes.byref(h)) == expect


def test_calls_on_null_or_foreign_handles_return_errors():
    lib = bc.load_library()
    assert lib.bconv_forward(None, None, None, None) == 1
    assert lib.bfc_forward(None, None, None, None) == 1
    assert lib.bconv_destroy(None) == 0
    assert lib.bfc_destroy(None) == 0
    assert lib.bconv_input_feature_channels(None) == -1
    assert lib.bfc_output_feature_channels(None) == -1
    assert lib.bconv_launches_per_forward(None) == -1
    junk = (ctypes.c_uint32 * 64)()
    assert lib.bconv_forward(ctypes.cast(junk, ctypes.c_void_p), None, None, None) == 1
    assert lib.bconv_destroy(ctypes.cast(junk, ctypes.c_void_p)) == 1
    assert lib.bconv_pack_bits(None, 1, 1, None) == 1
    assert lib.bconv_cta_mode(None) == -1
    assert lib.bfc_cta_mode(None) == -1
    assert lib.bconv_tc_codes(None) == -1
    assert lib.bfc_tc_codes(None) == -1


def test_cta_mode_setting_is_validated():
    lib = bc.load_library()
    for bad in (-1, 3, 100):
        assert lib.bconv_set_cta_mode(bad) == 1  # INVALID_ARG
    for good in (bc.CTA_SINGLE, bc.CTA_PAIR, bc.CTA_AUTO):
        assert lib.bconv_set_cta_mode(good) == 0
    for bad in (-1, 3, 7):  # BF16X3 is reported, not chosen
        assert lib.bconv_set_tc_codes(bad) == 1
    for good in (bc.CODES_INT8, bc.CODES_FP4, bc.CODES_AUTO):
        assert lib.bconv_set_tc_codes(good) == 0


def test_create_without_a_device_reports_no_device():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    st, h = _create_status(_desc())
    assert st == 6
    ops = ctypes.c_double()
    assert bc.load_library().bconv_measure_peak(0, ctypes.byref(ops), None) == 6


def test_python_layer_raises_on_bad_input():
    with pytest.raises((bc.BconvError, ValueError)):
        bc.BinaryConv2d(1, 4, 4, 8, 2, 3, 1, wbits=np.zeros((2, 3, 3, 8), np.uint8), groups=2)


@pytest.mark.parametrize("kw", [
    dict(kernel_h=65536, kernel_w=65536, in_h=1 << 20, in_w=1 << 20),  # 2^32 taps: rejected before any product
    dict(kernel_h=10, in_h=4),                                          # wider than 2 x the image + 1
    dict(kernel_h=4097, in_h=4096),
    dict(kernel_h=64, kernel_w=64, in_h=64, in_w=64, in_channels=1 << 20),  # 2^32-term sums overflow int32
])
def test_create_and_noalloc_reject_the_same_oversize_shapes(kw):
    """bconv_create and bconv_forward_noalloc share one shape check (status 2 = UNSUPPORTED),
    returned on the host before any weight is read or any device work is queued."""
    lib = bc.load_library()
    d = _desc(**kw)
    dummy = (ctypes.c_uint32 * 4)()
    h = ctypes.c_void_p()
    assert lib.bconv_create(ctypes.byref(d), dummy, None, None, None, None, 1, 0, ctypes.byref(h)) == 2
    assert h.value is None
    assert lib.bconv_forward_noalloc(ctypes.byref(d), nat.TYPE_XNOR, 0, 16, None, None, None, None, 16, 16,
                                     None) == 2
