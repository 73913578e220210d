"""bconv_forward_noalloc, the forward for callers that cannot allocate device memory (code
whose memory belongs to its own pool, real-time loops, work issued during graph capture).

It is called through the C ABI and its output is compared with the regular
bconv_create + bconv_forward path, within the float tolerance the parity tests use, on two
calls in a row with different inputs (the second must not see the first call's scratch
contents).  This file is collected last so that a run stopping at the first failure has run
every other test before it.
"""
import numpy as np
import pytest

import binarized_convolution_b200 as bc
import oracle
from binarized_convolution_b200 import _native as nat
from binarized_convolution_b200 import synth
import parity_util as pu

pytestmark = pytest.mark.gpu

CASES = [
    synth.small_case(batch=2, h=19, w=17, ni=70, no=150, k=3, op=synth.XNOR, use_beta=True, relu=True,
                     in_terms=True, seed=501),
    synth.small_case(batch=2, h=12, w=13, ni=512, no=40, k=3, op=synth.AND, use_beta=False, relu=False, p=0.3,
                     seed=502),
    synth.workload(1),  # XNOR + beta + input terms, batch 16, 56x56, 256 -> 256
]


def _noalloc_forward(w, inp, x_dev, stream):
    import torch

    dev = x_dev.device
    packed = torch.from_numpy(bc.bconv_pack_bits(inp.wbits).view(np.int32)).to(dev)
    scale = torch.from_numpy(inp.scale).to(dev)
    bias = torch.from_numpy(inp.bias).to(dev)
    in_s = torch.from_numpy(inp.in_scale).to(dev) if inp.in_scale is not None else None
    in_b = torch.from_numpy(inp.in_bias).to(dev) if inp.in_bias is not None else None
    out = torch.empty((w.batch, w.out_h, w.out_w, w.out_channels), dtype=torch.float32, device=dev)
    desc = nat.bconv_desc_t(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, w.kernel_h, w.kernel_w,
                            w.stride_y, w.stride_x, 1, nat.NEURON_RELU if w.relu else nat.NEURON_NONE, 1.0)
    op = {synth.XNOR: nat.TYPE_XNOR, synth.AND: nat.TYPE_AND}[w.op]
    flags = nat.FLAG_USE_BETA_SCALING if w.use_beta else nat.FLAG_NONE
    bc.bconv_forward_noalloc(desc, op, flags, packed.data_ptr(), scale.data_ptr(), bias.data_ptr(),
                             in_s.data_ptr() if in_s is not None else None,
                             in_b.data_ptr() if in_b is not None else None, x_dev.data_ptr(), out.data_ptr(),
                             stream.cuda_stream)
    return out


def _regular_forward(w, inp, x_np, sums=False):
    layer = pu.make_layer(w, inp, sums=sums)
    try:
        import torch

        y = layer(torch.from_numpy(x_np).cuda())
        layer.sync_status()
        return y.reshape(-1, w.out_channels).cpu().numpy()
    finally:
        layer.close()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_regular_forward_twice(w, cuda_device):
    import torch

    inp = synth.make_inputs(w)
    stream = torch.cuda.current_stream()
    for call, seed in enumerate((w.seed + 11, w.seed + 12)):
        x = synth.make_batch(w, seed=seed)
        y_new = _noalloc_forward(w, inp, torch.from_numpy(x).cuda(), stream)
        torch.cuda.synchronize()
        y_new = y_new.reshape(-1, w.out_channels).cpu().numpy()
        xin = synth.Inputs(x, inp.wbits, inp.scale, inp.bias, inp.in_scale, inp.in_bias)
        y_ref = _regular_forward(w, xin, x).astype(np.float64)
        S = _regular_forward(w, xin, x, sums=True).astype(np.float64)
        # beta does not depend on the weights: one output channel of the oracle gives it cheaply
        _, beta, _ = oracle.conv(x, inp.wbits[:1], type=oracle.ORACLE_XNOR, stride=(w.stride_y, w.stride_x),
                                 in_scale=inp.in_scale, in_bias=inp.in_bias, use_beta=w.use_beta)
        err = pu.relative_errors(w, xin, y_new, S, beta, y_ref)
        assert err.max() <= pu.REL_TOL, f"call {call}: max error {err.max():.3e}"


def test_noalloc_rejects_oversize_and_bad_arguments(cuda_device):
    lib = bc.load_library()
    import ctypes

    big = nat.bconv_desc_t(64, 224, 224, 512, 512, 3, 3, 1, 1, 1, 0, 1.0)  # bits alone need 205 MB
    st = lib.bconv_forward_noalloc(ctypes.byref(big), nat.TYPE_XNOR, 0, 16, None, None, None, None, 16, 16, None)
    assert st == 2  # BCONV_ERR_UNSUPPORTED, before any device work
    ok = nat.bconv_desc_t(1, 4, 4, 8, 2, 3, 3, 1, 1, 1, 0, 1.0)
    assert lib.bconv_forward_noalloc(ctypes.byref(ok), nat.TYPE_BINARY_WEIGHTS, 0, 16, None, None, None, None, 16,
                                     16, None) == 1
    assert lib.bconv_forward_noalloc(ctypes.byref(ok), nat.TYPE_XNOR, 0, None, None, None, None, None, 16, 16,
                                     None) == 1
