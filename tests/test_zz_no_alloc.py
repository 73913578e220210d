"""bconv_forward_noalloc, the forward for callers that cannot allocate device memory when they
run a layer (code whose device memory all belongs to its own pool allocator, or real-time
loops where an allocation may stall on a device-wide synchronisation).

It is called through the C ABI.  Its output is compared with the regular bconv_create +
bconv_forward path within the float tolerance the parity tests use, and with the oracle: the
raw integer window sums bit for bit (scale and bias left out, so the entry point's own
defaults apply: scale 1, bias 0; no beta; identity neuron), and the float outputs within the
tolerance with each optional operand left out in turn.  Every comparison runs on two calls
in a row with different inputs (the second must not see the first call's scratch
contents), and a repeated call must leave the device's free memory unchanged.  This file is
collected last so that a run stopping at the first failure has run every other test first.
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

SUM_CASES = [
    synth.small_case(batch=3, h=11, w=14, ni=100, no=36, k=3, op=synth.XNOR, in_terms=True, seed=511),
    synth.small_case(batch=2, h=9, w=10, ni=64, no=20, k=5, stride=2, op=synth.AND, p=0.3, seed=512),
]

_OTYPE = {synth.XNOR: oracle.ORACLE_XNOR, synth.AND: oracle.ORACLE_AND}


def _dev(a):
    import torch

    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _noalloc_forward(w, wbits, x_dev, stream, *, scale=None, bias=None, in_scale=None, in_bias=None,
                     use_beta=None, relu=None, scale_value=1.0):
    """One call through the C ABI; operands given as host arrays (or None) go to the device first."""
    import torch

    dev = x_dev.device
    packed = torch.from_numpy(bc.bconv_pack_bits(wbits).view(np.int32)).to(dev)
    ops = [_dev(a) for a in (scale, bias, in_scale, in_bias)]
    use_beta = w.use_beta if use_beta is None else use_beta
    relu = w.relu if relu is None else relu
    out = torch.empty((w.batch, w.out_h, w.out_w, w.out_channels), dtype=torch.float32, device=dev)
    desc = nat.bconv_desc_t(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, w.kernel_h, w.kernel_w,
                            w.stride_y, w.stride_x, 1, nat.NEURON_RELU if relu else nat.NEURON_NONE, scale_value)
    flags = nat.FLAG_USE_BETA_SCALING if use_beta else nat.FLAG_NONE
    bc.bconv_forward_noalloc(desc, {synth.XNOR: nat.TYPE_XNOR, synth.AND: nat.TYPE_AND}[w.op], flags,
                             packed.data_ptr(), *[None if t is None else t.data_ptr() for t in ops],
                             x_dev.data_ptr(), out.data_ptr(), stream.cuda_stream)
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
        y_new = _noalloc_forward(w, inp.wbits, torch.from_numpy(x).cuda(), stream, scale=inp.scale, bias=inp.bias,
                                 in_scale=inp.in_scale, in_bias=inp.in_bias)
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


@pytest.mark.parametrize("w", SUM_CASES, ids=lambda w: w.name)
def test_noalloc_integer_sums_equal_the_oracle_twice(w, cuda_device):
    """Scale and bias left out (so the entry point fills in scale_value = 1 and bias 0), no beta,
    identity neuron: the output is the window sum S, which must equal the oracle's bit for bit."""
    import torch

    inp = synth.make_inputs(w)
    stream = torch.cuda.current_stream()
    for seed in (w.seed + 21, w.seed + 22):
        x = synth.make_batch(w, seed=seed)
        y = _noalloc_forward(w, inp.wbits, torch.from_numpy(x).cuda(), stream, in_scale=inp.in_scale,
                             in_bias=inp.in_bias, use_beta=False, relu=False)
        torch.cuda.synchronize()
        y = y.reshape(-1, w.out_channels).cpu().numpy()
        S, _, _ = oracle.conv(x, inp.wbits, type=_OTYPE[w.op], stride=(w.stride_y, w.stride_x),
                              in_scale=inp.in_scale, in_bias=inp.in_bias)
        assert np.abs(S).max() < 2 ** 24  # every sum is exact in fp32
        pu.assert_sums_exact(y, S)


@pytest.mark.parametrize("missing", ["scale", "bias", "in_scale", "in_bias"])
def test_noalloc_fills_each_missing_operand_like_the_oracle(missing, cuda_device):
    """Each optional operand left out in turn (scale -> scale_value, bias -> 0, in_scale -> 1,
    in_bias -> 0), with beta and ReLU on, against the oracle given the same NULL."""
    import torch

    w = synth.small_case(batch=2, h=10, w=9, ni=45, no=24, k=3, op=synth.XNOR, use_beta=True, relu=True,
                         in_terms=True, seed=530)
    inp = synth.make_inputs(w)
    ops = dict(scale=inp.scale, bias=inp.bias, in_scale=inp.in_scale, in_bias=inp.in_bias)
    ops[missing] = None
    stream = torch.cuda.current_stream()
    for seed in (531, 532):
        x = synth.make_batch(w, seed=seed)
        y = _noalloc_forward(w, inp.wbits, torch.from_numpy(x).cuda(), stream, scale_value=0.75, **ops)
        torch.cuda.synchronize()
        y = y.reshape(-1, w.out_channels).cpu().numpy().astype(np.float64)
        S, beta, y_ref = oracle.conv(x, inp.wbits, type=oracle.ORACLE_XNOR, scale_value=0.75, use_beta=True,
                                     relu=True, **ops)
        scale = ops["scale"] if ops["scale"] is not None else np.full(w.out_channels, 0.75, np.float32)
        bias = ops["bias"] if ops["bias"] is not None else np.zeros(w.out_channels, np.float32)
        D = np.abs(scale.astype(np.float64))[None, :] * np.abs(beta)[:, None] * np.abs(S) + np.abs(bias)[None, :]
        err = np.abs(y - y_ref) / np.maximum(np.maximum(np.abs(y_ref), D), 1e-30)
        assert err.max() <= pu.REL_TOL, f"{missing} missing: max error {err.max():.3e}"


def test_noalloc_repeated_call_leaves_free_memory_unchanged(cuda_device):
    """After a first call (which looks up the scratch array's address and may load kernels), a
    call must not change the device's free memory: it allocates nothing."""
    import torch

    w = SUM_CASES[0]
    inp = synth.make_inputs(w)
    stream = torch.cuda.current_stream()
    x = torch.from_numpy(inp.x).cuda()
    packed = torch.from_numpy(bc.bconv_pack_bits(inp.wbits).view(np.int32)).cuda()
    out = torch.empty((w.batch, w.out_h, w.out_w, w.out_channels), dtype=torch.float32, device="cuda")
    desc = nat.bconv_desc_t(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, w.kernel_h, w.kernel_w,
                            w.stride_y, w.stride_x, 1, nat.NEURON_NONE, 1.0)

    def call():
        bc.bconv_forward_noalloc(desc, nat.TYPE_XNOR, nat.FLAG_USE_BETA_SCALING, packed.data_ptr(), None, None,
                                 None, None, x.data_ptr(), out.data_ptr(), stream.cuda_stream)

    call()
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before


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
