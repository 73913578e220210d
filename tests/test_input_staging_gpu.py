"""binaryWeights convolutions on the fp32-input contraction (staging INPUT): the kernel loads the
fp32 input per tap and forms x~ and its three bf16 parts in shared memory.

Each case is compared with the oracle on every output, and with the same layer on the parts
buffer (staging PER_TAP, one SM per tile) bit for bit: both form x~ = fma(x, in_scale, in_bias),
split it the same way and accumulate the same products in the same order.  The cases span
channel counts that leave part of the last 64-channel k-block empty, strides 1 and 2, 1 x 1 to
5 x 5 windows, ragged tiles and images smaller than a tile.
"""
import numpy as np
import pytest

from binarized_convolution_b200 import synth
import binarized_convolution_b200 as bc
import parity_util as pu

pytestmark = pytest.mark.gpu

CASES = [
    synth.small_case(batch=2, h=19, w=17, ni=36, no=40, k=3, op=synth.BINARY_WEIGHTS, use_beta=False, relu=True,
                     in_terms=True, seed=701),
    synth.small_case(batch=3, h=16, w=16, ni=128, no=128, k=3, stride=2, op=synth.BINARY_WEIGHTS, use_beta=False,
                     relu=False, in_terms=False, seed=702),
    synth.small_case(batch=1, h=23, w=29, ni=200, no=96, k=5, stride=2, op=synth.BINARY_WEIGHTS, use_beta=False,
                     relu=True, in_terms=True, seed=703),
    synth.small_case(batch=4, h=9, w=11, ni=64, no=100, k=1, op=synth.BINARY_WEIGHTS, use_beta=False, relu=False,
                     in_terms=True, seed=704),
    synth.small_case(batch=1, h=5, w=6, ni=12, no=32, k=3, op=synth.BINARY_WEIGHTS, use_beta=False, relu=False,
                     in_terms=True, seed=705),
    synth.small_case(batch=2, h=30, w=30, ni=68, no=128, k=3, op=synth.BINARY_WEIGHTS, use_beta=False, relu=True,
                     in_terms=False, seed=706),
    # edges: the fewest channels, a wide reduction (32 k-blocks a tap), even and non-square
    # windows, different strides per axis, a 1 x 1 image, a few output channels, and a batch
    # whose last tile holds one image
    synth.small_case(batch=3, h=7, w=9, ni=4, no=16, k=3, op=synth.BINARY_WEIGHTS, in_terms=True, seed=707),
    synth.small_case(batch=1, h=6, w=7, ni=2048, no=64, k=3, op=synth.BINARY_WEIGHTS, in_terms=True, relu=True,
                     seed=708),
    synth.small_case(batch=2, h=13, w=12, ni=96, no=48, k=2, op=synth.BINARY_WEIGHTS, in_terms=True, seed=709),
    synth.small_case(batch=2, h=11, w=14, ni=40, no=24, k=3, kw=1, stride=1, stride_x=2, op=synth.BINARY_WEIGHTS,
                     in_terms=True, seed=710),
    synth.small_case(batch=5, h=1, w=1, ni=64, no=8, k=3, op=synth.BINARY_WEIGHTS, in_terms=True, seed=711),
    synth.small_case(batch=9, h=8, w=8, ni=64, no=128, k=5, stride=2, op=synth.BINARY_WEIGHTS, relu=True,
                     in_terms=False, seed=712),
]


def _forward(w, inp, staging):
    bc.bconv_set_staging(staging)
    bc.bconv_set_cta_mode(bc.CTA_SINGLE)
    try:
        layer = pu.make_layer(w, inp)
    finally:
        bc.bconv_set_staging(bc.STAGING_AUTO)
        bc.bconv_set_cta_mode(bc.CTA_AUTO)
    try:
        import torch
        y = layer(torch.from_numpy(inp.x).cuda())
        layer.sync_status()
        return layer.staging(), y.reshape(-1, w.out_channels).cpu().numpy()
    finally:
        layer.close()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_input_staging_parity(w, cuda_device):
    inp = synth.make_inputs(w)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp)
    st, y = _forward(w, inp, bc.STAGING_AUTO)
    assert st == bc.STAGING_INPUT
    pu.assert_outputs_close(w, inp, y, S_ref, beta_ref, y_ref)
    st2, y2 = _forward(w, inp, bc.STAGING_PER_TAP)
    assert st2 == bc.STAGING_PER_TAP
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))


def test_input_staging_choice(cuda_device):
    """INPUT where it applies; beta, in_c % 4 != 0, more than 128 output channels, a forced
    per-tap setting and a bit-packed output keep the parts buffer."""
    def layer(ni=64, use_beta=False, no=64, **kw):
        c = synth.small_case(batch=2, h=12, w=12, ni=ni, no=no, k=3, op=synth.BINARY_WEIGHTS, use_beta=use_beta,
                             seed=9, **kw)
        return pu.make_layer(c, synth.make_inputs(c))

    with layer() as l:
        assert l.staging() == bc.STAGING_INPUT and l.tc_codes() == bc.CODES_BF16X3
        assert l.launches_per_forward() == 1  # no pack kernel
    with layer(use_beta=True) as l:
        assert l.staging() == bc.STAGING_PER_TAP
        assert l.launches_per_forward() == 2
    with layer(ni=30) as l:
        assert l.staging() == bc.STAGING_PER_TAP
    with layer(no=160) as l:  # more than 128 output channels
        assert l.staging() == bc.STAGING_PER_TAP
    with layer() as l:
        l.set_output_terms(None, None)
        assert l.staging() == bc.STAGING_PER_TAP
    bc.bconv_set_staging(bc.STAGING_PER_TAP)
    try:
        with layer() as l:
            assert l.staging() == bc.STAGING_PER_TAP
    finally:
        bc.bconv_set_staging(bc.STAGING_AUTO)


def test_input_not_16_byte_aligned(cuda_device):
    """An input 4 bytes past a 16-byte boundary cannot be mapped for the TMA: that forward runs
    on the SIMT family and must still match the oracle; an aligned one after it is back on the
    tensor cores."""
    import torch

    w = CASES[0]
    inp = synth.make_inputs(w)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp)
    layer = pu.make_layer(w, inp)
    try:
        assert layer.staging() == bc.STAGING_INPUT
        n_in = inp.x.size
        buf = torch.zeros(n_in + 4, dtype=torch.float32, device="cuda")
        x = buf[1:1 + n_in].view(inp.x.shape)
        x.copy_(torch.from_numpy(inp.x))
        assert x.data_ptr() % 16 == 4
        y = layer(x)
        layer.sync_status()
        pu.assert_outputs_close(w, inp, y.reshape(-1, w.out_channels).cpu().numpy(), S_ref, beta_ref, y_ref)
        y = layer(torch.from_numpy(inp.x).cuda())
        layer.sync_status()
        pu.assert_outputs_close(w, inp, y.reshape(-1, w.out_channels).cpu().numpy(), S_ref, beta_ref, y_ref)
    finally:
        layer.close()


def test_input_buffers_rotate(cuda_device):
    """Forwards over several input buffers in turn (more than the handle keeps maps of), then
    back to the first: each output follows its own input."""
    import torch

    w = CASES[1]
    outs = []
    refs = []
    base = synth.make_inputs(w)
    layer = pu.make_layer(w, base)
    try:
        xs = []
        for j in range(6):
            x = np.random.default_rng(900 + j).standard_normal(base.x.shape).astype(np.float32)
            xs.append(torch.from_numpy(x).cuda())
            refs.append(x)
        for j in list(range(6)) + [0, 3]:
            outs.append(layer(xs[j]).reshape(-1, w.out_channels).cpu().numpy())
        layer.sync_status()
    finally:
        layer.close()
    for j, y in zip(list(range(6)) + [0, 3], outs):
        inp = synth.Inputs(refs[j], base.wbits, base.scale, base.bias, base.in_scale, base.in_bias)
        S_ref, beta_ref, y_ref = pu.run_oracle(w, inp)
        pu.assert_outputs_close(w, inp, y, S_ref, beta_ref, y_ref)


# more tiles than SMs: the CTAs take equal contiguous shares of all tiles' k-blocks, and a tile
# cut between two CTAs is finished by the first with the second's fp32 partial sums -- another
# order of the same fp32 additions, so these are held to the oracle's tolerance only
SHARE_CASES = [
    synth.small_case(batch=8, h=64, w=64, ni=64, no=64, k=3, op=synth.BINARY_WEIGHTS, relu=True, in_terms=True,
                     seed=720),
    synth.small_case(batch=8, h=56, w=56, ni=200, no=40, k=3, op=synth.BINARY_WEIGHTS, in_terms=False, seed=721),
]


@pytest.mark.parametrize("w", SHARE_CASES, ids=lambda w: w.name)
def test_input_staging_equal_shares(w, cuda_device):
    """Every output against the oracle, over three forwards of one layer (the exchange flags must
    be back at zero after each launch)."""
    import torch

    inp = synth.make_inputs(w)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp)
    layer = pu.make_layer(w, inp)
    try:
        assert layer.staging() == bc.STAGING_INPUT
        x = torch.from_numpy(inp.x).cuda()
        for _ in range(3):
            y = layer(x)
            layer.sync_status()
            pu.assert_outputs_close(w, inp, y.reshape(-1, w.out_channels).cpu().numpy(), S_ref, beta_ref, y_ref)
    finally:
        layer.close()


def test_input_staging_host_buffers(cuda_device):
    """The host-buffer entry point (copies in, forward, copies out) on the fp32-input kernel: the
    same output as the device forward, bit for bit."""
    w = CASES[2]
    inp = synth.make_inputs(w)
    y_dev = pu.run_device(w, inp)
    layer = pu.make_layer(w, inp)
    try:
        assert layer.staging() == bc.STAGING_INPUT
        y_host = layer.forward_host(inp.x)
    finally:
        layer.close()
    np.testing.assert_array_equal(y_host.reshape(y_dev.shape), y_dev)
