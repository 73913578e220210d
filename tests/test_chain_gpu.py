"""Chained binary layers on the B200 against the oracle: a layer's output emitted in the
bit-packed form the next binary layer reads (sign bits of x~ = next_scale * y + next_bias,
and A = mean |x~|), a layer reading that form in place of fp32, and two layers in a chain.

Which bits are fixed: the device computes y in fp32 and decides the sign of
fmaf(y, next_scale, next_bias) in fp32; the oracle forms y in double, stores it as an fp32
image and decides on x~ of that.  Where |x~| is within the output tolerance of y (scaled by
|next_scale|) of zero, both decisions are correct readings and either bit is accepted; every
other bit must be equal.  A must agree within the same propagated tolerance."""
from dataclasses import replace

import numpy as np
import pytest

import oracle
import parity_util as pu
from binarized_convolution_b200 import synth
import binarized_convolution_b200 as bc

pytestmark = pytest.mark.gpu


def _unpack(words, c):
    """uint32 words [..., nw] (any 32-bit dtype) -> uint8 bits [..., c], LSB first."""
    w = np.ascontiguousarray(words).view(np.uint32)
    b = np.unpackbits(w.view(np.uint8), axis=-1, bitorder="little")
    return b[..., :c]


def _pack(bits):
    """uint8 bits [..., c] -> uint32 words [..., ceil(c/32)], LSB first (test-side packer)."""
    c = bits.shape[-1]
    nw = (c + 31) // 32
    padded = np.zeros(bits.shape[:-1] + (nw * 32,), np.uint8)
    padded[..., :c] = bits
    return np.packbits(padded, axis=-1, bitorder="little").view(np.uint32)


def _expected_view(w, inp, rows, ns, nb):
    """The oracle's bits and A of the layer output as the next layer reads it, the margin
    under which a bit is not fixed, and the tolerance of A (per row)."""
    S, beta, y = pu.run_oracle(w, inp, rows=rows)
    bits, A, xt = oracle.binarize(y.astype(np.float32), in_scale=ns, in_bias=nb)
    D = pu.error_scale(w, inp, S, beta, rows)
    dy = pu.REL_TOL * np.maximum(np.abs(y), D)  # the tolerance of each fp32 output
    if w.relu:  # a pre-activation clearly below zero is exactly 0 on both sides
        _, _, pre = pu.run_oracle(replace(w, relu=False), inp, rows=rows)
        dy = np.where(pre < -dy, 0.0, dy)
    slack = np.abs(ns.astype(np.float64))[None, :] * dy + 1e-6 * np.abs(nb.astype(np.float64))[None, :]
    fixed = np.abs(xt) > 2.0 * slack + 1e-30
    a_tol = 2.0 * slack.mean(axis=1) + 1e-5 * A
    return bits, A, fixed, a_tol


def _check_bits_out(w, inp, ns, nb, algo, rows=None):
    import torch

    layer = pu.make_layer(w, inp)
    try:
        layer.set_algo(algo)
        layer.set_output_terms(ns, nb)
        x = torch.from_numpy(inp.x).cuda()
        bits, a = layer.forward_to_bits(x)
        layer.sync_status()
        bits = bits.reshape(-1, bits.shape[-1]).cpu().numpy()
        a = a.reshape(-1).cpu().numpy().astype(np.float64)
    finally:
        layer.close()
    nw = (w.out_channels + 31) // 32
    assert bits.shape[1] == nw
    if w.out_channels % 32:  # bits past the last channel are written as 0
        tail = bits[:, -1].view(np.uint32) >> np.uint32(w.out_channels % 32)
        assert not tail.any()
    if rows is not None:
        bits, a = bits[rows], a[rows]
    got = _unpack(bits, w.out_channels)
    ref, A_ref, fixed, a_tol = _expected_view(w, inp, rows, ns, nb)
    bad = np.nonzero(fixed & (got != ref))
    assert bad[0].size == 0, f"{bad[0].size} fixed bits differ, first at {(bad[0][0], bad[1][0])}"
    assert fixed.mean() > 0.99
    assert 0.05 < ref.mean() < 0.95
    err = np.abs(a - A_ref)
    assert np.all(err <= a_tol), f"A off by {err.max():.3e} (tolerance {a_tol[np.argmax(err - a_tol)]:.3e})"
    return a


CASES = [
    # (workload, next-terms seed): channel counts around words and tiles, both kernel families
    synth.small_case(batch=2, h=9, w=11, ni=70, no=40, k=3, op=synth.XNOR, use_beta=True, relu=True,
                     in_terms=True, seed=51),
    synth.small_case(batch=1, h=13, w=12, ni=96, no=256, k=3, op=synth.AND, relu=False, seed=52),
    synth.small_case(batch=1, h=12, w=13, ni=64, no=512, k=3, op=synth.XNOR, use_beta=True, seed=53),
    synth.small_case(batch=2, h=7, w=9, ni=33, no=37, k=3, op=synth.XNOR, use_beta=True, relu=True, seed=54),
    synth.small_case(batch=1, h=10, w=10, ni=48, no=100, k=3, stride=2, op=synth.BINARY_WEIGHTS, use_beta=True,
                     relu=True, in_terms=True, seed=55),
    synth.small_case(batch=3, h=11, w=8, ni=130, no=64, k=2, op=synth.AND, use_beta=True, seed=56),
]


@pytest.mark.parametrize("algo", pu.FAMILIES)
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_bits_out(w, algo, cuda_device):
    inp = synth.make_inputs(w)
    ns, nb = synth.next_terms(w.out_channels, w.seed + 100, bias_spread=0.05)
    _check_bits_out(w, inp, ns, nb, pu.algo_for(w, algo))


def test_bits_out_a_is_deterministic(cuda_device):
    """512 output channels span two work items per pixel: A is added in a fixed order."""
    import torch

    w = CASES[2]
    inp = synth.make_inputs(w)
    ns, nb = synth.next_terms(w.out_channels, 7)
    layer = pu.make_layer(w, inp)
    layer.set_output_terms(ns, nb)
    x = torch.from_numpy(inp.x).cuda()
    first = layer.forward_to_bits(x)
    for _ in range(5):
        again = layer.forward_to_bits(x)
        assert torch.equal(first[0], again[0]) and torch.equal(first[1], again[1])
    layer.sync_status()
    layer.close()


def _bits_input(w, inp, rows=None):
    """Bit-packed view of the workload's input (the oracle's bits and A, packed here)."""
    bits, A, _ = oracle.binarize(inp.x, in_scale=inp.in_scale, in_bias=inp.in_bias)
    return _pack(bits), A.astype(np.float32)


@pytest.mark.parametrize("algo", pu.FAMILIES)
@pytest.mark.parametrize("w", [c for c in CASES if c.op != synth.BINARY_WEIGHTS] + [
    synth.small_case(batch=2, h=6, w=7, ni=31, no=8, k=5, op=synth.XNOR, use_beta=True, in_terms=True, seed=57),
    synth.small_case(batch=1, h=9, w=9, ni=200, no=12, k=3, stride=2, op=synth.AND, use_beta=True, seed=58),
], ids=lambda w: w.name)
def test_bits_in(w, algo, cuda_device):
    """A layer reading bit-packed input equals the oracle layer on the fp32 input whose view
    those bits are (the input terms move to the producer of the bits)."""
    import torch

    inp = synth.make_inputs(w)
    words, A = _bits_input(w, inp)
    # tail bits past the channel count are ignored on input: set them to 1
    if w.in_channels % 32:
        words[..., -1] |= np.uint32(0xFFFFFFFF) << np.uint32(w.in_channels % 32)
    bare = replace(inp, in_scale=None, in_bias=None)  # the consumer has no input terms
    xb = torch.from_numpy(words.view(np.int32)).cuda()
    xa = torch.from_numpy(A).cuda()
    a = pu.algo_for(w, algo)
    for sums in (True, False):
        layer = pu.make_layer(w, bare, sums=sums)
        try:
            layer.set_algo(a)
            y = layer.forward_from_bits(xb, xa if (w.use_beta and not sums) else None)
            layer.sync_status()
            y = y.reshape(-1, w.out_channels).cpu().numpy()
        finally:
            layer.close()
        S_ref, beta_ref, y_ref = pu.run_oracle(w, inp, sums=sums)
        if sums:
            pu.assert_sums_exact(y, S_ref)
        else:
            pu.assert_outputs_close(w, inp, y, S_ref, beta_ref, y_ref)


def test_two_layer_chain(cuda_device):
    """Layer 1 (fp32 in, bits out) -> layer 2 (bits in, fp32 out) against the oracle's two
    layers on the fp32 image of layer 1's output."""
    import torch

    w1 = synth.small_case(batch=2, h=10, w=12, ni=64, no=128, k=3, op=synth.XNOR, use_beta=True, relu=True,
                          in_terms=True, seed=61)
    inp1 = synth.make_inputs(w1)
    ns, nb = synth.next_terms(w1.out_channels, 62, bias_spread=0.05)
    w2 = synth.small_case(batch=2, h=10, w=12, ni=128, no=96, k=3, op=synth.AND, use_beta=True, seed=63)
    inp2 = synth.make_inputs(w2)
    # the oracle's chain: layer 1, its output as an fp32 image, layer 2 with the next terms
    _, _, y1 = pu.run_oracle(w1, inp1)
    x2 = y1.astype(np.float32).reshape(w2.batch, w2.in_h, w2.in_w, w2.in_channels)
    _, _, fixed, _ = _expected_view(w1, inp1, None, ns, nb)
    assert fixed.all(), "every bit between the layers must be fixed for an exact comparison of layer 2"
    inp2_ref = replace(inp2, x=x2, in_scale=ns, in_bias=nb)
    S2, beta2, y2_ref = pu.run_oracle(w2, inp2_ref)
    S2_sum, _, _ = pu.run_oracle(w2, inp2_ref, sums=True)

    l1 = pu.make_layer(w1, inp1)
    l2 = pu.make_layer(w2, replace(inp2, in_scale=None, in_bias=None))
    l2s = pu.make_layer(w2, replace(inp2, in_scale=None, in_bias=None), sums=True)
    try:
        l1.set_output_terms(ns, nb)
        bits, a = l1.forward_to_bits(torch.from_numpy(inp1.x).cuda())
        y2 = l2.forward_from_bits(bits, a).reshape(-1, w2.out_channels).cpu().numpy()
        s2 = l2s.forward_from_bits(bits).reshape(-1, w2.out_channels).cpu().numpy()
        for l in (l1, l2, l2s):
            l.sync_status()
    finally:
        for l in (l1, l2, l2s):
            l.close()
    pu.assert_sums_exact(s2, S2_sum)
    pu.assert_outputs_close(w2, inp2_ref, y2, S2, beta2, y2_ref)


@pytest.mark.parametrize("key", ["xnor_beta_n16_56x56_c256_k256_3x3", "and_n32_28x28_c512_k512_3x3"])
def test_bits_out_full_size(key, cuda_device):
    """The default launch configuration at full size, on sampled output pixels."""
    w = synth.workload(key)
    inp = synth.make_inputs(w)
    ns, nb = synth.next_terms(w.out_channels, 71, bias_spread=0.05 if w.relu else 0.5)
    rows = pu.sample_rows(w, ops_budget=1.5e8)
    _check_bits_out(w, inp, ns, nb, bc.ALGO_AUTO, rows)


def test_io_argument_errors(cuda_device):
    import torch

    w = CASES[0]
    inp = synth.make_inputs(w)
    layer = pu.make_layer(w, inp)  # has input terms and beta
    x = torch.from_numpy(inp.x).cuda()
    bshape, ashape = layer.bits_shape()
    bits = torch.zeros(bshape, dtype=torch.int32, device="cuda")
    a = torch.zeros(ashape, device="cuda")
    out = torch.empty(layer.out_dims, device="cuda")
    with pytest.raises(bc.BconvError):  # no next-layer terms yet
        layer.forward_io(x=x, out_bits=bits, out_a=a)
    with pytest.raises(bc.BconvError):  # both input forms
        layer.forward_io(x=x, x_bits=bits, out=out)
    with pytest.raises(bc.BconvError):  # no input
        layer.forward_io(out=out)
    xb = torch.zeros((w.batch, w.in_h, w.in_w, (w.in_channels + 31) // 32), dtype=torch.int32, device="cuda")
    with pytest.raises(bc.BconvError):  # the layer's own input terms cannot act on bits
        layer.forward_io(x_bits=xb, x_a=a, out=out)
    layer.set_output_terms(None, None)
    with pytest.raises(bc.BconvError):  # bits out needs A out
        layer.forward_io(x=x, out_bits=bits)
    layer.close()
    bare = pu.make_layer(w, replace(inp, in_scale=None, in_bias=None))
    with pytest.raises(bc.BconvError):  # beta needs the input's A
        bare.forward_io(x_bits=xb, out=out)
    bare.close()
    bw = synth.small_case(batch=1, h=5, w=5, ni=8, no=4, op=synth.BINARY_WEIGHTS, seed=3)
    lbw = pu.make_layer(bw, synth.make_inputs(bw))
    xb = torch.zeros((1, 5, 5, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(bc.BconvError) as e:  # binaryWeights needs the fp32 input
        lbw.forward_io(x_bits=xb, out=torch.empty(lbw.out_dims, device="cuda"))
    assert e.value.status == 2
    lbw.close()


FC_CASES = [
    synth.small_case(batch=5, h=3, w=5, ni=40, no=64, kind="fc", op=synth.XNOR, use_beta=True, relu=True,
                     in_terms=True, seed=81),
    synth.small_case(batch=130, h=2, w=3, ni=33, no=36, kind="fc", op=synth.AND, use_beta=True, seed=82),
    synth.small_case(batch=4, h=3, w=3, ni=20, no=30, kind="fc", op=synth.XNOR, seed=83),
]


@pytest.mark.parametrize("algo", pu.FAMILIES)
@pytest.mark.parametrize("w", FC_CASES + [synth.small_case(batch=3, h=2, w=2, ni=24, no=40, kind="fc",
                                                           op=synth.BINARY_WEIGHTS, use_beta=True, in_terms=True,
                                                           seed=84)], ids=lambda w: w.name)
def test_fc_bits_out(w, algo, cuda_device):
    inp = synth.make_inputs(w)
    ns, nb = synth.next_terms(w.out_channels, w.seed + 100, bias_spread=0.05)
    _check_bits_out(w, inp, ns, nb, pu.algo_for(w, algo))


@pytest.mark.parametrize("algo", pu.FAMILIES)
@pytest.mark.parametrize("w", FC_CASES, ids=lambda w: w.name)
def test_fc_bits_in(w, algo, cuda_device):
    """The FC reads a convolution's bit-packed output ([N][H][W][words] and A [N][H][W])."""
    import torch

    inp = synth.make_inputs(w)
    words, A = _bits_input(w, inp)
    bare = replace(inp, in_scale=None, in_bias=None)
    xb = torch.from_numpy(words.view(np.int32)).cuda()
    xa = torch.from_numpy(A).cuda()
    a = pu.algo_for(w, algo)
    for sums in (True, False):
        layer = pu.make_layer(w, bare, sums=sums)
        try:
            layer.set_algo(a)
            y = layer.forward_from_bits(xb, xa if (w.use_beta and not sums) else None)
            layer.sync_status()
            y = y.reshape(-1, w.out_channels).cpu().numpy()
        finally:
            layer.close()
        S_ref, beta_ref, y_ref = pu.run_oracle(w, inp, sums=sums)
        if sums:
            pu.assert_sums_exact(y, S_ref)
        else:
            pu.assert_outputs_close(w, inp, y, S_ref, beta_ref, y_ref)
