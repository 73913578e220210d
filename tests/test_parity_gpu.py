"""The CUDA library against the oracle, element by element (runs on the B200 machine).

Two kinds of cases:
  - sizes the oracle finishes in seconds that still span several 128 x 128 tiles and a
    ragged tail: every output compared;
  - the five workloads at full size, in the launch configuration the bench times: sampled
    outputs (corners, edges, the last tile's tail, random rows) compared with the oracle,
    plus invariants on every output.
Integer sums (XNOR/AND) are compared bit for bit through the sums configuration (scale 1,
bias 0, no beta, identity); float outputs within the tolerance in parity_util.
"""
import numpy as np
import pytest

from binarized_convolution_b200 import synth
import parity_util as pu

pytestmark = pytest.mark.gpu

MEDIUM = [
    synth.small_case(batch=2, h=19, w=17, ni=70, no=150, k=3, op=synth.XNOR, use_beta=True, relu=True,
                     in_terms=True, seed=101),
    synth.small_case(batch=2, h=19, w=17, ni=70, no=150, k=3, op=synth.AND, use_beta=True, relu=False,
                     in_terms=True, seed=102),
    synth.small_case(batch=2, h=19, w=17, ni=70, no=150, k=3, op=synth.BINARY_WEIGHTS, use_beta=True, relu=True,
                     in_terms=True, seed=103),
    synth.small_case(batch=3, h=14, w=15, ni=256, no=132, k=3, op=synth.XNOR, use_beta=False, relu=False,
                     in_terms=False, seed=104),
    synth.small_case(batch=1, h=23, w=29, ni=64, no=64, k=5, stride=2, op=synth.XNOR, use_beta=True, relu=True,
                     in_terms=True, seed=105),
    synth.small_case(batch=2, h=16, w=16, ni=128, no=256, k=3, stride=2, op=synth.BINARY_WEIGHTS, use_beta=False,
                     relu=True, in_terms=False, seed=106),
    synth.small_case(batch=2, h=12, w=12, ni=512, no=40, k=3, op=synth.AND, use_beta=False, relu=False,
                     in_terms=False, p=0.3, seed=107),
    synth.small_case(batch=37, h=3, w=3, ni=100, no=300, kind="fc", op=synth.XNOR, use_beta=True, relu=False,
                     in_terms=True, seed=108),
    synth.small_case(batch=130, h=2, w=3, ni=64, no=129, kind="fc", op=synth.AND, use_beta=True, relu=True,
                     in_terms=False, seed=109),
    synth.small_case(batch=20, h=4, w=4, ni=33, no=70, kind="fc", op=synth.BINARY_WEIGHTS, use_beta=True,
                     relu=False, in_terms=True, seed=110),
    synth.small_case(batch=300, h=2, w=3, ni=96, no=200, kind="fc", op=synth.XNOR, use_beta=True, relu=True,
                     in_terms=True, seed=111),
]


@pytest.mark.parametrize("algo", pu.FAMILIES)
@pytest.mark.parametrize("w", MEDIUM, ids=lambda w: w.name)
def test_medium_all_outputs(w, algo, cuda_device):
    a = pu.algo_for(w, algo)
    inp = synth.make_inputs(w)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp)
    y = pu.run_device(w, inp, algo=a)
    pu.assert_outputs_close(w, inp, y, S_ref, beta_ref, y_ref)
    S_dev = pu.run_device(w, inp, sums=True, algo=a)
    S_sum, _, _ = pu.run_oracle(w, inp, sums=True)
    if w.op == synth.BINARY_WEIGHTS:
        pu.assert_outputs_close(w, synth.Inputs(inp.x, inp.wbits, np.ones_like(inp.scale),
                                                np.zeros_like(inp.bias), inp.in_scale, inp.in_bias),
                                S_dev, S_sum, np.ones(len(S_sum)), S_sum)
    else:
        pu.assert_sums_exact(S_dev, S_sum)


@pytest.mark.parametrize("algo", pu.FAMILIES)
@pytest.mark.parametrize("idx", range(5), ids=lambda i: synth.WORKLOAD_ORDER[i])
def test_workload_full_size(idx, algo, cuda_device):
    w = synth.workload(idx)
    a = pu.algo_for(w, algo)
    inp = synth.make_inputs(w)
    rows = pu.sample_rows(w, seed=idx)
    y = pu.run_device(w, inp, algo=a)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp, rows=rows)
    pu.assert_outputs_close(w, inp, y[rows], S_ref, beta_ref, y_ref, rows=rows)

    S_dev = pu.run_device(w, inp, sums=True, algo=a)
    S_sum, _, _ = pu.run_oracle(w, inp, rows=rows, sums=True)
    if w.op == synth.BINARY_WEIGHTS:
        ones = synth.Inputs(inp.x, inp.wbits, np.ones_like(inp.scale), np.zeros_like(inp.bias), inp.in_scale,
                            inp.in_bias)
        pu.assert_outputs_close(w, ones, S_dev[rows], S_sum, np.ones(len(rows)), S_sum, rows=rows)
        return
    pu.assert_sums_exact(S_dev[rows], S_sum)
    # every output: range and parity of the integer sums
    assert np.all(S_dev == np.round(S_dev))
    if w.kind == "fc":
        nbits = np.full((w.batch, 1), w.in_h * w.in_w * w.in_channels, np.float64)
    else:
        import oracle_pins

        valid = oracle_pins._valid_taps(w.in_h, w.in_w, w.kernel_h, w.kernel_w, w.stride_y, w.stride_x)
        nbits = np.tile(valid.reshape(-1), w.batch)[:, None] * w.in_channels
    if w.op == synth.XNOR:
        assert np.all(np.abs(S_dev) <= nbits)
        assert np.all((S_dev - nbits) % 2 == 0)
    else:
        assert np.all(S_dev >= 0) and np.all(S_dev <= nbits)


LARGE = [
    # wide reductions: 4096 input channels x 9 taps = 36864 terms per output (|S| < 2^24,
    # so the fp32 reduce-add and epilogue stay exact for the integer part)
    synth.small_case(batch=2, h=9, w=10, ni=4096, no=64, k=3, op=synth.XNOR, use_beta=True, relu=True,
                     in_terms=True, seed=31),
    # many output channels: 1024 -> four 256-channel tiles per pixel
    synth.small_case(batch=1, h=12, w=12, ni=128, no=1024, k=3, op=synth.AND, use_beta=True, seed=32),
    # a large window: 11 x 11 taps on a 20 x 20 image
    synth.small_case(batch=2, h=20, w=20, ni=96, no=32, k=11, op=synth.XNOR, use_beta=True, seed=33),
    # a long FC reduction: 14 x 14 x 1024 = 200704 terms per output, split over many SMs
    synth.small_case(batch=160, h=14, w=14, ni=1024, no=64, kind="fc", op=synth.XNOR, use_beta=True, seed=34),
    # binaryWeights with a wide reduction (fp32 sums of 9 x 2048 terms)
    synth.small_case(batch=1, h=8, w=8, ni=2048, no=32, k=3, op=synth.BINARY_WEIGHTS, use_beta=True, in_terms=True,
                     seed=35),
]


@pytest.mark.parametrize("algo", pu.FAMILIES)
@pytest.mark.parametrize("w", LARGE, ids=lambda w: w.name)
def test_large_reductions_and_tiles(w, algo, cuda_device):
    """Sizes at the large end of what the kernels plan for, on sampled outputs."""
    a = pu.algo_for(w, algo)
    inp = synth.make_inputs(w)
    rows = pu.sample_rows(w, seed=w.seed, ops_budget=2e8)
    y = pu.run_device(w, inp, algo=a)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp, rows=rows)
    pu.assert_outputs_close(w, inp, y[rows], S_ref, beta_ref, y_ref, rows=rows)
    if w.op != synth.BINARY_WEIGHTS:
        S_dev = pu.run_device(w, inp, sums=True, algo=a)
        S_sum, _, _ = pu.run_oracle(w, inp, rows=rows, sums=True)
        pu.assert_sums_exact(S_dev[rows], S_sum)
