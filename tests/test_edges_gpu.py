"""Edge cases of the CUDA library against the oracle on tiny inputs (runs on the B200 machine):
channel counts around word boundaries, odd and even kernels, strides, non-square and tiny
images, signed zeros, empty batches, ragged output channels and the FC with a partial last
word."""
import itertools

import numpy as np
import pytest

from binarized_convolution_b200 import synth
import binarized_convolution_b200 as bc
import parity_util as pu

pytestmark = pytest.mark.gpu


def _check(w, inp=None):
    """Both kernel families (the library's choice and the SIMT one) against the oracle."""
    inp = inp if inp is not None else synth.make_inputs(w)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp)
    S_sum, _, _ = pu.run_oracle(w, inp, sums=True)
    for name in pu.FAMILIES:
        a = pu.algo_for(w, name)
        y = pu.run_device(w, inp, algo=a)
        pu.assert_outputs_close(w, inp, y, S_ref, beta_ref, y_ref)
        if w.op != synth.BINARY_WEIGHTS:
            S_dev = pu.run_device(w, inp, sums=True, algo=a)
            pu.assert_sums_exact(S_dev, S_sum)
    bc.bconv_set_cta_mode(bc.CTA_AUTO)
    bc.bconv_set_tc_codes(bc.CODES_AUTO)


SWEEP = []
for i, (ni, k, s, op) in enumerate(itertools.product([1, 31, 32, 33, 100], [1, 2, 3, 5, 7], [1, 2],
                                                     [synth.XNOR, synth.AND, synth.BINARY_WEIGHTS])):
    if (i % 3) != 0 and k not in (2, 3):  # keep the sweep small: every even/3x3 kernel, a third of the rest
        continue
    SWEEP.append(synth.small_case(batch=1 + (i % 2), h=7 + (i % 3), w=9 - (i % 4), ni=ni, no=5 + (i % 7), k=k,
                                  stride=s, op=op, use_beta=bool(i % 2), relu=bool((i // 2) % 2),
                                  in_terms=bool((i // 3) % 2), seed=1000 + i))


@pytest.mark.parametrize("w", SWEEP, ids=lambda w: w.name)
def test_sweep(w, cuda_device):
    _check(w)


@pytest.mark.parametrize("op", [synth.XNOR, synth.AND, synth.BINARY_WEIGHTS])
def test_kernel_larger_than_image(op, cuda_device):
    _check(synth.small_case(batch=2, h=3, w=2, ni=40, no=3, k=7, kw=5, op=op, use_beta=True, in_terms=True, seed=7))


@pytest.mark.parametrize("op", [synth.XNOR, synth.AND])
def test_signed_zeros_binarize_to_plus_one(op, cuda_device):
    w = synth.small_case(batch=1, h=6, w=5, ni=48, no=9, k=3, op=op, seed=8)
    inp = synth.make_inputs(w)
    inp.x[..., :8] = 0.0
    inp.x[..., 8:16] = -0.0
    _check(w, inp)
    # the same layer with in_bias that maps some inputs exactly onto +-0
    w2 = synth.small_case(batch=1, h=6, w=5, ni=48, no=9, k=3, op=op, in_terms=True, seed=9)
    inp2 = synth.make_inputs(w2)
    inp2.in_scale[:] = 1.0
    inp2.in_bias[:4] = 0.5
    inp2.x[..., :4] = -0.5
    _check(w2, inp2)


@pytest.mark.parametrize("op", [synth.XNOR, synth.AND, synth.BINARY_WEIGHTS])
def test_fc_partial_last_word(op, cuda_device):
    _check(synth.small_case(batch=5, h=3, w=5, ni=7, no=11, kind="fc", op=op, use_beta=True, in_terms=True, seed=10))
    _check(synth.small_case(batch=3, h=1, w=1, ni=1, no=1, kind="fc", op=op, use_beta=True, seed=11))


@pytest.mark.parametrize("op", [synth.XNOR, synth.AND, synth.BINARY_WEIGHTS])
def test_ragged_channels_and_tiles(op, cuda_device):
    # No = 1 and No = 129 (one past a 128-channel tile), M = 129 (one past a 128-pixel tile)
    _check(synth.small_case(batch=1, h=3, w=43, ni=65, no=1, k=3, op=op, use_beta=True, seed=12))
    _check(synth.small_case(batch=1, h=3, w=43, ni=65, no=129, k=3, op=op, relu=True, seed=13))


def test_empty_batch(cuda_device):
    import torch

    for op in (synth.XNOR, synth.BINARY_WEIGHTS):
        layer = bc.BinaryConv2d(0, 5, 5, 8, 4, 3, 1, wbits=np.ones((4, 3, 3, 8), np.uint8), op=op, use_beta=True)
        y = layer(torch.empty((0, 5, 5, 8), device="cuda"))
        layer.sync_status()
        assert tuple(y.shape) == (0, 5, 5, 4)
        layer.close()


def test_forward_host_matches_device(cuda_device):
    w = synth.small_case(batch=2, h=9, w=10, ni=96, no=40, k=3, op=synth.XNOR, use_beta=True, relu=True,
                         in_terms=True, seed=14)
    inp = synth.make_inputs(w)
    y_dev = pu.run_device(w, inp)
    layer = pu.make_layer(w, inp)
    y_host = layer.forward_host(inp.x)
    layer.close()
    np.testing.assert_array_equal(y_host.reshape(y_dev.shape), y_dev)


def test_properties_and_algo(cuda_device):
    w = synth.small_case(batch=1, h=5, w=5, ni=70, no=6, k=3, op=synth.XNOR, seed=15)
    inp = synth.make_inputs(w)
    layer = pu.make_layer(w, inp)
    assert layer.input_feature_channels == 70 and layer.output_feature_channels == 6
    layer.set_algo(bc.ALGO_POPC)
    with pytest.raises(bc.BconvError):
        layer.set_algo(bc.ALGO_SIMT_F32)
    assert layer.launches_per_forward() == 2
    layer.close()


def test_profile_window_and_stride(cuda_device):
    """bconv_profile_begin(n) times the contraction of the next n forwards; with
    bconv_profile_stride(k) only every k-th forward of the window is timed."""
    import torch

    w = synth.small_case(batch=1, h=8, w=8, ni=64, no=32, k=3, op=synth.XNOR, seed=16)
    inp = synth.make_inputs(w)
    layer = pu.make_layer(w, inp)
    x = torch.from_numpy(inp.x).cuda()
    bc.bconv_profile_begin(layer.handle, 100)
    for _ in range(5):
        layer(x)
    ms, n = bc.bconv_profile_end(layer.handle)
    assert n == 5 and ms > 0
    bc.bconv_profile_begin(layer.handle, 100)
    bc.bconv_profile_stride(layer.handle, 3)
    for _ in range(7):
        layer(x)
    ms, n = bc.bconv_profile_end(layer.handle)
    assert n == 3 and ms > 0  # forwards 0, 3 and 6
    with pytest.raises(bc.BconvError):
        bc.bconv_profile_stride(layer.handle, 0)
    layer.sync_status()
    layer.close()


@pytest.mark.parametrize("op,ni", [(synth.XNOR, 32), (synth.AND, 160), (synth.BINARY_WEIGHTS, 32)])
def test_reduction_split_between_sm_pairs(op, ni, cuda_device):
    """162 tiles of 128 pixels on the SM pairs (more pair items than pairs, a ragged last wave):
    the reduction is shared out evenly and items cut between two pairs are summed from both
    halves.  Every output is checked, and two runs must agree bit for bit."""
    import torch

    w = synth.small_case(batch=4, h=70, w=70, ni=ni, no=32, k=3, op=op, use_beta=True, relu=True, in_terms=True,
                         seed=17)
    inp = synth.make_inputs(w)
    _check(w, inp)
    layer = pu.make_layer(w, inp)
    x = torch.from_numpy(inp.x).cuda()
    y1 = layer(x)
    y2 = layer(x)
    layer.sync_status()
    layer.close()
    assert torch.equal(y1, y2)


def test_fc_split_reduction_repeated(cuda_device):
    """The FC's split reduction adds partial sums into a workspace that its last kernel zeroes
    as it reads it: consecutive forwards on different inputs must each match the oracle."""
    import torch

    w = synth.small_case(batch=130, h=7, w=7, ni=256, no=64, kind="fc", op=synth.XNOR, use_beta=True, relu=True,
                         in_terms=True, seed=18)
    inp = synth.make_inputs(w)
    layer = pu.make_layer(w, inp)
    sums = pu.make_layer(w, inp, sums=True)
    try:
        for seed in (18, 19, 20):
            x = synth.make_batch(w, seed)
            cur = synth.Inputs(x, inp.wbits, inp.scale, inp.bias, inp.in_scale, inp.in_bias)
            xt = torch.from_numpy(x).cuda()
            y = layer(xt).reshape(-1, w.out_channels).cpu().numpy()
            S = sums(xt).reshape(-1, w.out_channels).cpu().numpy()
            S_ref, beta_ref, y_ref = pu.run_oracle(w, cur)
            S_sum, _, _ = pu.run_oracle(w, cur, sums=True)
            pu.assert_sums_exact(S, S_sum)
            pu.assert_outputs_close(w, cur, y, S_ref, beta_ref, y_ref)
        layer.sync_status()
        sums.sync_status()
    finally:
        layer.close()
        sums.close()


def test_fc_int16_partials_at_their_limit(cuda_device):
    """The e2m1 FC sends each split's partial sums to the row's owner as int16, at most 127
    k-blocks of 256 codes a split (|partial| <= 32512).  With every product +1 (positive
    input, all weight bits set) the sums equal the code count: 508 k-blocks run on e2m1 codes
    (4 splits of 127, or 8 of 64 where clusters of 8 fit), 1016 on e2m1 codes with 8 splits of
    127 where those fit and on int8 codes otherwise, 1017 always on int8 codes."""
    for kb, want in ((508, bc.CODES_FP4), (1016, None), (1017, bc.CODES_INT8)):
        w = synth.small_case(batch=1, h=1, w=1, ni=kb * 256, no=32, kind="fc", op=synth.XNOR, p=1.0, seed=41)
        base = synth.make_inputs(w)
        inp = synth.Inputs(np.abs(base.x) + 0.01, base.wbits, base.scale, base.bias, None, None)
        layer = pu.make_layer(w, inp, sums=True)
        try:
            assert layer.tc_codes() in ((want,) if want is not None else (bc.CODES_FP4, bc.CODES_INT8))
        finally:
            layer.close()
        S_dev = pu.run_device(w, inp, sums=True)
        S_sum, _, _ = pu.run_oracle(w, inp, sums=True)
        assert np.all(S_sum == kb * 256)
        pu.assert_sums_exact(S_dev, S_sum)


def test_bounded_wait_gives_up_and_device_stays_usable(cuda_device):
    """The kernels' mbarrier waits are bounded: a wait on a barrier that nothing completes ends
    with a timeout status (not a hang), and the device keeps working afterwards."""
    assert bc.bconv_check_wait_timeout(20.0) == 5  # BCONV_ERR_TIMEOUT
    w = synth.small_case(batch=1, h=6, w=6, ni=64, no=32, k=3, op=synth.XNOR, seed=19)
    _check(w)


@pytest.mark.parametrize("family", pu.FAMILIES)
@pytest.mark.parametrize("op", [synth.XNOR, synth.BINARY_WEIGHTS])
def test_forward_host_in_chunks_matches_device(op, family, cuda_device):
    """A batch large enough for the host-buffer forward to run as image chunks (copies and
    compute overlapped on three streams; four two-image chunks that share the first chunk's
    weights) gives the device forward's result bit for bit, on every kernel family."""
    import torch

    w = synth.small_case(batch=8, h=64, w=64, ni=64, no=64, k=3, op=op, use_beta=True, relu=True, in_terms=True,
                         seed=21)
    inp = synth.make_inputs(w)
    a = pu.algo_for(w, family)
    y_dev = pu.run_device(w, inp, algo=a)
    layer = pu.make_layer(w, inp)
    try:
        layer.set_algo(a)
        hin = torch.from_numpy(inp.x).pin_memory()
        hout = torch.empty(layer.out_dims, dtype=torch.float32).pin_memory()
        for _ in range(2):  # the first call creates the chunk layers
            bc.bconv_forward_host(layer.handle, hin.data_ptr(), hout.data_ptr(), 0)
            np.testing.assert_array_equal(hout.numpy().reshape(y_dev.shape), y_dev)
        layer.sync_status()
    finally:
        layer.close()


def test_fc_forward_host_in_chunks_matches_device(cuda_device):
    """The FC's host-buffer forward in image chunks (each chunk a split-reduction FC of its
    own, all reading the first chunk's weights) against the device forward."""
    import torch

    # 128 images of 7 x 7 x 512: four chunks of 32 images
    w = synth.small_case(batch=128, h=7, w=7, ni=512, no=512, kind="fc", op=synth.XNOR, use_beta=True, relu=True,
                         in_terms=True, seed=26)
    inp = synth.make_inputs(w)
    y_dev = pu.run_device(w, inp)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp)
    pu.assert_outputs_close(w, inp, y_dev, S_ref, beta_ref, y_ref)
    layer = pu.make_layer(w, inp)
    try:
        hin = torch.from_numpy(inp.x).pin_memory()
        hout = torch.empty(layer.out_dims, dtype=torch.float32).pin_memory()
        for _ in range(2):  # exact integer sums and the same beta: equal bit for bit
            bc.bfc_forward_host(layer.handle, hin.data_ptr(), hout.data_ptr(), 0)
            np.testing.assert_array_equal(hout.numpy().reshape(y_dev.shape), y_dev)
        layer.sync_status()
    finally:
        layer.close()


def _spread(w, mode=None, codes=None):
    """(spread, operand codes) a layer of this shape is created with."""
    inp = synth.make_inputs(w)
    if mode is not None:
        bc.bconv_set_cta_mode(mode)
    if codes is not None:
        bc.bconv_set_tc_codes(codes)
    try:
        layer = pu.make_layer(w, inp)
    finally:
        bc.bconv_set_cta_mode(bc.CTA_AUTO)
        bc.bconv_set_tc_codes(bc.CODES_AUTO)
    try:
        return layer.cta_mode(), layer.tc_codes()
    finally:
        layer.close()


def test_spread_choice(cuda_device):
    """AUTO: XNOR/AND on e2m1 codes -- stride-1 layers rows-staged, on SM pairs above 128 output
    channels, else one SM per tile; with int8 codes one SM per tile where the pair plan is not
    clearly shorter (equal waves), SM pairs where their balanced split evens out a ragged last
    wave by more and for the FC with batch > 128; binaryWeights on bf16 parts (its 24 against 27
    stages on pairs is not enough for them); forced modes are kept where the layer allows them."""
    S, P, I8, F4, BF = bc.CTA_SINGLE, bc.CTA_PAIR, bc.CODES_INT8, bc.CODES_FP4, bc.CODES_BF16X3
    c2 = synth.workload("xnor_beta_n16_56x56_c256_k256_3x3")
    assert _spread(c2) == (P, F4)  # rows-staged on SM pairs, 256-channel MMAs
    assert _spread(c2, mode=S) == (S, F4)
    assert _spread(c2, codes=I8) == (S, I8)
    assert _spread(c2, mode=P) == (P, I8)  # forced pairs take the int8 per-tap pair kernel
    assert _spread(synth.workload("and_n32_28x28_c512_k512_3x3")) == (P, F4)
    assert _spread(synth.workload("binw_n8_112x112_c128_k128_3x3_s2")) == (S, BF)
    fc5 = synth.workload("fc_xnor_beta_n256_7x7x512_k4096")
    assert _spread(fc5) == (S, F4)  # the e2m1 FC kernel (one SM per item, clusters per tile)
    assert _spread(fc5, codes=I8) == (P, I8)
    ragged = synth.small_case(batch=4, h=70, w=70, ni=32, no=32, k=3, op=synth.XNOR, seed=27)
    assert _spread(ragged, codes=I8) == (P, I8)  # 162 tiles: 18 stages on single SMs, 10 on pairs
    assert _spread(ragged) == (S, F4)
    small = synth.small_case(batch=1, h=8, w=8, ni=64, no=32, k=3, op=synth.XNOR, seed=22)
    assert _spread(small, codes=I8) == (S, I8)
    assert _spread(small, mode=P) == (P, I8)
    fc = synth.small_case(batch=200, h=2, w=2, ni=64, no=64, kind="fc", op=synth.AND, seed=23)
    assert _spread(fc, codes=I8) == (P, I8)
    assert _spread(fc, mode=S, codes=I8) == (S, I8)
    fc_small = synth.small_case(batch=100, h=2, w=2, ni=64, no=64, kind="fc", op=synth.AND, seed=24)
    assert _spread(fc_small, mode=P) == (S, I8)  # the FC's pair tile needs batch > 128
    odd = synth.small_case(batch=1, h=5, w=5, ni=64, no=6, k=3, op=synth.XNOR, seed=25)
    assert _spread(odd) == (0, 0)  # out_channels % 4 != 0: no tensor-core path


def test_bit_output_replans_wide_e2m1_layer_on_int8(cuda_device):
    """A convolution on e2m1 codes with more than one 128-channel tile takes int8 codes (one
    256-channel tile) once it is asked for a bit-packed output, and still matches the oracle."""
    w = synth.small_case(batch=1, h=9, w=10, ni=96, no=256, k=3, op=synth.XNOR, use_beta=True, relu=True,
                         in_terms=True, seed=28)
    inp = synth.make_inputs(w)
    layer = pu.make_layer(w, inp)
    try:
        assert layer.tc_codes() == bc.CODES_FP4
        ns, nb = synth.next_terms(w.out_channels, 5)
        layer.set_output_terms(ns, nb)
        assert layer.tc_codes() == bc.CODES_INT8 and layer.cta_mode() == bc.CTA_SINGLE
    finally:
        layer.close()
    narrow = synth.small_case(batch=1, h=9, w=10, ni=96, no=64, k=3, op=synth.XNOR, seed=29)
    layer = pu.make_layer(narrow, synth.make_inputs(narrow))
    try:
        layer.set_output_terms(*synth.next_terms(64, 6))
        assert layer.tc_codes() == bc.CODES_FP4  # one tile: nothing to add across items
    finally:
        layer.close()


E2M1_CASES = [
    # channel counts around the e2m1 layout (two codes per byte, 256-channel rows) and the
    # 128-channel e2m1 tiles: a full row, two rows, the byte-wise path, mostly padding
    synth.small_case(batch=2, h=20, w=20, ni=256, no=96, k=3, op=synth.XNOR, use_beta=True, relu=True, in_terms=True,
                     seed=61),
    synth.small_case(batch=1, h=15, w=15, ni=512, no=128, k=1, op=synth.AND, use_beta=True, seed=62),
    synth.small_case(batch=1, h=7, w=9, ni=1000, no=40, k=3, op=synth.XNOR, in_terms=True, seed=63),
    synth.small_case(batch=2, h=11, w=13, ni=20, no=200, k=5, stride=2, op=synth.AND, use_beta=True, relu=True,
                     in_terms=True, seed=64),
]


@pytest.mark.parametrize("w", E2M1_CASES, ids=lambda w: w.name)
def test_e2m1_code_layouts(w, cuda_device):
    """Layers whose codes take the e2m1 layout's different paths, against the oracle on every
    family (the library's choice is e2m1 here)."""
    layer = pu.make_layer(w, synth.make_inputs(w))
    try:
        assert layer.tc_codes() == bc.CODES_FP4
    finally:
        layer.close()
    _check(w)


@pytest.mark.parametrize("op", [synth.AND, synth.XNOR])
def test_window_sums_past_2p24_stay_exact(op, cuda_device):
    """A window sum of more than 2^24 unit terms (1 x 17 kernel over 2^20 channels, every input
    bit 1, 99 % of the weight bits 1): fp32 accumulation would round such sums, so the library
    keeps int32 sums even when e2m1 codes are asked for.  With scale 1 and no bias the fp32
    output must be the exact integer sum rounded once to fp32, on every kernel family."""
    import oracle
    import torch

    ni, no, width, k = 1 << 20, 4, 17, 17
    rng = np.random.default_rng(77)
    x = (np.abs(rng.standard_normal((1, 1, width, ni), dtype=np.float32)) + 0.25).astype(np.float32)
    wbits = np.ones((no, 1, k, ni), np.uint8)
    flat = wbits.reshape(-1)
    flat[rng.integers(0, flat.size, flat.size // 100)] = 0
    otype = {synth.AND: oracle.ORACLE_AND, synth.XNOR: oracle.ORACLE_XNOR}[op]
    S, _, _ = oracle.conv(x, wbits, type=otype, scale_value=1.0)
    assert np.abs(S).max() > 2 ** 24
    if op == synth.AND:  # XNOR sums have the parity of the window size (even here); AND sums need not
        assert np.any(S % 2 == 1)
    want = S.astype(np.float32)
    for name in ("auto", "alt", "single", "pair"):
        algo = pu.algo_for(synth.small_case(op=op), name)
        if name == "auto":
            bc.bconv_set_tc_codes(bc.CODES_FP4)  # asked for e2m1: the sums must still stay int32
        layer = bc.BinaryConv2d(1, 1, width, ni, no, (1, k), (1, 1), wbits=wbits, op=op, scale=None,
                                scale_value=1.0)
        try:
            layer.set_algo(algo)
            if layer.effective_algo() == bc.ALGO_TCGEN05:
                assert layer.tc_codes() == bc.CODES_INT8
            y = layer(torch.from_numpy(x).cuda())
            layer.sync_status()
            y = y.reshape(-1, no).cpu().numpy()
        finally:
            layer.close()
        assert np.array_equal(y, want), f"{name}: {np.abs(y.astype(np.float64) - S).max()}"
    bc.bconv_set_cta_mode(bc.CTA_AUTO)
    bc.bconv_set_tc_codes(bc.CODES_AUTO)


def test_staging_choice(cuda_device):
    """The rows-staged kernel serves e2m1 stride-1 convolutions whose padded rows fit a tile; strided
    layers, wide images, a forced per-tap setting and a bit-packed output use the per-tap kernel."""
    def layer(h, w, stride=1, no=64):
        c = synth.small_case(batch=2, h=h, w=w, ni=64, no=no, k=3, stride=stride, op=synth.XNOR, seed=7)
        inp = synth.make_inputs(c)
        return bc.BinaryConv2d(c.batch, c.in_h, c.in_w, c.in_channels, c.out_channels, 3, stride, wbits=inp.wbits)

    with layer(12, 56) as l:
        assert l.staging() == bc.STAGING_ROWS and l.tc_codes() == bc.CODES_FP4
    with layer(12, 56, stride=2) as l:
        assert l.staging() == bc.STAGING_PER_TAP
    with layer(4, 500) as l:  # a window reaching 2 x 502 + 2 slots past the tile is too long
        assert l.staging() == bc.STAGING_PER_TAP
    with layer(4, 200) as l:  # wide rows are fine: tiles run across them
        assert l.staging() == bc.STAGING_ROWS
    with layer(12, 56) as l:
        l.set_output_terms(None, None)
        assert l.staging() == bc.STAGING_PER_TAP
    bc.bconv_set_staging(bc.STAGING_PER_TAP)
    with layer(12, 56) as l:
        assert l.staging() == bc.STAGING_PER_TAP
    bc.bconv_set_staging(bc.STAGING_AUTO)


@pytest.mark.parametrize("kind", ["conv", "fc"])
def test_output_not_16_byte_aligned(kind, cuda_device):
    """An output buffer 4 bytes past a 16-byte boundary: the tensor-core kernels write 16-byte
    pieces, so such a forward runs on the SIMT family and must still match the oracle."""
    import torch

    w = synth.small_case(batch=3, h=6, w=7, ni=40, no=36, k=3, kind=kind, op=synth.XNOR, use_beta=True, relu=True,
                         in_terms=True, seed=61)
    inp = synth.make_inputs(w)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp)
    layer = pu.make_layer(w, inp)
    try:
        n_out = int(np.prod(layer.out_dims))
        buf = torch.zeros(n_out + 4, dtype=torch.float32, device="cuda")
        out = buf[1:1 + n_out].view(layer.out_dims)
        assert out.data_ptr() % 16 == 4
        layer.forward_into(torch.from_numpy(inp.x).cuda(), out)
        layer.sync_status()
        y = out.reshape(-1, w.out_channels).cpu().numpy()
    finally:
        layer.close()
    pu.assert_outputs_close(w, inp, y, S_ref, beta_ref, y_ref)
