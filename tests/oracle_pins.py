"""Checks that pin the oracle to facts other than itself.

Each ``pin_*`` function takes an object with the oracle's ``conv`` and ``fc`` entry points
and raises AssertionError when the oracle disagrees with

  - values printed on the pages (the fixtures under ``tests/golden/``),
  - a library routine that computes the same thing in a special case
    (float64 ``torch.nn.functional.conv2d``, float64 matrix-vector products),
  - brute force on tiny inputs (zero-padded windows, numpy),
  - closed forms (beta on a constant-magnitude image) and invariants (parity, ranges,
    the identity that links the XNOR and AND sums).

``test_oracle_pins.py`` runs every pin against the oracle; ``test_oracle_mutants.py``
plants plausible mistakes in copies of the oracle and checks that some pin fails for each.
"""
from __future__ import annotations

import os

import numpy as np

import oracle as _oracle

XNOR, AND, BW = _oracle.ORACLE_XNOR, _oracle.ORACLE_AND, _oracle.ORACLE_BINARY_WEIGHTS
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [line.split() for line in f if line.strip() and not line.startswith("#")]


def _rand_case(rng, n, h, w, ni, no, kh, kw, p=0.5):
    x = rng.standard_normal((n, h, w, ni)).astype(np.float32)
    wb = (rng.random((no, kh, kw, ni)) < p).astype(np.uint8)
    return x, wb


def _popcount(v: int) -> int:
    return bin(v).count("1")


# ----------------------------------------------------------------------------------------
# Values printed on the pages
# ----------------------------------------------------------------------------------------
def pin_truth_table(orc):
    """XNOR truth table (Bitwise XNOR page, Truth Table) with the implicit scaling
    r = 2*!(x^y) - 1 of the MPSCNNBinaryConvolution XNOR bullet; bit 1 <-> +1."""
    for a, b, out in _rows("xnor_truth_table.txt"):
        for mag in (1.0, 0.3, 7.5):
            x = np.full((1, 1, 1, 1), mag if a == "1" else -mag, np.float32)
            wb = np.full((1, 1, 1, 1), int(b), np.uint8)
            S, _, _ = orc.conv(x, wb, type=XNOR)
            assert S[0, 0] == 2 * int(out) - 1, (a, b, out, S[0, 0])


def pin_pm1_products(orc):
    """+-1 products and their logical values (Bitwise XNOR page); AND is 1 only when
    both operands are +1 (MPSCNNBinaryConvolution AND bullet, x == y == 1)."""
    for a, b, prod, logical in _rows("pm1_products.txt"):
        x = np.full((1, 1, 1, 1), float(a), np.float32)
        wb = np.full((1, 1, 1, 1), 1 if b == "+1" else 0, np.uint8)
        S, _, _ = orc.conv(x, wb, type=XNOR)
        assert S[0, 0] == float(prod)
        assert (S[0, 0] + 1) / 2 == int(logical)
        S, _, _ = orc.conv(x, wb, type=AND)
        assert S[0, 0] == (1.0 if (a == "+1" and b == "+1") else 0.0)


def pin_word_results(orc):
    """Per-32-bit-word results: XNOR gives 32 - 2*popcount(x^y) in {-32,-30,...,32},
    AND gives popcount(x&y) in {0..32} (MPSCNNBinaryConvolution XNOR / AND bullets)."""
    sets = {}
    for mode, first, last, step in _rows("word_results.txt"):
        sets[mode] = set(range(int(first), int(last) + 1, int(step)))
    rng = np.random.default_rng(11)
    words = [0, 0xFFFFFFFF, 0x55555555, 0xAAAAAAAA, 1, 0x80000000]
    words += [int(v) for v in rng.integers(0, 2**32, 60, dtype=np.uint64)]
    pairs = [(a, b) for a in words[:6] for b in words[:6]]
    pairs += list(zip(words[6:36], words[36:66]))
    mags = rng.uniform(0.1, 3.0, 32).astype(np.float32)
    for a, b in pairs:
        bits_a = [(a >> i) & 1 for i in range(32)]
        bits_b = [(b >> i) & 1 for i in range(32)]
        x = np.array([m if bit else -m for m, bit in zip(mags, bits_a)], np.float32).reshape(1, 1, 1, 32)
        wb = np.array(bits_b, np.uint8).reshape(1, 1, 1, 32)
        Sx, _, _ = orc.conv(x, wb, type=XNOR)
        Sa, _, _ = orc.conv(x, wb, type=AND)
        assert Sx[0, 0] == 32 - 2 * _popcount(a ^ b), (hex(a), hex(b))
        assert Sx[0, 0] == 2 * _popcount(~(a ^ b) & 0xFFFFFFFF) - 32
        assert Sa[0, 0] == _popcount(a & b)
        assert int(Sx[0, 0]) in sets["xnor"] and int(Sa[0, 0]) in sets["and"]


# ----------------------------------------------------------------------------------------
# Brute force and library routines
# ----------------------------------------------------------------------------------------
def _brute_conv(x, wb, op, stride, in_scale, in_bias, use_beta, relu, scale, bias):
    """Zero-padded windows and einsum, float64.  Window rows [-floor(k/2), floor((k-1)/2)]."""
    xt = x.astype(np.float64)
    if in_scale is not None:
        xt = xt * in_scale.astype(np.float64)
    if in_bias is not None:
        xt = xt + in_bias.astype(np.float64)
    sign = np.where(xt.astype(np.float32) < 0, -1.0, 1.0)
    if op == XNOR:
        a, wv = sign, 2.0 * wb - 1.0
    elif op == AND:
        a, wv = (sign > 0).astype(np.float64), wb.astype(np.float64)
    else:
        a, wv = xt, 2.0 * wb - 1.0
    n, h, w, ni = x.shape
    no, kh, kw, _ = wb.shape
    sy, sx = stride
    ho, wo = -(-h // sy), -(-w // sx)
    pad = ((0, 0), (kh // 2, (kh - 1) // 2), (kw // 2, (kw - 1) // 2), (0, 0))
    ap = np.pad(a, pad)
    Ap = np.pad(np.abs(xt).mean(axis=3, keepdims=True), pad)
    S = np.zeros((n, ho, wo, no))
    beta = np.ones((n, ho, wo))
    for oy in range(ho):
        for ox in range(wo):
            win = ap[:, oy * sy:oy * sy + kh, ox * sx:ox * sx + kw, :]
            S[:, oy, ox, :] = np.einsum("nhwf,chwf->nc", win, wv)
            if use_beta:
                beta[:, oy, ox] = Ap[:, oy * sy:oy * sy + kh, ox * sx:ox * sx + kw, 0].sum(axis=(1, 2)) / (kh * kw)
    y = S * scale.astype(np.float64) * beta[..., None] + bias.astype(np.float64)
    if relu:
        y = np.maximum(y, 0.0)
    return S.reshape(-1, no), beta.reshape(-1), y.reshape(-1, no)


def pin_brute_force_tiny(orc):
    """Every mode, beta on/off, ReLU, input terms, strides 1-2, kernels 1-4 (odd and even),
    against zero-padded brute force in float64."""
    rng = np.random.default_rng(5)
    cases = [
        (1, 4, 5, 3, 2, 3, 3, (1, 1)), (2, 5, 4, 5, 3, 2, 2, (1, 1)), (1, 6, 7, 4, 2, 4, 3, (2, 1)),
        (1, 5, 5, 2, 3, 1, 1, (1, 1)), (1, 7, 6, 3, 2, 3, 2, (2, 2)), (2, 3, 3, 6, 2, 3, 3, (2, 3)),
    ]
    for (n, h, w, ni, no, kh, kw, stride) in cases:
        x, wb = _rand_case(rng, n, h, w, ni, no, kh, kw)
        scale = rng.uniform(0.5, 1.5, no).astype(np.float32)
        bias = rng.normal(0, 0.5, no).astype(np.float32)
        in_s = rng.uniform(0.8, 1.2, ni).astype(np.float32)
        in_b = rng.normal(0, 0.3, ni).astype(np.float32)
        for op in (XNOR, AND, BW):
            for terms in (False, True):
                for use_beta, relu in ((False, False), (True, True), (True, False)):
                    kw_ = dict(scale=scale, bias=bias, in_scale=in_s if terms else None,
                               in_bias=in_b if terms else None, use_beta=use_beta, relu=relu)
                    S, beta, y = orc.conv(x, wb, type=op, stride=stride, **kw_)
                    Sb, betab, yb = _brute_conv(x, wb, op, stride, kw_["in_scale"], kw_["in_bias"],
                                                use_beta, relu, scale, bias)
                    if op == BW:
                        np.testing.assert_allclose(S, Sb, rtol=1e-12, atol=1e-12)
                    else:
                        np.testing.assert_array_equal(S, Sb)
                    np.testing.assert_allclose(beta, betab, rtol=1e-12)
                    np.testing.assert_allclose(y, yb, rtol=1e-12, atol=1e-12)


def pin_torch_conv2d(orc):
    """float64 torch.nn.functional.conv2d (cross-correlation with zero padding) on +-1,
    {0,1} or full-precision operands; zero padding is exactly 'out-of-image taps add 0'.
    Weights [No][kh][kw][Ni] permute to torch's [No][Ni][kh][kw]."""
    import torch
    import torch.nn.functional as F

    rng = np.random.default_rng(7)
    for (n, h, w, ni, no, kh, kw, sy, sx) in [(2, 9, 7, 37, 5, 3, 3, 1, 1), (1, 11, 10, 33, 4, 5, 5, 2, 2),
                                               (2, 6, 8, 20, 3, 2, 4, 1, 2), (1, 8, 8, 64, 6, 7, 1, 3, 1)]:
        x, wb = _rand_case(rng, n, h, w, ni, no, kh, kw, p=0.4)
        xt = torch.from_numpy(x.astype(np.float64)).permute(0, 3, 1, 2)
        sign = torch.where(xt < 0, -1.0, 1.0).double()
        wt = torch.from_numpy(wb.astype(np.float64)).permute(0, 3, 1, 2)
        for op, a, wv in ((XNOR, sign, 2 * wt - 1), (AND, (sign > 0).double(), wt), (BW, xt, 2 * wt - 1)):
            ap = F.pad(a, (kw // 2, (kw - 1) // 2, kh // 2, (kh - 1) // 2))
            ref = F.conv2d(ap, wv, stride=(sy, sx)).permute(0, 2, 3, 1).reshape(-1, no).numpy()
            S, _, _ = orc.conv(x, wb, type=op, stride=(sy, sx))
            assert S.shape == ref.shape, (S.shape, ref.shape)
            if op == BW:
                np.testing.assert_allclose(S, ref, rtol=1e-12, atol=1e-11)
            else:
                np.testing.assert_array_equal(S, ref)


def pin_signed_zero(orc):
    """bin(x) = x < 0 ? -1 : 1 makes +0 and -0 map to +1; any negative value to -1."""
    rng = np.random.default_rng(3)
    x, wb = _rand_case(rng, 1, 4, 4, 8, 3, 3, 3)
    x[0, :, :, :3] = 0.0
    x[0, :, :, 3:5] = -0.0
    x[0, :, :, 5] = -1e-30
    ones = x.copy()
    ones[0, :, :, :5] = 1.0
    for op in (XNOR, AND):
        S0, _, _ = orc.conv(x, wb, type=op)
        S1, _, _ = orc.conv(ones, wb, type=op)
        np.testing.assert_array_equal(S0, S1)
    neg = x.copy()
    neg[0, :, :, 5] = -1.0
    np.testing.assert_array_equal(orc.conv(x, wb, type=XNOR)[0], orc.conv(neg, wb, type=XNOR)[0])


def pin_fc_matvec(orc):
    """Fully connected = the flattened W*H*Ni vector times an No x (W*H*Ni) matrix
    (MPSCNNFullyConnected Overview); with beta the window is the whole image, so
    beta_n = ||x~_n||_1 / (H*W*Ni)."""
    rng = np.random.default_rng(9)
    for (n, h, w, ni, no) in [(3, 3, 3, 5, 4), (2, 2, 5, 33, 7), (4, 4, 4, 2, 3), (1, 1, 1, 70, 2)]:
        x, wb = _rand_case(rng, n, h, w, ni, no, h, w)
        scale = rng.uniform(0.001, 0.01, no).astype(np.float32)
        bias = rng.normal(0, 0.1, no).astype(np.float32)
        in_s = rng.uniform(0.8, 1.2, ni).astype(np.float32)
        in_b = rng.normal(0, 0.1, ni).astype(np.float32)
        xt = x.astype(np.float64) * in_s + in_b
        v = xt.reshape(n, -1)
        sign = np.where(v.astype(np.float32) < 0, -1.0, 1.0)
        m = wb.reshape(no, -1).astype(np.float64)
        for op, a, wm in ((XNOR, sign, 2 * m - 1), (AND, (sign > 0) * 1.0, m), (BW, v, 2 * m - 1)):
            S, beta, y = orc.fc(x, wb, type=op, scale=scale, bias=bias, in_scale=in_s, in_bias=in_b,
                                use_beta=True)
            ref = a @ wm.T
            if op == BW:
                np.testing.assert_allclose(S, ref, rtol=1e-12, atol=1e-11)
            else:
                np.testing.assert_array_equal(S, ref)
            np.testing.assert_allclose(beta, np.abs(v).sum(axis=1) / v.shape[1], rtol=1e-12)


def pin_fc_is_conv_at_centre(orc):
    """MPSCNNFullyConnected Note: the layer equals a convolution with kernel = source size,
    offset (kW/2, kH/2), a 1x1 clip and stride 1 -- the conv output at (H/2, W/2)."""
    rng = np.random.default_rng(13)
    for (n, h, w, ni, no) in [(2, 3, 3, 4, 3), (2, 4, 5, 6, 2), (1, 2, 2, 40, 3), (3, 7, 7, 3, 2)]:
        x, wb = _rand_case(rng, n, h, w, ni, no, h, w)
        scale = rng.uniform(0.5, 1.5, no).astype(np.float32)
        bias = rng.normal(0, 0.2, no).astype(np.float32)
        pix = np.array([(i * h + h // 2) * w + w // 2 for i in range(n)], np.int64)
        for op in (XNOR, AND, BW):
            for use_beta in (False, True):
                a = orc.fc(x, wb, type=op, scale=scale, bias=bias, use_beta=use_beta, relu=True)
                b = orc.conv(x, wb, type=op, scale=scale, bias=bias, use_beta=use_beta, relu=True, pixels=pix)
                for u, v in zip(a, b):
                    np.testing.assert_allclose(u, v, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------------------
# Closed forms and invariants
# ----------------------------------------------------------------------------------------
def _valid_taps(h, w, kh, kw, sy, sx):
    ho, wo = -(-h // sy), -(-w // sx)
    cnt = np.zeros((ho, wo))
    for oy in range(ho):
        for ox in range(wo):
            for dy in range(-(kh // 2), (kh - 1) // 2 + 1):
                for dx in range(-(kw // 2), (kw - 1) // 2 + 1):
                    y, x = oy * sy + dy, ox * sx + dx
                    cnt[oy, ox] += (0 <= y < h) and (0 <= x < w)
    return cnt


def pin_beta_closed_form(orc):
    """Constant |x~| = a gives A = a everywhere, so beta = a * (valid taps) / (kx*ky): the
    interior gets a, a 3x3 corner 4a/9, an edge 6a/9 (MPSCNNBinaryConvolution beta formulas;
    the window holds exactly k taps for odd and even k)."""
    rng = np.random.default_rng(17)
    a = 0.75
    for (h, w, kh, kw, sy, sx) in [(5, 6, 3, 3, 1, 1), (4, 4, 2, 2, 1, 1), (6, 5, 4, 3, 1, 1), (7, 7, 3, 3, 2, 2),
                                   (5, 5, 5, 1, 2, 1)]:
        x = (np.where(rng.random((2, h, w, 6)) < 0.5, -a, a)).astype(np.float32)
        wb = (rng.random((2, kh, kw, 6)) < 0.5).astype(np.uint8)
        _, beta, _ = orc.conv(x, wb, type=XNOR, stride=(sy, sx), use_beta=True)
        expect = np.tile((a * _valid_taps(h, w, kh, kw, sy, sx) / (kh * kw)).reshape(-1), 2)
        np.testing.assert_allclose(beta, expect, rtol=1e-15)
    x = np.full((1, 5, 5, 4), a, np.float32)
    wb = np.ones((1, 3, 3, 4), np.uint8)
    _, beta, _ = orc.conv(x, wb, type=AND, use_beta=True)
    assert beta[0] == a * 4 / 9 and beta[1] == a * 6 / 9 and beta[6] == a


def pin_input_terms(orc):
    """x~ = inScale*x + inBias is applied before binarization and before beta: on inputs
    where the affine map is exact in fp32, passing the terms equals passing x~ itself."""
    rng = np.random.default_rng(19)
    n, h, w, ni, no = 2, 5, 4, 6, 3
    x = (rng.integers(-16, 17, (n, h, w, ni)) / 8.0).astype(np.float32)
    wb = (rng.random((no, 3, 3, ni)) < 0.5).astype(np.uint8)
    in_s = np.array([2.0, 0.5, -1.0, 1.5, 0.25, -2.0], np.float32)
    in_b = np.array([0.125, -0.5, 0.0, 1.0, -0.25, 0.375], np.float32)
    xt = (x * in_s + in_b).astype(np.float32)  # exact: small multiples of 1/32
    assert np.array_equal(xt.astype(np.float64), x.astype(np.float64) * in_s + in_b)
    scale = rng.uniform(0.5, 1.5, no).astype(np.float32)
    bias = rng.normal(0, 0.2, no).astype(np.float32)
    for op in (XNOR, AND, BW):
        a = orc.conv(x, wb, type=op, scale=scale, bias=bias, in_scale=in_s, in_bias=in_b, use_beta=True)
        b = orc.conv(xt, wb, type=op, scale=scale, bias=bias, use_beta=True)
        for u, v in zip(a, b):
            np.testing.assert_array_equal(u, v)
        a = orc.fc(x, np.ascontiguousarray(np.repeat(wb[:, :1, :1], h, 1).repeat(w, 2)), type=op,
                   in_scale=in_s, in_bias=in_b, use_beta=True)
        b = orc.fc(xt, np.ascontiguousarray(np.repeat(wb[:, :1, :1], h, 1).repeat(w, 2)), type=op, use_beta=True)
        for u, v in zip(a, b):
            np.testing.assert_array_equal(u, v)


def pin_invariants(orc):
    """Parity and range of the sums, the XNOR/AND identity
    S_xnor = K_v - 2 P_a - 2 P_w + 4 S_and (from (2a-1)(2w-1) = 4aw - 2a - 2w + 1),
    negation under flipped weights, and binaryWeights on bin(x) = XNOR."""
    rng = np.random.default_rng(23)
    n, h, w, ni, no = 2, 6, 5, 19, 4
    for (kh, kw, s) in ((3, 3, 1), (2, 2, 1), (3, 3, 2), (5, 3, 1)):
        x, wb = _rand_case(rng, n, h, w, ni, no, kh, kw, p=0.3)
        Sx = orc.conv(x, wb, type=XNOR, stride=(s, s))[0]
        Sa = orc.conv(x, wb, type=AND, stride=(s, s))[0]
        pos = np.abs(x) + 1.0
        K_v = orc.conv(pos, np.ones_like(wb), type=AND, stride=(s, s))[0]
        P_a = orc.conv(x, np.ones_like(wb), type=AND, stride=(s, s))[0]
        P_w = orc.conv(pos, wb, type=AND, stride=(s, s))[0]
        valid = np.repeat(_valid_taps(h, w, kh, kw, s, s).reshape(1, -1), n, 0).reshape(-1, 1) * ni
        np.testing.assert_array_equal(K_v, np.broadcast_to(valid, K_v.shape))
        assert np.all(np.abs(Sx) <= K_v) and np.all((Sx - K_v) % 2 == 0)
        assert np.all(Sa >= 0) and np.all(Sa <= np.minimum(P_a, P_w))
        np.testing.assert_array_equal(Sx, K_v - 2 * P_a - 2 * P_w + 4 * Sa)
        np.testing.assert_array_equal(orc.conv(x, 1 - wb, type=XNOR, stride=(s, s))[0], -Sx)
        signs = np.where(x < 0, -1.0, 1.0).astype(np.float32)
        np.testing.assert_array_equal(orc.conv(signs, wb, type=BW, stride=(s, s))[0], Sx)


def pin_epilogue(orc):
    """out = S*scale[c]*beta + bias[c], then the neuron: special cases that fix each term."""
    rng = np.random.default_rng(29)
    n, h, w, ni, no = 2, 5, 5, 7, 5
    x, wb = _rand_case(rng, n, h, w, ni, no, 3, 3)
    scale = rng.uniform(0.5, 1.5, no).astype(np.float32)
    bias = rng.normal(0, 2.0, no).astype(np.float32)
    for op in (XNOR, AND, BW):
        S, _, y = orc.conv(x, wb, type=op)
        np.testing.assert_array_equal(y, S)  # scale 1, bias 0, no beta, identity
        _, _, y1 = orc.conv(x, wb, type=op, scale=scale)
        np.testing.assert_array_equal(y1, S * scale.astype(np.float64))
        _, _, y2 = orc.conv(x, wb, type=op, scale=scale, bias=bias)
        np.testing.assert_array_equal(y2, y1 + bias.astype(np.float64))
        _, _, y3 = orc.conv(x, wb, type=op, scale=scale, bias=bias, relu=True)
        np.testing.assert_array_equal(y3, np.maximum(y2, 0.0))
        assert (y2 < 0).any() and (y2 > 0).any()
        _, _, y4 = orc.conv(x, wb, type=op, scale_value=0.75)
        np.testing.assert_array_equal(y4, S * 0.75)
        _, beta, y5 = orc.conv(x, wb, type=op, scale=scale, use_beta=True)
        assert np.all(beta > 0)
        np.testing.assert_allclose(y5, y1 * beta[:, None], rtol=1e-15)


# ----------------------------------------------------------------------------------------
# The binarized view of an image (what a following binary layer reads)
# ----------------------------------------------------------------------------------------
def pin_binarize_golden(orc):
    """Hand-worked bits and A (tests/golden/binarize_examples.txt): input terms before the
    sign, bin(+-0) = +1, the sign decided in fp32, A = mean |x~| (MPSCNNBinaryConvolution)."""
    terms, xs, bits, As = {}, {}, {}, {}
    for row in _rows("binarize_examples.txt"):
        tag, idx, vals = row[0], int(row[1]), row[2:]
        if tag == "T":
            terms[idx] = (float(vals[0]), float(vals[1]))
        elif tag == "P":
            xs[idx] = [float(v) for v in vals]
        elif tag == "B":
            bits[idx] = [int(v) for v in vals]
        elif tag == "A":
            As[idx] = float(vals[0])
    c = len(terms)
    s = np.array([terms[i][0] for i in range(c)], np.float32)
    b = np.array([terms[i][1] for i in range(c)], np.float32)
    x = np.array([xs[p] for p in sorted(xs)], np.float32)
    got_bits, got_A, _ = orc.binarize(x, in_scale=s, in_bias=b)
    np.testing.assert_array_equal(got_bits, np.array([bits[p] for p in sorted(bits)], np.uint8))
    np.testing.assert_allclose(got_A, np.array([As[p] for p in sorted(As)]), rtol=1e-12)


def pin_binarize_is_the_conv_input(orc):
    """The bits and A of the binarized view are exactly what the (separately pinned) binary
    convolution sums and averages: brute-force XNOR/AND sums over the bits equal the conv's S,
    and the window mean of A equals its beta."""
    rng = np.random.default_rng(41)
    n, h, w, ni, no = 2, 5, 6, 37, 4
    x, wb = _rand_case(rng, n, h, w, ni, no, 3, 3)
    in_scale = rng.uniform(-1.5, 1.5, ni).astype(np.float32)
    in_bias = rng.normal(0, 0.5, ni).astype(np.float32)
    bits, A, xt = orc.binarize(x, in_scale=in_scale, in_bias=in_bias)
    assert bits.shape == x.shape and A.shape == x.shape[:3]
    assert 0 < bits.mean() < 1
    pad = ((0, 0), (1, 1), (1, 1), (0, 0))
    for op in (XNOR, AND):
        a = (2.0 * bits - 1.0) if op == XNOR else bits.astype(np.float64)
        wv = (2.0 * wb - 1.0) if op == XNOR else wb.astype(np.float64)
        ap = np.pad(a, pad)
        ref = np.zeros((n, h, w, no))
        for oy in range(h):
            for ox in range(w):
                ref[:, oy, ox, :] = np.einsum("nhwf,chwf->nc", ap[:, oy:oy + 3, ox:ox + 3, :], wv)
        S, beta, _ = orc.conv(x, wb, type=op, in_scale=in_scale, in_bias=in_bias, use_beta=True)
        np.testing.assert_array_equal(S, ref.reshape(-1, no))
        Ap = np.pad(A, ((0, 0), (1, 1), (1, 1)))
        bref = np.stack([Ap[:, oy:oy + 3, ox:ox + 3].sum(axis=(1, 2)) / 9.0 for oy in range(h) for ox in range(w)], 1)
        np.testing.assert_allclose(beta, bref.reshape(-1), rtol=1e-12)
    np.testing.assert_allclose(np.abs(xt).mean(axis=-1), A, rtol=1e-12)


ALL_PINS = [
    pin_truth_table, pin_pm1_products, pin_word_results, pin_brute_force_tiny, pin_torch_conv2d,
    pin_signed_zero, pin_fc_matvec, pin_fc_is_conv_at_centre, pin_beta_closed_form, pin_input_terms,
    pin_invariants, pin_epilogue, pin_binarize_golden, pin_binarize_is_the_conv_input,
]
