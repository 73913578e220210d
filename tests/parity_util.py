"""Shared helpers of the parity tests: run a workload through the library and the oracle,
and compare with the tolerance of the float outputs.

Tolerance (float outputs).  The device computes S exactly (XNOR/AND) or as an FP32 sum
(binaryWeights), beta in FP32, and out = act(S*scale*beta + bias) in FP32; the oracle does
everything in double.  For output i the error is measured against the size of the terms
whose FP32 rounding produces it:

    err_i = |y_dev - y_ref| / max(|y_ref|, D_i),
    D_i   = |scale_c * beta| * |S| + |bias_c|                (XNOR, AND)
    D_i   = |scale_c * beta| * sum_window |x~| + |bias_c|     (binaryWeights)

and every err_i must be <= 1e-5 (the relative bound the workloads are specified with).
Where |y_ref| >= D_i this is the plain relative error; near a zero crossing of the
pre-activation the plain relative error of any FP32 evaluation is unbounded, and D_i is
the standard forward-error scale there.  Integer sums (XNOR/AND) are compared bit for bit.
"""
from __future__ import annotations

import numpy as np

import oracle
from binarized_convolution_b200 import BinaryConv2d, BinaryFC
from binarized_convolution_b200 import synth

REL_TOL = 1e-5

_ORACLE_TYPE = {synth.XNOR: oracle.ORACLE_XNOR, synth.AND: oracle.ORACLE_AND,
                synth.BINARY_WEIGHTS: oracle.ORACLE_BINARY_WEIGHTS}


def make_layer(w: synth.Workload, inp: synth.Inputs, *, sums: bool = False):
    """The library layer for a workload.  sums=True keeps the weights and input terms but
    sets scale 1, bias 0, no beta and no neuron, so the output is the raw sum S."""
    kw = dict(op=w.op, in_scale=inp.in_scale, in_bias=inp.in_bias)
    if sums:
        kw.update(scale=None, scale_value=1.0, bias=None, use_beta=False, relu=False)
    else:
        kw.update(scale=inp.scale, bias=inp.bias, use_beta=w.use_beta, relu=w.relu)
    if w.kind == "fc":
        return BinaryFC(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, wbits=inp.wbits, **kw)
    return BinaryConv2d(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, (w.kernel_h, w.kernel_w),
                        (w.stride_y, w.stride_x), wbits=inp.wbits, **kw)


# Kernel families a parity case runs on: the library's choice (e2m1 codes for XNOR/AND; the
# rows-staged kernel for stride-1 convolutions it fits, on SM pairs above 128 output channels),
# the same codes with the per-tap staging forced, the rows-staged kernel forced onto one SM per
# tile, the SIMT family, and the tensor cores with int8 codes forced onto one SM per tile or onto
# SM pairs.
FAMILIES = ["auto", "per_tap", "rows_single", "alt", "single", "pair"]


def algo_for(w: synth.Workload, name: str):
    """Library algorithm code for a test parameter: 'auto' (the library's choice: the tensor
    cores where they apply), 'alt' (the SIMT family: POPC for XNOR/AND, the FP32 signed-add
    kernel for binaryWeights), or 'single' / 'pair' (the library's choice, with the
    tensor-core contraction of the layers created after this call forced onto one SM per
    tile or onto SM pairs, XNOR/AND with int8 codes; the test fixture puts the process-wide
    settings back to AUTO)."""
    import binarized_convolution_b200 as bc

    bc.bconv_set_cta_mode({"single": bc.CTA_SINGLE, "pair": bc.CTA_PAIR, "rows_single": bc.CTA_SINGLE}.get(
        name, bc.CTA_AUTO))
    bc.bconv_set_tc_codes(bc.CODES_INT8 if name in ("single", "pair") else bc.CODES_AUTO)
    bc.bconv_set_staging(bc.STAGING_PER_TAP if name == "per_tap" else bc.STAGING_AUTO)
    if name == "alt":
        return bc.ALGO_SIMT_F32 if w.op == synth.BINARY_WEIGHTS else bc.ALGO_POPC
    return bc.ALGO_AUTO


def run_device(w: synth.Workload, inp: synth.Inputs, *, sums: bool = False, algo=None):
    """Output of the library, as float32 [rows, No] (rows = output pixels or images)."""
    import torch

    layer = make_layer(w, inp, sums=sums)
    try:
        if algo is not None:
            layer.set_algo(algo)
        x = torch.from_numpy(inp.x).cuda()
        y = layer(x)
        layer.sync_status()
        torch.cuda.synchronize()
        return y.reshape(-1, w.out_channels).cpu().numpy()
    finally:
        layer.close()


def run_oracle(w: synth.Workload, inp: synth.Inputs, *, rows=None, sums: bool = False):
    """(S, beta, y) from the oracle for the given output rows (all when None)."""
    t = _ORACLE_TYPE[w.op]
    kw = dict(type=t, in_scale=inp.in_scale, in_bias=inp.in_bias)
    if sums:
        kw.update(scale_value=1.0)
    else:
        kw.update(scale=inp.scale, bias=inp.bias, use_beta=w.use_beta, relu=w.relu)
    if w.kind == "fc":
        return oracle.fc(inp.x, inp.wbits, rows=rows, **kw)
    return oracle.conv(inp.x, inp.wbits, stride=(w.stride_y, w.stride_x), pixels=rows, **kw)


def window_abs_sum(w: synth.Workload, inp: synth.Inputs, rows=None):
    """sum over the valid window of |x~| for each output row (from the oracle's beta)."""
    t = _ORACLE_TYPE[w.op]
    if w.kind == "fc":
        _, beta, _ = oracle.fc(inp.x, inp.wbits, type=t, in_scale=inp.in_scale, in_bias=inp.in_bias,
                               use_beta=True, rows=rows)
    else:
        _, beta, _ = oracle.conv(inp.x, inp.wbits, type=t, stride=(w.stride_y, w.stride_x), in_scale=inp.in_scale,
                                 in_bias=inp.in_bias, use_beta=True, pixels=rows)
    return beta * (w.kernel_h * w.kernel_w * w.in_channels)


def assert_sums_exact(S_dev, S_ref):
    S_ref = np.asarray(S_ref)
    assert np.all(np.abs(S_ref) < 2 ** 24)
    bad = np.nonzero(S_dev.astype(np.float64) != S_ref)
    assert bad[0].size == 0, (
        f"{bad[0].size} integer sums differ; first at {tuple(b[0] for b in bad)}: "
        f"device {S_dev[tuple(b[0] for b in bad)]} oracle {S_ref[tuple(b[0] for b in bad)]}")


def error_scale(w, inp, S_ref, beta_ref, rows=None):
    """D_i of the tolerance for each output (see the module docstring)."""
    scale = np.abs(inp.scale.astype(np.float64))[None, :]
    bias = np.abs(inp.bias.astype(np.float64))[None, :]
    beta = np.abs(beta_ref)[:, None]
    if w.op == synth.BINARY_WEIGHTS:
        mag = window_abs_sum(w, inp, rows)[:, None]
    else:
        mag = np.abs(S_ref)
    return scale * beta * mag + bias


def relative_errors(w, inp, y_dev, S_ref, beta_ref, y_ref, rows=None):
    D = error_scale(w, inp, S_ref, beta_ref, rows)
    denom = np.maximum(np.abs(y_ref), D)
    denom = np.where(denom == 0, 1.0, denom)
    return np.abs(y_dev.astype(np.float64) - y_ref) / denom


def assert_outputs_close(w, inp, y_dev, S_ref, beta_ref, y_ref, rows=None, tol=REL_TOL):
    err = relative_errors(w, inp, y_dev, S_ref, beta_ref, y_ref, rows)
    worst = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= tol, (f"max error {err.max():.3e} > {tol:g} at {worst}: device {y_dev[worst]!r} "
                              f"oracle {y_ref[worst]!r}")
    return float(err.max())


def sample_rows(w: synth.Workload, n_random: int | None = None, seed: int = 0, ops_budget: float = 3e8) -> np.ndarray:
    """Output rows to check at full size: every image's corners and edge midpoints, the
    last row (the ragged tail of the last tile), and n_random rows drawn at random (by
    default as many as fit about ops_budget bit operations of oracle work, 4 to 512)."""
    if n_random is None:
        per_row = w.nominal_ops / (w.batch * w.out_h * w.out_w)
        n_random = int(min(512, max(4, ops_budget // per_row)))
    if w.kind == "fc":
        rng = np.random.default_rng(seed)
        rows = set(rng.choice(w.batch, size=min(n_random, w.batch), replace=False).tolist())
        rows |= {0, w.batch - 1}
        return np.array(sorted(rows), np.int64)
    ho, wo = w.out_h, w.out_w
    rows = set()
    for n in sorted({0, w.batch // 2, w.batch - 1}):
        for oy in (0, ho // 2, ho - 1):
            for ox in (0, wo // 2, wo - 1):
                rows.add((n * ho + oy) * wo + ox)
    total = w.batch * ho * wo
    rng = np.random.default_rng(seed)
    rows |= set(rng.choice(total, size=min(n_random, total), replace=False).tolist())
    rows.add(total - 1)
    return np.array(sorted(rows), np.int64)
