"""The vectorised CPU baseline (cpu_simd/) against the oracle, on the CPU: exact integer window
sums for XNOR / AND and float outputs within the parity tolerance, on every vector path this CPU
has (AVX-512 VPOPCNTQ, AVX2 nibble lookup, scalar POPCNT), over word-boundary channel counts,
odd and even kernels, strides, beta, input terms and the fully-connected case."""
import itertools

import numpy as np
import pytest

import cpu_simd
import parity_util as pu
from binarized_convolution_b200 import synth
import binarized_convolution_b200 as bc

ISAS = list(range(cpu_simd.best_isa() + 1))
_TYPE = {synth.XNOR: cpu_simd.XNOR, synth.AND: cpu_simd.AND, synth.BINARY_WEIGHTS: cpu_simd.BINARY_WEIGHTS}

CASES = []
for i, (ni, k, s, op) in enumerate(itertools.product([1, 31, 32, 33, 100], [1, 2, 3, 5], [1, 2],
                                                     [synth.XNOR, synth.AND, synth.BINARY_WEIGHTS])):
    if i % 4 and k != 3:
        continue
    CASES.append(synth.small_case(batch=1 + i % 2, h=6 + i % 3, w=8 - i % 3, ni=ni, no=3 + i % 5, k=k, stride=s,
                                  op=op, use_beta=bool(i % 2), relu=bool((i // 2) % 2),
                                  in_terms=bool((i // 3) % 2), seed=3000 + i))
CASES += [synth.small_case(batch=3, h=3, w=4, ni=70, no=9, kind="fc", op=op, use_beta=True, in_terms=True,
                           seed=3200 + j) for j, op in enumerate([synth.XNOR, synth.AND, synth.BINARY_WEIGHTS])]


def _run(w, inp, isa, sums=False):
    packed = bc.bconv_pack_bits(inp.wbits.reshape(-1, w.in_channels)).reshape(*inp.wbits.shape[:3], -1)
    kw = dict(type=_TYPE[w.op], in_scale=inp.in_scale, in_bias=inp.in_bias, isa=isa)
    if sums:
        kw.update(scale_value=1.0)
    else:
        kw.update(scale=inp.scale, bias=inp.bias, use_beta=w.use_beta, relu=w.relu)
    if w.kind == "fc":
        return cpu_simd.fc(inp.x, packed, **kw)
    return cpu_simd.conv(inp.x, packed, stride=(w.stride_y, w.stride_x), **kw)


@pytest.mark.parametrize("isa", ISAS, ids=lambda i: cpu_simd.ISA_NAMES[i])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_simd_baseline_matches_oracle(w, isa):
    inp = synth.make_inputs(w)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp)
    _, y = _run(w, inp, isa)
    pu.assert_outputs_close(w, inp, y, S_ref, beta_ref, y_ref)
    if w.op != synth.BINARY_WEIGHTS:
        S_sum, _, _ = pu.run_oracle(w, inp, sums=True)
        S, _ = _run(w, inp, isa, sums=True)
        pu.assert_sums_exact(S, S_sum)


def test_simd_baseline_sampled_rows_of_a_large_layer():
    """A workload-sized layer (XNOR, beta, input terms, 56 x 56 x 256 -> 256) on sampled outputs."""
    w = synth.workload(1).with_batch(2)
    inp = synth.make_inputs(w)
    rows = pu.sample_rows(w, n_random=48)
    S_ref, beta_ref, y_ref = pu.run_oracle(w, inp, rows=rows)
    packed = bc.bconv_pack_bits(inp.wbits.reshape(-1, w.in_channels)).reshape(*inp.wbits.shape[:3], -1)
    S, y = cpu_simd.conv(inp.x, packed, type=cpu_simd.XNOR, scale=inp.scale, bias=inp.bias, in_scale=inp.in_scale,
                         in_bias=inp.in_bias, use_beta=True, relu=True, pixels=rows)
    pu.assert_outputs_close(w, inp, y, S_ref, beta_ref, y_ref, rows=rows)
    S_sum, _, _ = pu.run_oracle(w, inp, rows=rows, sums=True)
    S1, _ = cpu_simd.conv(inp.x, packed, type=cpu_simd.XNOR, in_scale=inp.in_scale, in_bias=inp.in_bias,
                          pixels=rows)
    pu.assert_sums_exact(S1, S_sum)
