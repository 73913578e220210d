"""Seeded synthetic inputs for the binary convolution workloads.

This module only draws random numbers; it holds none of the method's arithmetic, and
both the CUDA library's tests and the oracle take their inputs from it.

Every workload draws, in this order, from ``numpy.random.default_rng(seed)``:
input x (fp32 N(0,1), NHWC), weight bits (Bernoulli(p) as uint8 0/1, layout
``[No][kh][kw][Ni]``), scale[c] ~ U(lo, hi), bias[c] ~ N(0, 0.1), and, when the workload
uses input terms, inputScale[f] ~ U(0.8, 1.2) and inputBias[f] ~ N(0, 0.1).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

XNOR = "xnor"
AND = "and"
BINARY_WEIGHTS = "binary_weights"


@dataclass(frozen=True)
class Workload:
    """Shape and value distribution of one binary-convolution workload."""

    name: str
    kind: str  # "conv" or "fc" (kernel = source size)
    batch: int
    in_h: int
    in_w: int
    in_channels: int
    out_channels: int
    kernel_h: int
    kernel_w: int
    stride_y: int
    stride_x: int
    op: str  # XNOR, AND or BINARY_WEIGHTS
    use_beta: bool
    relu: bool
    in_terms: bool
    scale_lo: float
    scale_hi: float
    p_weight: float
    seed: int

    @property
    def out_h(self) -> int:
        return 1 if self.kind == "fc" else -(-self.in_h // self.stride_y)

    @property
    def out_w(self) -> int:
        return 1 if self.kind == "fc" else -(-self.in_w // self.stride_x)

    @property
    def nominal_ops(self) -> int:
        """Bit multiply-accumulates of the full window at every output (1 op = 1 bit MAC)."""
        return (self.batch * self.out_h * self.out_w * self.out_channels
                * self.kernel_h * self.kernel_w * self.in_channels)

    def with_batch(self, batch: int) -> "Workload":
        return replace(self, batch=batch)


def _conv(name, n, h, w, ni, no, k, s, op, beta, relu, in_terms, lo, hi, p, seed):
    return Workload(name, "conv", n, h, w, ni, no, k, k, s, s, op, beta, relu, in_terms, lo, hi, p, seed)


# The five workloads the library is measured and checked on.
WORKLOADS = {
    w.name: w
    for w in (
        _conv("xnor_n1_8x8_c64_k32_3x3", 1, 8, 8, 64, 32, 3, 1, XNOR, False, False, False, 0.5, 1.5, 0.5, 0),
        _conv("xnor_beta_n16_56x56_c256_k256_3x3", 16, 56, 56, 256, 256, 3, 1, XNOR, True, True, True,
              0.5, 1.5, 0.5, 1),
        _conv("and_n32_28x28_c512_k512_3x3", 32, 28, 28, 512, 512, 3, 1, AND, False, False, False,
              0.01, 0.05, 0.3, 2),
        _conv("binw_n8_112x112_c128_k128_3x3_s2", 8, 112, 112, 128, 128, 3, 2, BINARY_WEIGHTS, False, True,
              False, 0.01, 0.1, 0.5, 3),
        Workload("fc_xnor_beta_n256_7x7x512_k4096", "fc", 256, 7, 7, 512, 4096, 7, 7, 1, 1, XNOR, True, False,
                 False, 0.001, 0.01, 0.5, 4),
    )
}
WORKLOAD_ORDER = list(WORKLOADS)


def workload(key) -> Workload:
    """Look a workload up by name or by its position (0-4) in WORKLOAD_ORDER."""
    if isinstance(key, int):
        return WORKLOADS[WORKLOAD_ORDER[key]]
    return WORKLOADS[key]


@dataclass
class Inputs:
    x: np.ndarray  # float32 [N, H, W, Ni]
    wbits: np.ndarray  # uint8 {0,1} [No, kh, kw, Ni]
    scale: np.ndarray  # float32 [No]
    bias: np.ndarray  # float32 [No]
    in_scale: np.ndarray | None  # float32 [Ni]
    in_bias: np.ndarray | None  # float32 [Ni]


def make_inputs(w: Workload, seed: int | None = None) -> Inputs:
    """Draw one workload's inputs (order: x, weight bits, scale, bias, inScale, inBias)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    x = rng.standard_normal((w.batch, w.in_h, w.in_w, w.in_channels), dtype=np.float32)
    wshape = (w.out_channels, w.kernel_h, w.kernel_w, w.in_channels)
    wbits = (rng.random(wshape, dtype=np.float32) < w.p_weight).astype(np.uint8)
    scale = rng.uniform(w.scale_lo, w.scale_hi, w.out_channels).astype(np.float32)
    bias = rng.normal(0.0, 0.1, w.out_channels).astype(np.float32)
    in_scale = in_bias = None
    if w.in_terms:
        in_scale = rng.uniform(0.8, 1.2, w.in_channels).astype(np.float32)
        in_bias = rng.normal(0.0, 0.1, w.in_channels).astype(np.float32)
    return Inputs(x, wbits, scale, bias, in_scale, in_bias)


def make_batch(w: Workload, seed: int) -> np.ndarray:
    """A fresh input batch of the workload's shape (fp32 N(0,1)), for rotating buffers."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((w.batch, w.in_h, w.in_w, w.in_channels), dtype=np.float32)


def small_case(*, batch=1, h=5, w=5, ni=3, no=2, k=3, kw=None, stride=1, stride_x=None, op=XNOR,
               use_beta=False, relu=False, in_terms=False, p=0.5, seed=0, kind="conv",
               scale=(0.5, 1.5)) -> Workload:
    """A small workload for parity and edge-case tests."""
    kw = k if kw is None else kw
    sx = stride if stride_x is None else stride_x
    if kind == "fc":
        k, kw, stride, sx = h, w, 1, 1
    return Workload(f"case_{kind}_{op}_{batch}x{h}x{w}x{ni}_k{no}_{k}x{kw}_s{stride}{sx}_{seed}", kind,
                    batch, h, w, ni, no, k, kw, stride, sx, op, use_beta, relu, in_terms, scale[0], scale[1],
                    p, seed)


def next_terms(no: int, seed: int, bias_spread: float = 0.1) -> tuple[np.ndarray, np.ndarray]:
    """Input terms of a following binary layer (chained layers): scales of random sign and
    magnitude U(0.5, 1.5), biases N(0, bias_spread), as float32 [no] each."""
    rng = np.random.default_rng(seed)
    mag = rng.uniform(0.5, 1.5, no)
    sign = np.where(rng.random(no) < 0.5, -1.0, 1.0)
    return (mag * sign).astype(np.float32), rng.normal(0.0, bias_spread, no).astype(np.float32)
