"""Throughput of the binary convolution on B200: one JSON line per run.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload all|NAME|INDEX] [--seconds S] [--io f32|bits]
                    [--no-e2e] [--no-cpu-baseline]

A step is one forward of a layer (input transform + pack + A, beta, contraction and
epilogue) over one batch of a workload.  By default every one of the five workloads is
timed; the line's own fields (``value``, ``roofline``, ``e2e``, ``clocks`` ...) are those of
the headline workload -- XNOR with beta scaling and input terms, batch 16, 56x56, 256 -> 256
channels, 3x3, ReLU -- and ``workloads`` holds the same record for each of the five.

Timing: after W warm-up steps each workload runs at least K steps, and as many more as fill
about ``--seconds`` (default 2 s) of device time, so that the clock record and the sampled
kernel timings rest on many launches whatever K is; ``steps`` reports how many were timed
(``steps_requested`` is K).  The timed region is bracketed by a barrier and a device
synchronize on each side and measured with CUDA events on the launching stream; multi-GPU
runs (torchrun) are independent replicas with a batch each (weak scaling) and report the
maximum time over ranks.  Input/output buffer sets rotate so that one step's data has left
the L2 by the time it is used again (at least four sets, together more than 1.5 x the L2).

``value`` is nominal bit multiply-accumulates (every window tap, 1 op = 1 bit MAC) per second
over all ranks with inputs resident in HBM.  ``roofline`` is that of the contraction kernel:
its nominal ops over its mean launch time (CUDA events around every 8th launch inside the
timed region) against the peak of the pipe it runs on; ``forward_roofline`` compares the
whole step with max(algorithmic bytes / HBM bandwidth, ops / pipe peak).  ``clocks`` comes
from NVML reads every 5 ms during the timed region (read only; no setting is changed).
``e2e`` is the same metric through bconv_forward_host / bfc_forward_host with page-locked
host buffers (host-to-device copy, forward, device-to-host copy inside every step).
Two CPU figures sit beside it: ``cpu_baseline``, the oracle (plain double-precision loops) on
a sample of output rows, and ``cpu_simd_baseline``, the vectorised CPU implementation in
cpu_simd/ (bit-packed XOR / AND + popcount on AVX-512 or AVX2 registers) on the whole workload.

``--io bits`` times one workload as the middle of a chain of such layers instead: it reads
the bit-packed output of the previous layer (sign bits and A) and writes its own for the next
(bconv_forward_io); the input terms move to the previous layer's epilogue.

``--impl reference`` times the oracle (the plain double-precision CPU loops) on the headline
workload, each step a bounded sample of output pixels, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from binarized_convolution_b200 import synth  # noqa: E402

DEFAULT_WORKLOAD = "xnor_beta_n16_56x56_c256_k256_3x3"  # the headline workload
METRIC = "binary conv TOPS (1 op = 1 bit MAC) and images/s on 1 B200; % of roofline"
UNIT = "TOPS"
ROTATE_MIN = 4
L2_BYTES = 126 * 1024 * 1024  # B200 L2 (the device property is used when available)
TIMED_SECONDS = 2.0  # device time each workload's timed region fills (at least --steps steps)
CLOCK_PERIOD_S = 0.005  # NVML sampling period inside the timed region
PROFILE_EVERY = 8  # time the contraction of one step in 8 (at least once for any step count)
POPC_PER_CLK_PER_SM = 16  # 32-bit POPC lanes per clock per SM
FP32_PER_CLK_PER_SM = 128  # FFMA lanes per clock per SM
HBM_FALLBACK_GBS = 6650.0  # recipe fallback when MEASURED_PEAKS.json is absent
BF16_FALLBACK_TFLOPS = 1590.0  # recipe fallback when MEASURED_PEAKS.json is absent
CODES_INT8, CODES_FP4, CODES_BF16X3 = 1, 2, 3  # bconv_tc_codes


def rotation_count(set_bytes: int, l2_bytes: int, minimum: int = ROTATE_MIN) -> int:
    """Input/output sets to rotate through so that together they exceed 1.5 x the L2: a
    step's data has then been evicted by the time the step comes round again."""
    return max(minimum, -(-int(1.5 * l2_bytes) // max(int(set_bytes), 1)))


def timed_step_count(requested: int, est_step_ms: float, seconds: float) -> int:
    """Steps of the timed region: at least `requested`, and enough to fill `seconds` of device
    time at the calibrated step time."""
    fill = int(math.ceil(seconds * 1e3 / max(est_step_ms, 1e-6)))
    return max(int(requested), fill, 1)


def profile_stride(steps: int, every: int = PROFILE_EVERY) -> int:
    """Sampling stride of the contraction timing: every `every`-th step, but at least three
    samples even for a short run."""
    return max(1, min(every, steps // 3))


# ----------------------------------------------------------------------------------------
# ranks
# ----------------------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(
        os.environ.get("LOCAL_RANK", "0"))


def dist_init(backend: str):
    import datetime

    import torch.distributed as dist

    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a float over all ranks (identity for a single process)."""
    import torch
    import torch.distributed as dist

    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def replica_seed(base: int, rank: int) -> int:
    """Each replica draws its own batch; rank 0 uses the workload's own seed."""
    return base + 7919 * rank


# ----------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; no setting is changed)
# ----------------------------------------------------------------------------------------
class ClockSampler:
    """Samples the SM clock and the clock-event reasons every `period_s` between start() and
    stop(), which the caller places around the timed region."""

    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
               "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100}
    REJECT = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")

    def __init__(self, device=None, period_s: float = CLOCK_PERIOD_S):
        self.period = period_s
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        self._h = None
        self._device = device

    def _handle(self, p):
        """The NVML handle of the CUDA device (by UUID, which survives CUDA_VISIBLE_DEVICES)."""
        import torch

        idx = self._device.index if self._device is not None else 0
        try:
            uuid = str(torch.cuda.get_device_properties(idx).uuid)
            return p.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:  # noqa: BLE001 -- fall back to the index
            return p.nvmlDeviceGetHandleByIndex(idx)

    def open(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = self._handle(pynvml)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 -- clocks are reported as unavailable
            self._nvml = None
        return self

    def start(self):
        self.samples, self.reasons = [], 0
        self._stop.clear()
        if self._nvml is None:
            return self
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _run(self):
        p = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(p.nvmlDeviceGetClockInfo(self._h, p.NVML_CLOCK_SM))
                self.reasons |= p.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:  # noqa: BLE001
                pass
            self._stop.wait(self.period)

    def stop(self) -> dict:
        self._stop.set()
        if self._thread:
            self._thread.join()
            self._thread = None
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        names = [k for k, v in self.REASONS.items() if self.reasons & v and k != "gpu_idle"]
        s = self.samples
        return {"sm_mhz": statistics.median(s) if s else None, "sm_max_mhz": self.max_mhz,
                "sm_min_mhz": min(s) if s else None, "reasons": names, "samples": len(s),
                "period_ms": self.period * 1e3, "rejected": [r for r in names if r in self.REJECT]}


# ----------------------------------------------------------------------------------------
# roofline bookkeeping
# ----------------------------------------------------------------------------------------
def kernel_source_digest(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str, sources) -> float | None:
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None
    rec = table.get(f"{kernel}:{workload}")
    if not rec or rec.get("source_digest") != kernel_source_digest(sources):
        return None
    return rec.get("dram_bytes_per_launch")


_TC_COMMON = ["binarized_convolution_b200/csrc/tc_device.cuh", "binarized_convolution_b200/csrc/tc_conv.cuh",
              "binarized_convolution_b200/csrc/common.cuh"]
# the sources each contraction kernel is built from (a change voids its recorded DRAM traffic)
KERNEL_SOURCES = {
    "popc_gemm": ["binarized_convolution_b200/csrc/popc_gemm.cu", "binarized_convolution_b200/csrc/common.cuh"],
    "bw_conv": ["binarized_convolution_b200/csrc/bw_conv.cu", "binarized_convolution_b200/csrc/common.cuh"],
    "tc_conv": ["binarized_convolution_b200/csrc/tc_conv.cu", "binarized_convolution_b200/csrc/tc_bits.cuh"] + _TC_COMMON,
    "tc_conv2": ["binarized_convolution_b200/csrc/tc_conv2.cu", "binarized_convolution_b200/csrc/tc_bits.cuh"] + _TC_COMMON,
    "tc_halo": ["binarized_convolution_b200/csrc/tc_halo.cu"] + _TC_COMMON,
    "tc_halo2": ["binarized_convolution_b200/csrc/tc_halo2.cu"] + _TC_COMMON,
    "tc_fc": ["binarized_convolution_b200/csrc/tc_fc.cu"] + _TC_COMMON,
}
ALGO_KERNEL = {1: "popc_gemm", 2: "bw_conv", 3: "tc_conv"}


def tc_kernel_name(bc, layer, w: synth.Workload) -> str:
    """The tensor-core kernel a layer's plan runs: the e2m1 FC kernel, the rows-staged
    convolution (one SM or SM pairs) or the per-tap convolution (one SM or SM pairs)."""
    pair = layer.cta_mode() == bc.CTA_PAIR
    if w.kind == "fc":
        return "tc_fc" if layer.tc_codes() == CODES_FP4 else ("tc_conv2" if pair else "tc_conv")
    if layer.staging() == bc.STAGING_ROWS:
        return "tc_halo2" if pair else "tc_halo"
    return "tc_conv2" if pair else "tc_conv"


def measured_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


def hbm_peak() -> tuple[float, str]:
    """HBM bandwidth in GB/s: the measured copy bandwidth, else the recipe's fallback."""
    p = measured_peaks()
    if "hbm_gbs" in p:
        return float(p["hbm_gbs"]), f"of measured: copy {float(p['hbm_gbs']):.1f} GB/s"
    return HBM_FALLBACK_GBS, f"of fallback: {HBM_FALLBACK_GBS:.0f} GB/s"


def bf16_peak() -> tuple[float, str]:
    """Dense bf16 TFLOP/s (burst): measured, else the recipe's fallback."""
    p = measured_peaks()
    if "bf16_tflops" in p:
        return float(p["bf16_tflops"]), "of measured"
    return BF16_FALLBACK_TFLOPS, "of fallback"


def tensor_peak() -> tuple[float, str]:
    """Dense int8 tensor-core multiply-accumulates per second, in T: the bf16 burst TFLOP/s x 2
    (the nominal int8/bf16 ratio, 4.5/2.25) / 2 (ops per MAC)."""
    v, src = bf16_peak()
    return v, f"{src}: bf16 burst {v:.1f} TFLOP/s x 2 (int8/bf16 nominal) / 2 ops per MAC"


def derived_peak(w: synth.Workload, sms: int, sm_mhz: float, kernel: str = "", codes: int = 0) -> tuple[float, str, str]:
    """(peak in TOPS of the method's own operations, bound, how it was derived) for the
    contraction's instruction mix (`codes`: the tensor-core operand codes, CODES_*)."""
    if kernel == "tc_conv" and codes == CODES_FP4:
        v, src = bf16_peak()
        # block-scaled fp4 runs at twice the int8 rate (nominal 9 / 4.5 PFLOP/s dense)
        return 2 * v, "tensor", f"{src}: bf16 burst {v:.1f} TFLOP/s x 4 (fp4/bf16 nominal) / 2 ops per MAC"
    if kernel == "tc_conv" and w.op == synth.BINARY_WEIGHTS:
        bf16, src = bf16_peak()
        # bf16 MAC/s = TFLOP/s / 2; each fp32 x (+-1) term costs three bf16 MACs (hi, mid, lo)
        return bf16 / 2 / 3, "tensor", f"{src}: bf16 burst {bf16:.1f} TFLOP/s / 2 ops per MAC / 3 bf16 parts per term"
    if kernel == "tc_conv":
        v, how = tensor_peak()
        return v, "tensor", how
    if w.op == synth.BINARY_WEIGHTS:
        p = sms * FP32_PER_CLK_PER_SM * sm_mhz * 1e6 / 1e12
        return p, "alu", f"{sms} SMs x {FP32_PER_CLK_PER_SM} FP32 lanes/clk x {sm_mhz:.0f} MHz (1 op = 1 signed add)"
    p = sms * POPC_PER_CLK_PER_SM * 32 * sm_mhz * 1e6 / 1e12
    return p, "alu", f"{sms} SMs x {POPC_PER_CLK_PER_SM} POPC/clk x 32 bits x {sm_mhz:.0f} MHz"


def algorithmic_bytes(w: synth.Workload) -> int:
    """Bytes a forward must move at least: the fp32 input read once, the weights as packed
    bits, the fp32 output written once."""
    taps = w.kernel_h * w.kernel_w
    words = (w.in_channels + 31) // 32
    return (w.batch * w.in_h * w.in_w * w.in_channels * 4 + w.out_channels * taps * words * 4
            + w.batch * w.out_h * w.out_w * w.out_channels * 4)


def forward_roofline(w: synth.Workload, step_ms: float, pipe_peak_tops: float) -> dict:
    """The whole step against max(algorithmic bytes / HBM bandwidth, ops / pipe peak)."""
    gbs, hbm_src = hbm_peak()
    b = algorithmic_bytes(w)
    t_bytes = b / (gbs * 1e9)
    t_ops = w.nominal_ops / (pipe_peak_tops * 1e12)
    t_roof = max(t_bytes, t_ops)
    return {"bound": "hbm" if t_bytes >= t_ops else "tensor", "t_roof_us": t_roof * 1e6,
            "t_step_us": step_ms * 1e3, "frac": t_roof / (step_ms * 1e-3), "algorithmic_bytes": b,
            "hbm_peak_gbs": gbs, "hbm_peak_source": hbm_src, "t_bytes_us": t_bytes * 1e6, "t_ops_us": t_ops * 1e6}


# ----------------------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of output pixels
# ----------------------------------------------------------------------------------------
def oracle_sample_rate(w: synth.Workload, inp, target_s: float, rng_seed: int = 0):
    """Times the oracle on output pixels of the workload; returns (TOPS, seconds, pixels, threads)."""
    import oracle

    otype = {synth.XNOR: oracle.ORACLE_XNOR, synth.AND: oracle.ORACLE_AND,
             synth.BINARY_WEIGHTS: oracle.ORACLE_BINARY_WEIGHTS}[w.op]
    rows_total = w.batch * w.out_h * w.out_w
    ops_per_row = w.nominal_ops / rows_total
    rng = np.random.default_rng(rng_seed)

    def run(n, repeats=1):
        # n rows (a workload smaller than the sample is run `repeats` times over)
        rows = np.sort(rng.choice(rows_total, size=min(n, rows_total), replace=False)).astype(np.int64)
        kw = dict(type=otype, scale=inp.scale, bias=inp.bias, in_scale=inp.in_scale, in_bias=inp.in_bias,
                  use_beta=w.use_beta, relu=w.relu)
        t0 = time.perf_counter()
        for _ in range(repeats):
            if w.kind == "fc":
                oracle.fc(inp.x, inp.wbits, rows=rows, **kw)
            else:
                oracle.conv(inp.x, inp.wbits, stride=(w.stride_y, w.stride_x), pixels=rows, **kw)
        return time.perf_counter() - t0, len(rows) * repeats

    threads = oracle.num_threads()
    n = max(threads, 8)
    dt, n = run(n)
    while dt < 0.5 and n < rows_total and dt < target_s:
        n = min(rows_total, n * 4)
        dt, n = run(n)
    want = max(1, int(n * target_s / max(dt, 1e-6)))
    if want <= rows_total:
        dt, n = run(want)
    else:
        dt, n = run(rows_total, repeats=max(1, want // rows_total))
    return n * ops_per_row / dt / 1e12, dt, n, threads


def simd_baseline_record(w: synth.Workload, inp, seconds: float) -> dict:
    """The vectorised CPU baseline (cpu_simd/: bit-packed XOR / AND + popcount on AVX-512 or AVX2,
    OpenMP) on the whole workload, repeated for about `seconds`."""
    import binarized_convolution_b200 as bc
    import cpu_simd

    t = {synth.XNOR: cpu_simd.XNOR, synth.AND: cpu_simd.AND, synth.BINARY_WEIGHTS: cpu_simd.BINARY_WEIGHTS}[w.op]
    packed = bc.bconv_pack_bits(inp.wbits.reshape(-1, w.in_channels)).reshape(*inp.wbits.shape[:3], -1)
    kw = dict(type=t, scale=inp.scale, bias=inp.bias, in_scale=inp.in_scale, in_bias=inp.in_bias,
              use_beta=w.use_beta, relu=w.relu)

    def run():
        if w.kind == "fc":
            cpu_simd.fc(inp.x, packed, **kw)
        else:
            cpu_simd.conv(inp.x, packed, stride=(w.stride_y, w.stride_x), **kw)

    run()  # first call builds and warms up
    t0 = time.perf_counter()
    run()
    one = time.perf_counter() - t0
    reps = max(1, int(seconds / max(one, 1e-6)))
    t0 = time.perf_counter()
    for _ in range(reps):
        run()
    dt = time.perf_counter() - t0
    return {"value": w.nominal_ops * reps / dt / 1e12, "unit": UNIT, "cores": cpu_simd.num_threads(),
            "kind": f"simd ({cpu_simd.ISA_NAMES[cpu_simd.best_isa()]})", "ms_per_step": dt * 1e3 / reps,
            "sample": f"the whole workload x {reps}, {dt:.1f} s"}


def cpu_baseline_record(w: synth.Workload, inp, seconds: float) -> dict:
    v, dt, n, thr = oracle_sample_rate(w, inp, target_s=seconds)
    return {"value": v, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": f"{n} output rows of {w.batch * w.out_h * w.out_w} (all {w.out_channels} channels each; "
                      f"the whole workload repeated when it is smaller), {dt:.1f} s"}


# ----------------------------------------------------------------------------------------
# native arm
# ----------------------------------------------------------------------------------------
def _make_layer(bc, w, inp, args, in_terms=True):
    layer_kw = dict(op=w.op, scale=inp.scale, bias=inp.bias, use_beta=w.use_beta, relu=w.relu)
    if in_terms:
        layer_kw.update(in_scale=inp.in_scale, in_bias=inp.in_bias)
    if w.kind == "fc":
        layer = bc.BinaryFC(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, wbits=inp.wbits, **layer_kw)
    else:
        layer = bc.BinaryConv2d(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, (w.kernel_h, w.kernel_w),
                                (w.stride_y, w.stride_x), wbits=inp.wbits, **layer_kw)
    if args.algo != "auto":
        layer.set_algo({"popc": bc.ALGO_POPC, "tcgen05": bc.ALGO_TCGEN05, "simt_f32": bc.ALGO_SIMT_F32}[args.algo])
    return layer


def measure_workload(args, w: synth.Workload, device, bits_io: bool = False, cpu_seconds: float = 0.0) -> dict:
    """Time one workload (every rank takes the same collective steps); returns its record."""
    import torch

    import binarized_convolution_b200 as bc

    rank, world, _ = dist_env()
    inp = synth.make_inputs(w, seed=replica_seed(w.seed, rank))
    layer = _make_layer(bc, w, inp, args)
    if w.kind == "fc":
        prof_begin, prof_end, prof_stride = bc.bfc_profile_begin, bc.bfc_profile_end, bc.bfc_profile_stride
    else:
        prof_begin, prof_end, prof_stride = bc.bconv_profile_begin, bc.bconv_profile_end, bc.bconv_profile_stride
    out_shape = layer.out_dims
    l2_bytes = getattr(torch.cuda.get_device_properties(device), "L2_cache_size", 0) or L2_BYTES
    set_bytes = inp.x.nbytes + int(np.prod(out_shape)) * 4
    bits_set_bytes = 2 * ((int(np.prod(out_shape)) + 31) // 32 * 4 + int(np.prod(out_shape[:-1])) * 4)
    ROTATE = rotation_count(set_bytes, l2_bytes)
    ROTATE_BITS = rotation_count(bits_set_bytes, l2_bytes)
    xs = [torch.from_numpy(inp.x).to(device)]
    for r in range(1, min(ROTATE, ROTATE_BITS) if bits_io else ROTATE):
        xs.append(torch.from_numpy(synth.make_batch(w, seed=replica_seed(w.seed, rank) * 1000 + r)).to(device))
    stream = torch.cuda.current_stream(device)
    if bits_io:
        # A middle layer of a chain of identical layers: it reads the bit-packed output of the
        # previous one (made here by the same layer with fp32 input) and writes its own for the
        # next, whose input terms are this layer's.  The timed layer has no input terms.
        if w.kind == "fc" or w.op == synth.BINARY_WEIGHTS or w.in_channels != w.out_channels or \
                (w.stride_y, w.stride_x) != (1, 1):
            raise SystemExit("--io bits needs an XNOR/AND convolution with in = out channels and stride 1")
        layer.set_output_terms(inp.in_scale, inp.in_bias)
        feeds = [layer.forward_to_bits(x) for x in xs]
        del xs
        for r in range(ROTATE, ROTATE_BITS):  # enough sets that one step's data has left L2
            x = torch.from_numpy(synth.make_batch(w, seed=replica_seed(w.seed, rank) * 1000 + r)).to(device)
            feeds.append(layer.forward_to_bits(x))
            del x
        torch.cuda.synchronize(device)
        layer.close()
        layer = _make_layer(bc, w, inp, args, in_terms=False)
        layer.set_output_terms(inp.in_scale, inp.in_bias)
        bshape, ashape = layer.bits_shape()
        outs = [(torch.empty(bshape, dtype=torch.int32, device=device), torch.empty(ashape, device=device))
                for _ in range(ROTATE_BITS)]
        n_sets = ROTATE_BITS

        def fwd(i):
            xb, xa = feeds[i % ROTATE_BITS]
            ob, oa = outs[i % ROTATE_BITS]
            layer.forward_io(x_bits=xb, x_a=xa if w.use_beta else None, out_bits=ob, out_a=oa)
    else:
        ys = [torch.empty(out_shape, dtype=torch.float32, device=device) for _ in range(ROTATE)]
        n_sets = ROTATE

        def fwd(i):
            layer.forward_into(xs[i % ROTATE], ys[i % ROTATE])

    for i in range(args.warmup):
        fwd(i)
    layer.sync_status(stream.cuda_stream)
    torch.cuda.synchronize(device)

    # calibration: the step count that fills the timed region (the same on every rank)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_cal = max(2 * n_sets, 8)
    ev0.record(stream)
    for i in range(n_cal):
        fwd(i)
    ev1.record(stream)
    torch.cuda.synchronize(device)
    est_ms = max_over_ranks(ev0.elapsed_time(ev1) / n_cal, device)
    steps = timed_step_count(args.steps, est_ms, args.seconds)
    every = profile_stride(steps)

    clocks = ClockSampler(device).open()
    prof_begin(layer.handle, steps // every + 2)
    prof_stride(layer.handle, every)
    barrier(device)
    torch.cuda.synchronize(device)
    clocks.start()
    ev0.record(stream)
    for i in range(steps):
        fwd(i)
    ev1.record(stream)
    torch.cuda.synchronize(device)
    clock_info = clocks.stop()
    barrier(device)
    elapsed_ms = ev0.elapsed_time(ev1)
    kern_ms, kern_n = prof_end(layer.handle)
    layer.sync_status(stream.cuda_stream)
    elapsed_ms = max_over_ranks(elapsed_ms, device)
    kern_ms_max = max_over_ranks(kern_ms / max(kern_n, 1), device)

    ops_step = w.nominal_ops
    value = ops_step * steps * world / (elapsed_ms * 1e-3) / 1e12
    images_s = w.batch * steps * world / (elapsed_ms * 1e-3)
    step_ms = elapsed_ms / steps

    # roofline of the contraction kernel: nominal ops of one launch / its mean event time
    props = torch.cuda.get_device_properties(device)
    sms = props.multi_processor_count
    max_mhz = clock_info.get("sm_max_mhz") or 1965.0
    kname = ALGO_KERNEL[layer.effective_algo()]
    codes = layer.tc_codes() if kname == "tc_conv" else 0
    kernel = tc_kernel_name(bc, layer, w) if kname == "tc_conv" else kname
    peak, bound, how = derived_peak(w, sms, max_mhz, kname, codes)
    achieved = ops_step / (kern_ms_max * 1e-3) / 1e12
    # the captured traffic is that of the library's own choice of spread and codes
    traffic = (measured_traffic(kernel, w.name, KERNEL_SOURCES[kernel])
               if args.cta == "auto" and args.codes == "auto" and not bits_io else None)
    roof = {"bound": bound, "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
            "traffic": traffic, "kernel": kernel, "kernel_ms": kern_ms_max,
            "kernel_launches_timed": kern_n, "timed_every": every,
            "peak_source": how if bound == "tensor" else f"derived: {how}"}
    if kname == "tc_conv":
        roof["spread"] = {bc.CTA_SINGLE: "one SM per tile", bc.CTA_PAIR: "SM pairs (cta_group::2)"}.get(
            layer.cta_mode(), "?")
        roof["codes"] = {CODES_INT8: "int8", CODES_FP4: "e2m1 (fp4), kind::mxf4",
                         CODES_BF16X3: "bf16 x3"}.get(codes, "?")
        if w.kind != "fc":
            roof["staging"] = {bc.STAGING_PER_TAP: "per tap", bc.STAGING_ROWS: "rows-staged",
                               bc.STAGING_INPUT: "fp32 input split in shared memory (no pack kernel)"}.get(
                layer.staging(), "?")
    sm_mhz = clock_info.get("sm_mhz")
    if sm_mhz and bound == "alu":
        p_obs, _, _ = derived_peak(w, sms, sm_mhz, kname, codes)
        roof["frac_at_observed_clock"] = achieved / p_obs
    if sm_mhz and max_mhz:
        roof["frac_at_observed_clock_scaled"] = achieved / (peak * sm_mhz / max_mhz)

    rec = {
        "workload": w.name, "value": value, "unit": UNIT, "steps": steps, "steps_requested": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "images_per_s": images_s,
        "dtype": ("bf16x3 / f32" if (kname == "tc_conv" and w.op == synth.BINARY_WEIGHTS) else
                  "e2m1 (fp4) codes / f32" if codes == CODES_FP4 else
                  {"popc_gemm": "u32 bits / int32", "tc_conv": "int8 codes / int32", "bw_conv": "f32"}[kname]),
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "global_batch": w.batch * world,
                   "in": [w.in_h, w.in_w, w.in_channels], "out_channels": w.out_channels,
                   "kernel": [w.kernel_h, w.kernel_w], "stride": [w.stride_y, w.stride_x], "op": w.op,
                   "beta": w.use_beta, "relu": w.relu, "input_terms": w.in_terms,
                   "parallelism": f"replicas x{world}", "algo": kname,
                   "io": "bit-packed in and out (chain middle layer)" if bits_io else "fp32 in and out",
                   "l2": (f"inputs larger than L2: {n_sets} rotating input/output sets, "
                          f"{n_sets * (bits_set_bytes if bits_io else set_bytes) / 1e6:.0f} MB > "
                          f"{l2_bytes / 1e6:.0f} MB L2")},
        "roofline": roof,
        "forward_roofline": forward_roofline(w, step_ms, peak),
        "clocks": clock_info,
        "gpu_launches": layer.launches_per_forward() * steps,
        "launches_per_step": layer.launches_per_forward(),
    }

    # end to end through the C ABI with page-locked host buffers
    if not args.no_e2e and not bits_io:
        hin = torch.from_numpy(inp.x).pin_memory()
        hout = torch.empty(out_shape, dtype=torch.float32).pin_memory()
        fwd_host = bc.bfc_forward_host if w.kind == "fc" else bc.bconv_forward_host
        for _ in range(2):
            fwd_host(layer.handle, hin.data_ptr(), hout.data_ptr(), stream.cuda_stream)
        t0 = time.perf_counter()
        fwd_host(layer.handle, hin.data_ptr(), hout.data_ptr(), stream.cuda_stream)
        one = time.perf_counter() - t0
        e2e_steps = max(20, min(2000, int(args.e2e_seconds / max(one, 1e-6))))
        e2e_steps = int(max_over_ranks(e2e_steps, device))
        barrier(device)
        torch.cuda.synchronize(device)
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            fwd_host(layer.handle, hin.data_ptr(), hout.data_ptr(), stream.cuda_stream)
        t_e2e = time.perf_counter() - t0
        t_e2e = max_over_ranks(t_e2e, device)
        rec["e2e"] = {"value": ops_step * e2e_steps * world / t_e2e / 1e12, "unit": UNIT,
                      "h2d_bytes_per_step": int(hin.numel() * 4), "d2h_bytes_per_step": int(hout.numel() * 4),
                      "steps": e2e_steps, "ms_per_step": t_e2e * 1e3 / e2e_steps,
                      "images_per_s": w.batch * e2e_steps * world / t_e2e,
                      "api": "bfc_forward_host" if w.kind == "fc" else "bconv_forward_host"}
        del hin, hout
    layer.close()
    fwd = None  # drop the closure's references to the rotating buffers before the next workload

    if rank == 0 and world == 1 and cpu_seconds > 0:
        rec["cpu_baseline"] = cpu_baseline_record(w, inp, cpu_seconds)
        rec["cpu_simd_baseline"] = simd_baseline_record(w, inp, args.simd_seconds)
    torch.cuda.empty_cache()
    return rec


def run_native(args):
    import torch

    import binarized_convolution_b200 as bc

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init("nccl")
    bc.bconv_set_cta_mode({"auto": bc.CTA_AUTO, "single": bc.CTA_SINGLE, "pair": bc.CTA_PAIR}[args.cta])
    bc.bconv_set_tc_codes({"auto": bc.CODES_AUTO, "int8": bc.CODES_INT8, "fp4": bc.CODES_FP4}[args.codes])

    bits_io = args.io == "bits"
    if args.workload == "all" and not bits_io:
        names = list(synth.WORKLOAD_ORDER)
        headline = DEFAULT_WORKLOAD
    else:
        key = DEFAULT_WORKLOAD if args.workload == "all" else args.workload
        w0 = synth.workload(int(key) if key.isdigit() else key)
        names, headline = [w0.name], w0.name
    want_cpu = not args.no_cpu_baseline
    recs = {}
    for name in names:
        cpu_s = (args.cpu_seconds if name == headline else args.cpu_seconds_other) if want_cpu else 0.0
        recs[name] = measure_workload(args, synth.workload(name), device, bits_io=bits_io, cpu_seconds=cpu_s)

    h = recs[headline]
    result = {
        "metric": METRIC, "value": h["value"], "unit": UNIT, "n_gpus": world, "steps": h["steps"],
        "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": h["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": h["dtype"],
        "data": "synthetic (seeded N(0,1) inputs, Bernoulli weight bits)",
        "config": h["config"], "images_per_s": h["images_per_s"], "roofline": h["roofline"],
        "forward_roofline": h["forward_roofline"], "clocks": h["clocks"], "gpu_launches": h["gpu_launches"],
    }
    for k in ("e2e", "cpu_baseline", "cpu_simd_baseline"):
        if k in h:
            result[k] = h[k]
    if len(recs) > 1:
        result["workloads"] = {
            n: {k: r[k] for k in ("value", "ms_per_step", "steps", "images_per_s", "dtype", "roofline",
                                  "forward_roofline", "clocks", "gpu_launches", "e2e", "cpu_baseline",
                                  "cpu_simd_baseline") if k in r}
            for n, r in recs.items()}
        result["total_gpu_launches"] = sum(r["gpu_launches"] for r in recs.values())
    if rank == 0:
        print(json.dumps(result), flush=True)
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()


# ----------------------------------------------------------------------------------------
# reference arm: the oracle, timed as it stands
# ----------------------------------------------------------------------------------------
def run_reference(args, w: synth.Workload):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    inp = synth.make_inputs(w)
    total_steps = args.steps + args.warmup
    per_step_s = min(10.0, args.reference_seconds / max(total_steps, 1))
    rate, dt, n, thr = oracle_sample_rate(w, inp, target_s=per_step_s)  # calibrates the sample size
    import oracle

    otype = {synth.XNOR: oracle.ORACLE_XNOR, synth.AND: oracle.ORACLE_AND,
             synth.BINARY_WEIGHTS: oracle.ORACLE_BINARY_WEIGHTS}[w.op]
    rows_total = w.batch * w.out_h * w.out_w
    ops_per_row = w.nominal_ops / rows_total
    rng = np.random.default_rng(1)
    kw = dict(type=otype, scale=inp.scale, bias=inp.bias, in_scale=inp.in_scale, in_bias=inp.in_bias,
              use_beta=w.use_beta, relu=w.relu)

    def step():
        rows = np.sort(rng.choice(rows_total, size=n, replace=False)).astype(np.int64)
        if w.kind == "fc":
            oracle.fc(inp.x, inp.wbits, rows=rows, **kw)
        else:
            oracle.conv(inp.x, inp.wbits, stride=(w.stride_y, w.stride_x), pixels=rows, **kw)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    t = time.perf_counter() - t0
    value = n * ops_per_row * args.steps / t / 1e12
    result = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) inputs, Bernoulli weight bits)",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "global_batch": w.batch * world,
                   "parallelism": "rank 0 only (CPU oracle)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": f"each step: {n} of {rows_total} output rows (all {w.out_channels} channels)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20, help="minimum timed steps per workload")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--seconds", type=float, default=TIMED_SECONDS,
                    help="device time each workload's timed region fills (at least --steps steps)")
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="all", help="all (headline + the other four), a name or an index 0-4")
    ap.add_argument("--algo", choices=["auto", "popc", "tcgen05", "simt_f32"], default="auto",
                    help="kernel family of the contraction (auto = the library's choice)")
    ap.add_argument("--cta", choices=["auto", "single", "pair"], default="auto",
                    help="tensor-core contraction on one SM per tile or on SM pairs (auto = the library's choice)")
    ap.add_argument("--codes", choices=["auto", "int8", "fp4"], default="auto",
                    help="operand codes of the XNOR/AND tensor-core path (auto = the library's choice)")
    ap.add_argument("--io", choices=["f32", "bits"], default="f32",
                    help="bits: time a middle layer of a chain (bit-packed input and output)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-seconds", type=float, default=1.0, help="host time of each e2e measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle time of the headline's cpu_baseline")
    ap.add_argument("--cpu-seconds-other", type=float, default=3.0,
                    help="oracle time of the other workloads' cpu_baseline")
    ap.add_argument("--simd-seconds", type=float, default=2.0,
                    help="time of each workload's vectorised CPU baseline (cpu_simd_baseline)")
    ap.add_argument("--reference-seconds", type=float, default=120.0, help="oracle time budget of --impl reference")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload != "all":
        key = int(args.workload) if args.workload.isdigit() else args.workload
        try:
            synth.workload(key)
        except (KeyError, IndexError):
            ap.error(f"unknown workload {args.workload}")
    if args.impl == "reference":
        key = DEFAULT_WORKLOAD if args.workload == "all" else args.workload
        run_reference(args, synth.workload(int(key) if key.isdigit() else key))
    else:
        run_native(args)


if __name__ == "__main__":
    main()
