"""Throughput of the binary convolution on B200: one JSON line per run.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload NAME|INDEX] [--io f32|bits] [--no-e2e] [--no-cpu-baseline]

A step is one forward of the layer (input transform + pack + A, beta, contraction and
epilogue) over one batch of the workload: by default XNOR with beta scaling and input terms,
batch 16, 56x56, 256 -> 256 channels, 3x3, ReLU.  ``value`` is nominal bit multiply-
accumulates (every window tap, 1 op = 1 bit MAC) per second over all ranks, with inputs
resident in HBM; input/output buffer sets rotate so that one step's data is not in L2 when it
is next used (at least four sets and together more than 1.5 x the L2: 411 MB for the default
workload).  ``e2e`` is the same metric through
bconv_forward_host with page-locked host buffers (host-to-device copy, forward,
device-to-host copy inside every step).  Multi-GPU runs (torchrun) are independent replicas
with a batch each (weak scaling); their time is the maximum over ranks.

``--io bits`` times the same layer as the middle of a chain of such layers instead: it reads
the bit-packed output of the previous layer (sign bits and A) and writes its own for the next
(bconv_forward_io); the input terms move to the previous layer's epilogue.

``--impl reference`` times the oracle (the plain double-precision CPU loops) on the same
workload, each step a bounded sample of output pixels, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from binarized_convolution_b200 import synth  # noqa: E402

DEFAULT_WORKLOAD = "xnor_beta_n16_56x56_c256_k256_3x3"
METRIC = "binary conv TOPS (1 op = 1 bit MAC) and images/s on 1 B200; % of roofline"
UNIT = "TOPS"
ROTATE_MIN = 4
L2_BYTES = 126 * 1024 * 1024  # B200 L2 (the device property is used when available)


def rotation_count(set_bytes: int, l2_bytes: int, minimum: int = ROTATE_MIN) -> int:
    """Input/output sets to rotate through so that together they exceed 1.5 x the L2: a
    step's data has then been evicted by the time the step comes round again."""
    return max(minimum, -(-int(1.5 * l2_bytes) // max(int(set_bytes), 1)))
PROFILE_EVERY = 8  # time the contraction of one step in 8 (at least 1 for any --steps)
POPC_PER_CLK_PER_SM = 16  # 32-bit POPC lanes per clock per SM
FP32_PER_CLK_PER_SM = 128  # FFMA lanes per clock per SM


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
    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
               "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100}

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None

    def start(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self._h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 -- clocks are reported as unavailable
            self._nvml = None
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

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join()
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [k for k, v in self.REASONS.items() if self.reasons & v and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


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


KERNEL_SOURCES = {
    "popc_gemm": ["binarized_convolution_b200/csrc/popc_gemm.cu", "binarized_convolution_b200/csrc/common.cuh"],
    "bw_conv": ["binarized_convolution_b200/csrc/bw_conv.cu", "binarized_convolution_b200/csrc/common.cuh"],
    "tc_conv": ["binarized_convolution_b200/csrc/tc_conv.cu", "binarized_convolution_b200/csrc/tc_conv2.cu",
                "binarized_convolution_b200/csrc/tc_conv.cuh", "binarized_convolution_b200/csrc/tc_device.cuh",
                "binarized_convolution_b200/csrc/tc_bits.cuh"],
}
ALGO_KERNEL = {1: "popc_gemm", 2: "bw_conv", 3: "tc_conv"}
CODES_FP4 = 2  # bconv_tc_codes: e2m1 operand codes
BF16_FALLBACK_TFLOPS = 1590.0  # recipe fallback when MEASURED_PEAKS.json is absent


def measured_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


def tensor_peak() -> tuple[float, str]:
    """Dense int8 tensor-core multiply-accumulates per second, in T: the measured bf16 burst
    TFLOP/s x 2 (the nominal int8/bf16 ratio, 4.5/2.25) / 2 (ops per MAC)."""
    p = measured_peaks()
    if "bf16_tflops" in p:
        v = float(p["bf16_tflops"])
        return v, f"of measured: bf16 burst {v:.1f} TFLOP/s x 2 (int8/bf16 nominal) / 2 ops per MAC"
    return BF16_FALLBACK_TFLOPS, "of fallback: 1590 TFLOP/s bf16 x 2 / 2 ops per MAC"


def derived_peak(w: synth.Workload, sms: int, sm_mhz: float, kernel: str = "", codes: int = 0) -> tuple[float, str, str]:
    """(peak in TOPS of the method's own operations, bound, how it was derived) for the
    contraction's instruction mix (`codes`: the tensor-core operand codes, CODES_*)."""
    if kernel == "tc_conv" and codes == CODES_FP4:
        v, how = tensor_peak()
        # block-scaled fp4 runs at twice the int8 rate (nominal 9 / 4.5 PFLOP/s dense)
        return 2 * v, "tensor", how.replace("x 2 (int8/bf16 nominal)", "x 4 (fp4/bf16 nominal)")
    if kernel == "tc_conv" and w.op == synth.BINARY_WEIGHTS:
        p = measured_peaks()
        bf16 = float(p.get("bf16_tflops", BF16_FALLBACK_TFLOPS))
        src = "of measured" if "bf16_tflops" in p else "of fallback"
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

    def run(n):
        rows = np.sort(rng.choice(rows_total, size=min(n, rows_total), replace=False)).astype(np.int64)
        kw = dict(type=otype, scale=inp.scale, bias=inp.bias, in_scale=inp.in_scale, in_bias=inp.in_bias,
                  use_beta=w.use_beta, relu=w.relu)
        t0 = time.perf_counter()
        if w.kind == "fc":
            oracle.fc(inp.x, inp.wbits, rows=rows, **kw)
        else:
            oracle.conv(inp.x, inp.wbits, stride=(w.stride_y, w.stride_x), pixels=rows, **kw)
        return time.perf_counter() - t0, len(rows)

    threads = oracle.num_threads()
    n = max(threads, 8)
    dt, n = run(n)
    while dt < 0.5 and n < rows_total:
        n = min(rows_total, n * 4)
        dt, n = run(n)
    want = int(n * target_s / max(dt, 1e-6))
    want = max(1, min(rows_total, want))
    dt, n = run(want)
    return n * ops_per_row / dt / 1e12, dt, n, threads


# ----------------------------------------------------------------------------------------
# native arm
# ----------------------------------------------------------------------------------------
def run_native(args, w: synth.Workload):
    import torch

    import binarized_convolution_b200 as bc

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init("nccl")

    inp = synth.make_inputs(w, seed=replica_seed(w.seed, rank))
    bc.bconv_set_cta_mode({"auto": bc.CTA_AUTO, "single": bc.CTA_SINGLE, "pair": bc.CTA_PAIR}[args.cta])
    bc.bconv_set_tc_codes({"auto": bc.CODES_AUTO, "int8": bc.CODES_INT8, "fp4": bc.CODES_FP4}[args.codes])
    layer_kw = dict(op=w.op, scale=inp.scale, bias=inp.bias, in_scale=inp.in_scale, in_bias=inp.in_bias,
                    use_beta=w.use_beta, relu=w.relu)
    if w.kind == "fc":
        layer = bc.BinaryFC(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, wbits=inp.wbits, **layer_kw)
        prof_begin, prof_end, prof_stride = bc.bfc_profile_begin, bc.bfc_profile_end, bc.bfc_profile_stride
    else:
        layer = bc.BinaryConv2d(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, (w.kernel_h, w.kernel_w),
                                (w.stride_y, w.stride_x), wbits=inp.wbits, **layer_kw)
        prof_begin, prof_end, prof_stride = bc.bconv_profile_begin, bc.bconv_profile_end, bc.bconv_profile_stride
    if args.algo != "auto":
        layer.set_algo({"popc": bc.ALGO_POPC, "tcgen05": bc.ALGO_TCGEN05, "simt_f32": bc.ALGO_SIMT_F32}[args.algo])
    out_shape = layer.out_dims
    l2_bytes = getattr(torch.cuda.get_device_properties(device), "L2_cache_size", 0) or L2_BYTES
    set_bytes = inp.x.nbytes + int(np.prod(out_shape)) * 4
    bits_set_bytes = 2 * ((int(np.prod(out_shape)) + 31) // 32 * 4 + int(np.prod(out_shape[:-1])) * 4)
    ROTATE = rotation_count(set_bytes, l2_bytes)
    ROTATE_BITS = rotation_count(bits_set_bytes, l2_bytes)
    xs = [torch.from_numpy(inp.x).to(device)]
    for r in range(1, min(ROTATE, ROTATE_BITS) if args.io == "bits" else ROTATE):
        xs.append(torch.from_numpy(synth.make_batch(w, seed=replica_seed(w.seed, rank) * 1000 + r)).to(device))
    stream = torch.cuda.current_stream(device)
    bits_io = args.io == "bits"
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
        layer = bc.BinaryConv2d(w.batch, w.in_h, w.in_w, w.in_channels, w.out_channels, (w.kernel_h, w.kernel_w),
                                (w.stride_y, w.stride_x), wbits=inp.wbits, op=w.op, scale=inp.scale, bias=inp.bias,
                                use_beta=w.use_beta, relu=w.relu)
        if args.algo != "auto":
            layer.set_algo({"popc": bc.ALGO_POPC, "tcgen05": bc.ALGO_TCGEN05}[args.algo])
        layer.set_output_terms(inp.in_scale, inp.in_bias)
        bshape, ashape = layer.bits_shape()
        outs = [(torch.empty(bshape, dtype=torch.int32, device=device), torch.empty(ashape, device=device))
                for _ in range(ROTATE_BITS)]

        def fwd(i):
            xb, xa = feeds[i % ROTATE_BITS]
            ob, oa = outs[i % ROTATE_BITS]
            layer.forward_io(x_bits=xb, x_a=xa if w.use_beta else None, out_bits=ob, out_a=oa)
    else:
        ys = [torch.empty(out_shape, dtype=torch.float32, device=device) for _ in range(ROTATE)]

        def fwd(i):
            layer.forward_into(xs[i % ROTATE], ys[i % ROTATE])

    for i in range(args.warmup):
        fwd(i)
    layer.sync_status(stream.cuda_stream)
    torch.cuda.synchronize(device)

    clocks = ClockSampler(local).start()
    # the contraction of every PROFILE_EVERY-th step is timed with an event pair on the
    # library's stream; the pairs serialise the stream around it, so they stay sparse
    prof_begin(layer.handle, args.steps)
    prof_stride(layer.handle, PROFILE_EVERY)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    ev0.record(stream)
    for i in range(args.steps):
        fwd(i)
    ev1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clock_info = clocks.stop()
    elapsed_ms = ev0.elapsed_time(ev1)
    kern_ms, kern_n = prof_end(layer.handle)
    layer.sync_status(stream.cuda_stream)
    elapsed_ms = max_over_ranks(elapsed_ms, device)
    kern_ms_max = max_over_ranks(kern_ms / max(kern_n, 1), device)

    ops_step = w.nominal_ops
    total_ops = ops_step * args.steps * world
    value = total_ops / (elapsed_ms * 1e-3) / 1e12
    images_s = w.batch * args.steps * world / (elapsed_ms * 1e-3)

    # roofline of the contraction kernel: nominal ops of one launch / its mean event time
    props = torch.cuda.get_device_properties(device)
    sms = props.multi_processor_count
    max_mhz = clock_info.get("sm_max_mhz") or 1965.0
    kname = ALGO_KERNEL[layer.effective_algo()]
    codes = layer.tc_codes() if kname == "tc_conv" else 0
    peak, bound, how = derived_peak(w, sms, max_mhz, kname, codes)
    achieved = ops_step / (kern_ms_max * 1e-3) / 1e12
    # the captured traffic is that of the library's own choice of spread and codes
    traffic = (measured_traffic(kname, w.name, KERNEL_SOURCES[kname])
               if args.cta == "auto" and args.codes == "auto" else None)
    roof = {"bound": bound, "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
            "traffic": traffic, "kernel": kname, "kernel_ms": kern_ms_max,
            "kernel_launches_timed": kern_n, "timed_every": PROFILE_EVERY,
            "peak_source": how if bound == "tensor" else f"derived: {how}"}
    if kname == "tc_conv":
        roof["spread"] = {bc.CTA_SINGLE: "one SM per tile", bc.CTA_PAIR: "SM pairs (cta_group::2)"}.get(
            layer.cta_mode(), "?")
        roof["codes"] = {bc.CODES_INT8: "int8", bc.CODES_FP4: "e2m1 (fp4), kind::mxf4",
                         bc.CODES_BF16X3: "bf16 x3"}.get(codes, "?")
    sm_mhz = clock_info.get("sm_mhz")
    if sm_mhz and bound == "alu":
        p_obs, _, _ = derived_peak(w, sms, sm_mhz, kname, codes)
        roof["frac_at_observed_clock"] = achieved / p_obs
    try:
        probe = 0 if kname == "popc_gemm" else None
        if probe is not None and rank == 0:
            ops_s, mhz = bc.bconv_measure_peak(probe)
            roof["probe_peak"] = ops_s / 1e12
            roof["probe_sm_mhz"] = mhz
    except Exception as e:  # noqa: BLE001
        roof["probe_peak"] = f"unavailable: {e}"

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("bf16x3 / f32" if (kname == "tc_conv" and w.op == synth.BINARY_WEIGHTS) else
                  "e2m1 (fp4) codes / f32" if codes == CODES_FP4 else
                  {"popc_gemm": "u32 bits / int32", "tc_conv": "int8 codes / int32", "bw_conv": "f32"}[kname]),
        "data": "synthetic (seeded N(0,1) inputs, Bernoulli weight bits)",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "global_batch": w.batch * world,
                   "in": [w.in_h, w.in_w, w.in_channels], "out_channels": w.out_channels,
                   "kernel": [w.kernel_h, w.kernel_w], "stride": [w.stride_y, w.stride_x], "op": w.op,
                   "beta": w.use_beta, "relu": w.relu, "input_terms": w.in_terms,
                   "parallelism": f"replicas x{world}", "algo": kname,
                   "io": "bit-packed in and out (chain middle layer)" if bits_io else "fp32 in and out",
                   "l2": (f"{ROTATE} rotating input/output sets, {ROTATE * set_bytes / 1e6:.0f} MB > "
                          f"{l2_bytes / 1e6:.0f} MB L2")
                   if not bits_io else
                   f"{ROTATE_BITS} rotating bit-packed input/output sets, {ROTATE_BITS * bits_set_bytes / 1e6:.0f}"
                   f" MB > {l2_bytes / 1e6:.0f} MB L2"},
        "images_per_s": images_s,
        "roofline": roof,
        "clocks": clock_info,
        "gpu_launches": layer.launches_per_forward() * args.steps,
    }

    # end to end through the C ABI with page-locked host buffers
    if not args.no_e2e and not bits_io:
        e2e_steps = max(3, min(args.steps, 20))
        hin = torch.from_numpy(inp.x).pin_memory()
        hout = torch.empty(out_shape, dtype=torch.float32).pin_memory()
        fwd_host = bc.bfc_forward_host if w.kind == "fc" else bc.bconv_forward_host
        for _ in range(2):
            fwd_host(layer.handle, hin.data_ptr(), hout.data_ptr(), stream.cuda_stream)
        barrier(device)
        torch.cuda.synchronize(device)
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            fwd_host(layer.handle, hin.data_ptr(), hout.data_ptr(), stream.cuda_stream)
        t_e2e = time.perf_counter() - t0
        t_e2e = max_over_ranks(t_e2e, device)
        result["e2e"] = {"value": ops_step * e2e_steps * world / t_e2e / 1e12, "unit": UNIT,
                         "h2d_bytes_per_step": int(hin.numel() * 4), "d2h_bytes_per_step": int(hout.numel() * 4),
                         "steps": e2e_steps, "ms_per_step": t_e2e * 1e3 / e2e_steps,
                         "api": "bfc_forward_host" if w.kind == "fc" else "bconv_forward_host"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, n, thr = oracle_sample_rate(w, inp, target_s=args.cpu_seconds)
        result["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": thr, "kind": "oracle",
                                  "sample": f"{n} of {w.batch * w.out_h * w.out_w} output rows (all {w.out_channels} "
                                            f"channels each), {dt:.1f} s"}
    layer.close()
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
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--algo", choices=["auto", "popc", "tcgen05", "simt_f32"], default="auto",
                    help="kernel family of the contraction (auto = the library's choice)")
    ap.add_argument("--cta", choices=["auto", "single", "pair"], default="auto",
                    help="tensor-core contraction on one SM per tile or on SM pairs (auto = the library's choice)")
    ap.add_argument("--codes", choices=["auto", "int8", "fp4"], default="auto",
                    help="operand codes of the XNOR/AND tensor-core path (auto = the library's choice)")
    ap.add_argument("--io", choices=["f32", "bits"], default="f32",
                    help="bits: time a middle layer of a chain (bit-packed input and output)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle time of the cpu_baseline sample")
    ap.add_argument("--reference-seconds", type=float, default=120.0, help="oracle time budget of --impl reference")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    key = int(args.workload) if args.workload.isdigit() else args.workload
    w = synth.workload(key)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_native(args, w)


if __name__ == "__main__":
    main()
