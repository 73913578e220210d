"""The bench's multi-rank logic on CPU: two gloo ranks (127.0.0.1) agree on the max-over-ranks
time, replicas draw distinct batches, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    try:
        r, w = bench.dist_init("gloo")
        bench.barrier()
        got = bench.max_over_ranks(1.5 + rank)
        seed = bench.replica_seed(4, rank)
        seeds = [None] * w
        dist.all_gather_object(seeds, seed)
        q.put((rank, r, w, got, seeds))
        dist.destroy_process_group()
    except Exception as e:  # noqa: BLE001
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_max_time_and_distinct_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    for res in results:
        assert res[1] != "error", res
        rank, r, w, got, seeds = res
        assert r == rank and w == 2
        assert got == 2.5
        assert len(set(seeds)) == 2


def test_reference_arm_only_on_rank_zero(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_warmup_below_three_is_rejected():
    sys.path.insert(0, ROOT)
    import bench

    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_forcing_options_are_validated():
    """--cta and --codes take only the library's settings (checked before any device work)."""
    sys.path.insert(0, ROOT)
    import bench

    for bad in (["--cta", "both"], ["--codes", "int4"]):
        with pytest.raises(SystemExit):
            bench.main(bad)


def test_fp4_peak_is_twice_the_int8_peak():
    """The e2m1 (kind::mxf4) roofline is the int8 one doubled (nominal 9 / 4.5 PFLOP/s)."""
    sys.path.insert(0, ROOT)
    import bench
    from binarized_convolution_b200 import synth

    w = synth.workload("xnor_beta_n16_56x56_c256_k256_3x3")
    p_int8, bound8, _ = bench.derived_peak(w, 148, 1965.0, "tc_conv", 1)
    p_fp4, bound4, how = bench.derived_peak(w, 148, 1965.0, "tc_conv", bench.CODES_FP4)
    assert bound8 == bound4 == "tensor"
    assert p_fp4 == pytest.approx(2 * p_int8)
    assert "fp4" in how


def test_timed_region_fills_the_seconds_whatever_the_step_count():
    """The timed region holds at least --steps steps and enough to fill the requested device time;
    the contraction sampling keeps at least three timed launches."""
    sys.path.insert(0, ROOT)
    import bench

    assert bench.timed_step_count(20, 0.044, 2.0) == 45455  # 2 s of 44 us steps
    assert bench.timed_step_count(100000, 0.044, 2.0) == 100000
    assert bench.timed_step_count(20, 50.0, 2.0) == 40
    assert bench.profile_stride(45455) == bench.PROFILE_EVERY
    assert bench.profile_stride(9) == 3 and bench.profile_stride(2) == 1


def test_forward_roofline_is_the_slower_of_bytes_and_ops():
    """Whole-step roofline: algorithmic bytes (fp32 in + packed weight bits + fp32 out) over HBM
    against nominal ops over the pipe's peak."""
    sys.path.insert(0, ROOT)
    import bench
    from binarized_convolution_b200 import synth

    w = synth.workload("xnor_beta_n16_56x56_c256_k256_3x3")
    b = bench.algorithmic_bytes(w)
    assert b == 16 * 56 * 56 * 256 * 4 * 2 + 256 * 9 * 8 * 4
    gbs, _ = bench.hbm_peak()
    r = bench.forward_roofline(w, step_ms=0.05, pipe_peak_tops=1e6)  # ops cost nothing: HBM-bound
    assert r["bound"] == "hbm" and r["t_roof_us"] == pytest.approx(b / (gbs * 1e3))
    assert r["frac"] == pytest.approx(r["t_roof_us"] / 50.0)
    r = bench.forward_roofline(w, step_ms=1.0, pipe_peak_tops=1.0)  # 1 TOPS: ops-bound
    assert r["bound"] == "tensor" and r["t_roof_us"] == pytest.approx(w.nominal_ops / 1e12 * 1e6)
