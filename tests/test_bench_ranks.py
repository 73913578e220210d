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
