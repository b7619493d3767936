"""The multi-rank measurement logic of bench.py, run as two gloo ranks on
the CPU: the job's time is the slowest rank's, the value counts every
replica's bytes, and the reference arm runs on rank 0 only.  The forward has
no exchange step, so ranks are independent replicas and these reductions are
the only collectives the benchmark issues."""

import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.elapsed_max_over_ranks(10.0 + 5.0 * rank)       # rank 1 is the slow one
        w = bench.world_size()
        v = bench.whole_job_gbs(1e9, 4, ms, w)
        bench.barrier()

        class NoOracle:
            def __init__(self):
                raise AssertionError("the reference arm must not run on rank != 0")

        bench.OracleDecode = NoOracle if rank != 0 else bench.OracleDecode

        class A:
            steps, gpus = 1, world
        rc = bench.reference_arm(A) if rank != 0 else 0
        q.put((rank, ms, w, v, rc))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_total_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, w, v, rc in res:
        assert ms == 15.0                 # max over ranks, seen by every rank
        assert w == 2
        # 2 replicas x 1 GB x 4 steps over 15 ms
        assert v == pytest.approx(2 * 1e9 * 4 / 15e-3 / 1e9)
        assert rc == 0


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.world_size() == 1
    assert bench.elapsed_max_over_ranks(3.5) == 3.5
    assert bench.whole_job_gbs(2e9, 10, 1000.0, 1) == pytest.approx(20.0)


def test_reference_arm_prints_one_contract_line(capsys):
    # --impl reference on one process: the CPU oracle timed on the decode
    # sweep, printed as the reference arm's JSON line
    sys.path.insert(0, ROOT)
    import json
    import bench

    class A:
        steps, gpus = 1, 1

    assert bench.reference_arm(A) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "workload" in d["config"]
    # the plain C++ oracle timed beside the numpy one, on one thread
    cpp = d["cpu_baseline"]["cpp_oracle"]
    assert "unavailable" not in cpp, cpp
    assert cpp["value"] > 0 and cpp["cores"] == 1 and cpp["kind"] == "oracle" and cpp["unit"] == "GB/s"
