"""The N > 1 bench path on the CPU: two gloo ranks check the whole-job
aggregation (slowest rank's time, every rank's work) and the barrier, and the
reference arm's rule that only rank 0 runs and prints."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env()[:2] == (world, rank)
        bench.barrier(world)
        # rank r took (r + 1) ms for 10 (r + 1) units
        ms, units = bench.aggregate(float(rank + 1), 10.0 * (rank + 1), world)
        out[rank] = (ms, units)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_and_barrier():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        codes = [p.exitcode for p in procs]
        result = dict(out)
    assert codes == [0, 0], codes
    # the job's time is the slowest rank's, its work the sum over ranks
    assert result[0] == result[1] == (2.0, 30.0)


def test_single_rank_aggregation_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(3.5, 7.0, 1) == (3.5, 7.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_oracle_timing_per_config_restores_threads():
    """The per-configuration oracle baseline: a bounded token prefix, one
    thread where asked, and the OpenMP thread count put back afterwards."""
    sys.path.insert(0, ROOT)
    import bench
    before = bench.omp_threads()
    out = bench.time_oracle_other_configs(0.3, ids=(0,), single_thread=(0,))
    assert bench.omp_threads() == before
    assert set(out["0"]) == {"all", "1"}
    assert out["0"]["1"]["cores"] == 1 and out["0"]["all"]["cores"] == before
    for run in out["0"].values():
        assert run["kind"] == "oracle" and run["value"] > 0 and "of 8 tokens" in run["sample"]
