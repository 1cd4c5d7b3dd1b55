"""The N > 1 path of bench.py on CPU with gloo (world size 2).

The path does not shard, so N ranks run N replicas and the job's time is the
largest per-rank device time; rank 0 alone reports.  These tests run the
aggregation helpers across two real gloo ranks, and the reference arm's rank
handling (only rank 0 works)."""
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


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]  # rank 1 is the slow one
        job_ms = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.job_throughput(world, 1000, job_ms)
        w, r, l = bench._dist_init()
        q.put((rank, job_ms, value, (w, r, l)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, job_ms, value, env in got:
        assert job_ms == 5.0  # the max over ranks, on every rank
        assert value == pytest.approx(2 * 1000 / 5e-3)
        assert env == (2, rank, rank)


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(2.5) == 2.5
    assert bench.job_throughput(1, 2_097_152, 4.0) == pytest.approx(2_097_152 / 4e-3)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload, warmup, steps = "tiny", 0, 1
        tokens_per_rank = ffn = None

    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(Args()) is None
    monkeypatch.setenv("RANK", "0")
    line = bench.run_reference(Args())
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["cores"] == 1
    # the step as run: its wall time, not the whole-layer estimate the value uses
    cb = line["cpu_baseline"]
    assert line["ms_per_step"] == cb["ms_per_step_measured"]
    assert line["steps"] * line["ms_per_step"] <= 1e3 * line["wall_s"] + 1.0
    assert cb["oracle_plan_ms"] > 0 and cb["host_cpu_count"] >= 1 and "cpu_model" in cb
    # both arms describe the workload with the same config
    assert line["config"] == bench._config(bench._workload(Args()), 2)


def test_traffic_record_hash_ignores_comments(tmp_path):
    sys.path.insert(0, ROOT)
    import bench

    code = "int a; // note\n/* block\n comment */ int b;\n\n  // only a comment\nint c;\n"
    assert bench._code_only(code) == "int a;\n int b;\nint c;"
    assert bench._code_only(code.replace("note", "other note")) == bench._code_only(code)
    assert bench._code_only(code.replace("int c", "int d")) != bench._code_only(code)
