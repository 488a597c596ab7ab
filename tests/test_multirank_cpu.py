"""The benchmark's multi-rank logic on CPU ranks (gloo, world size 2): the
layer has no exchange step, so N GPUs run N replicas; the only collectives
are the start/stop barriers and the max of the step time over the ranks, and
the whole-job value counts every rank's work over the slowest rank's time.
The reference arm runs on rank 0 alone."""
import json
import os
import socket
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        local_ms = 2.0 + rank                       # rank 1 is the slow one
        mx = bench.allreduce_max(local_ms, world)
        bench.barrier(world)
        value = bench.whole_job_tflops(1e12, world, mx)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max_ms": mx, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_two_cpu_ranks_take_the_max_and_count_both_replicas(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["max_ms"] == 3.0                   # the slowest rank's time, on every rank
        # 2 replicas x 1e12 flops in 3 ms
        assert r["value"] == pytest.approx(2 * 1e12 / 3e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.allreduce_max(1.5, 1) == 1.5
    bench.barrier(1)
    assert bench.whole_job_tflops(2e12, 1, 2.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    # ranks other than 0 exit without work or output
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = types.SimpleNamespace(gpus=2, steps=1, warmup=0)
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""


def test_a_failing_secondary_section_is_recorded_not_fatal():
    errors = {}
    assert bench.guarded(errors, "ok", lambda: 7) == 7
    assert errors == {}

    def broken():
        raise RuntimeError("device lost " + "x" * 1000)

    assert bench.guarded(errors, "lora", broken) is None
    assert list(errors) == ["lora"] and errors["lora"].startswith("RuntimeError: device lost")
    assert len(errors["lora"]) <= 400
