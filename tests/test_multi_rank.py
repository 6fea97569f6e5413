"""The N > 1 bench path on CPU: two gloo ranks.  Each GPU runs an independent
replica of the workload (no data-path collective), the timed region is the
slowest rank's, and the whole-job value counts every rank's work."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        m = bench.max_over_ranks(local_ms[rank], dist, "cpu")
        v = bench.whole_job_rate(1000.0, world, m)
        out[rank] = (m, v)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    local = [1.5, 4.0]
    mp.spawn(_rank_main, args=(2, port, local, out), nprocs=2, join=True)
    assert out[0][0] == out[1][0] == 4.0
    # 2 replicas x 1000 units in 4 ms
    assert out[0][1] == pytest.approx(2 * 1000.0 / 4e-3)


def test_single_process_is_identity():
    assert bench.max_over_ranks(2.5) == 2.5
    assert bench.whole_job_rate(10.0, 1, 2.0) == pytest.approx(5000.0)


def test_reference_arm_only_on_rank_zero(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup, gpus, ref_step_s = 1, 3, 2, 0.01
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(monkeypatch, capsys):
    """The reference arm (the CPU oracle on a bounded sample) prints one JSON
    line with the ours-arm's metric, unit and workload config, and its own
    cpu_baseline and e2e objects."""
    import json
    from semi_structured_sparse_nm_b200 import inputs
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class A:
        steps, warmup, gpus, ref_step_s = 1, 0, 1, 0.01
    assert bench.run_reference(A()) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s" and line["higher_is_better"]
    assert line["config"] == bench.workload_config(inputs.WORKLOADS[bench.HEADLINE], 1)
    assert line["config"]["workload"] == bench.HEADLINE
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
