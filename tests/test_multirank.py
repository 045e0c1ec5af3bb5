"""The N > 1 host path of bench.py on CPU: two ranks over gloo (127.0.0.1).

`bench.py --gpus N` runs one replica of the layer per GPU on its own tokens (weak scaling, no
collective on the data path); the ranks only agree on the job's time (the slowest rank's)
and rank 0 prints the whole-job rate.  The same helpers run here with gloo on CPU tensors.
"""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        t_local = 0.5 * (rank + 1)  # rank 1 is the slow one
        t = bench.max_over_ranks(t_local, world, device="cpu")
        bench.barrier(world)
        v = bench.job_throughput(1000.0, t, world)
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def _run(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_two_ranks_agree_on_the_slowest_time_and_the_job_rate():
    out = _run(2)
    assert [r for r, _, _ in out] == [0, 1]
    for _, t, v in out:
        assert t == 1.0                      # max over ranks
        assert v == pytest.approx(2000.0)    # 2 ranks x 1000 units / 1.0 s


def test_reference_arm_runs_on_rank_0_only(capsys):
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_27_b200 import inputs as IN

    class Args:  # the reference arm's arguments; rank 1 must return before doing any work
        gpus, steps, warmup, wgrad_fp32, persistent, mx_wgrad = 2, 1, 3, False, False, False
    bench.run_reference(Args, IN.WORKLOADS["tiny"], world=2, rank=1)
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_line_on_rank_0(capsys):
    import json
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_27_b200 import inputs as IN

    class Args:
        gpus, steps, warmup, wgrad_fp32, persistent, mx_wgrad = 2, 2, 3, False, False, False
    w = IN.WORKLOADS["tiny"]
    bench.run_reference(Args, w, world=2, rank=0)
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    # the same config as the GPU arm's line, and a rate that is the timed steps' own
    assert line["config"] == bench.run_config(w, Args)
    assert line["config"]["wgrad_dtype"] == "bf16" and line["config"]["forward"] == "launches"
    tokens = bench.oracle_sample(w, bench.cpu_inputs(w))[1] / w.k  # tokens of work per step
    assert abs(line["value"] * line["ms_per_step"] / 1e3 - tokens) < 1e-6 * tokens
