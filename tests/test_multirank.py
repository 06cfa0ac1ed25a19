"""The multi-GPU bench logic on CPU: two gloo ranks, max-over-ranks timing and the job value."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local = [80.0, 95.5][rank]                 # each rank's own step time
        m = bench.max_over_ranks_on(local, "cpu", world)
        q.put((rank, m, bench.job_ms_per_layer(m, 1, world)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_take_the_max_and_divide_by_layers():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 95.5, 47.75), (1, 95.5, 47.75)]


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks_on(12.5, "cpu", 1) == 12.5
    assert bench.job_ms_per_layer(12.5, 1, 1) == 12.5


def _bench_reference(env_extra):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]


def test_reference_arm_prints_the_same_metric_and_config():
    """The oracle arm's line names the metric, unit and config of the CUDA arm's line."""
    import bench
    import oracle.vsa_oracle as O
    from vsa_synth import get_config
    lines = _bench_reference({"RANK": "0", "WORLD_SIZE": "1"})
    assert len(lines) == 1
    d = lines[0]
    cfg = get_config("tiny")
    pt, ph, pw = cfg.tile_shapes[0]
    k0 = O.k_from_sparsity(cfg.sparsity[0], -(-cfg.T // pt) * -(-cfg.H // ph) * -(-cfg.W // pw))
    assert d["impl"] == "reference" and d["metric"] == bench.metric_for(cfg) and d["unit"] == "ms"
    assert d["higher_is_better"] is False and d["value"] > 0
    assert d["config"] == bench.workload_config(cfg, cfg.sparsity[0], k0, 1)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    # the steps it ran were samples of the layer, and the line says the value is extrapolated
    assert d["extrapolated"] is True and d["steps"] == 1 and 0 < d["ms_per_step"] < 600e3
    assert d["e2e"] == {"value": d["value"], "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    assert _bench_reference({"RANK": "1", "WORLD_SIZE": "2"}) == []
