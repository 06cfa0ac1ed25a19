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


def _split_rank(rank, world, port, q, cfg_name):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import numpy as np
    import torch
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle.vsa_oracle as O
        from tile_sparse_video_pack_b200.shard import partition_heads, shard_config, shard_heads_of
        from vsa_synth import get_config
        cfg = get_config(cfg_name)
        s = cfg.sparsity[0]
        h0, h1 = partition_heads(cfg.heads, world, rank)
        sub = shard_config(cfg, h0, h1)
        ks = bench.k_list(sub, s)
        ntv = [O.head_tiling(sub, h).n_video for h in range(sub.heads)]
        # this rank's share: FLOPs, video tiles, index rows (tiles x k) and packed tiles
        mine = torch.tensor([bench.attention_flops(sub, ks), sum(ntv), sum(n * k for n, k in zip(ntv, ks)),
                             sub.heads * (O.head_tiling(sub, 0).n_prefix + max(ntv))], dtype=torch.float64)
        total = mine.clone()
        dist.all_reduce(total, op=dist.ReduceOp.SUM)
        ranges = [None] * world
        dist.all_gather_object(ranges, (h0, h1))
        # the rank's slice of a token-major tensor and of per-head projections
        x = np.arange(2 * 3 * cfg.heads * 4).reshape(2, 3, cfg.heads, 4)
        w = np.arange(cfg.heads * 6).reshape(cfg.heads, 3, 2)
        parts = [None] * world
        dist.all_gather_object(parts, (shard_heads_of(x, h0, h1, 2), shard_heads_of(w, h0, h1, 0)))
        q.put((rank, ranges, total.tolist(), mine.tolist(),
               bool(np.array_equal(np.concatenate([p[0] for p in parts], axis=2), x)),
               bool(np.array_equal(np.concatenate([p[1] for p in parts], axis=0), w))))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("cfg_name", ["full", "veda"])
def test_head_split_ranks_tile_the_layer(cfg_name):
    """Two gloo ranks split one layer's heads (--split heads): their head ranges tile [0, H), and
    their FLOP counts, video tiles and index rows add up to the single-rank layer's."""
    import bench
    import oracle.vsa_oracle as O
    from vsa_synth import get_config
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_rank, args=(r, 2, port, q, cfg_name)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    cfg = get_config(cfg_name)
    ks = bench.k_list(cfg, cfg.sparsity[0])
    ntv = [O.head_tiling(cfg, h).n_video for h in range(cfg.heads)]
    want = [bench.attention_flops(cfg, ks), sum(ntv), sum(n * k for n, k in zip(ntv, ks))]
    for rank, ranges, total, mine, x_ok, w_ok in got:
        assert ranges == [(0, cfg.heads // 2), (cfg.heads // 2, cfg.heads)]
        assert total[:3] == want
        assert x_ok and w_ok
    # each rank holds half the heads' packed tiles
    assert got[0][3][3] + got[1][3][3] >= cfg.heads * (O.head_tiling(cfg, 0).n_prefix + min(ntv))


def test_partition_heads_covers_uneven_splits():
    from tile_sparse_video_pack_b200.shard import partition_heads
    for heads in (1, 5, 24, 64):
        for world in range(1, min(heads, 9) + 1):
            r = [partition_heads(heads, world, k) for k in range(world)]
            assert r[0][0] == 0 and r[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [b - a for a, b in r]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        partition_heads(4, 5, 0)
