"""Benchmark: one tile-sparse attention layer of a 1344x768-like clip on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one whole layer -- tile pack, tile score, top-k select, block-sparse
attention, tile unpack -- through the C ABI of libvsa, on inputs already in
HBM. Workload: B=1, 24 heads, head_dim 128, video grid 28x48x80 (107,520
tokens, 1,680 tiles of 4x4x4) after a 4,992-token prefix (512 text, 3,840
reference-image, 640 reference-audio tokens), mean-pool gate scoring, 75% video
sparsity (420 kept tiles); the 90% line is measured in the same run. Inputs are
seeded synthetic tensors (3 x 691 MB, larger than L2).

Other workloads (--config): veda (head-aware tiles, TripPool, 90% and 95%), long
(230k video tokens, sparsity 0 ... 0.95), r2va, medium, tiny. Every sparsity level
of the workload other than the first is measured in the same run ("sweep").

Multi-GPU (torchrun): by default every rank runs its own layer (independent
problems, weak scaling); with --split heads the ranks share one layer, each
running its block of heads (strong scaling). Neither has a collective on the data
path; the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference there is) on a
fixed bounded sample of the same workload and extrapolates to one layer.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

CONFIG = "full"
METRIC = "ms per attention layer at 107k video tokens, 75% video sparsity (90% in sweep); effective TFLOP/s"


def metric_for(cfg):
    """The metric string: the headline one for the full clip, a workload-specific one otherwise."""
    if cfg.name == CONFIG:
        return METRIC
    return (f"ms per attention layer, {cfg.name} workload ({cfg.n_video_tokens} video tokens), "
            f"sparsity {cfg.sparsity[0]} (other levels in sweep); effective TFLOP/s")
KERNELS_PER_STEP = 6  # pack + pool 1, score 2 (both projections in one launch, scores), select 1, attention 1, unpack 1
KERNELS_PER_STEP_DIRECT = 5  # pool 1, score 2, select 1, attention straight from q, k, v into o 1


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=CONFIG)
    ap.add_argument("--sparsity", type=float, default=None,
                    help="video-key sparsity (default: the workload's first level, 0.75 for the full clip)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", "--no-sweep", dest="no_secondary", action="store_true",
                    help="measure only the first sparsity level of the workload")
    ap.add_argument("--split", default="layers", choices=["layers", "heads"],
                    help="multi-GPU: each rank its own layer (weak scaling) or its block of one layer's heads")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (profiling runs)")
    ap.add_argument("--direct", action="store_true",
                    help="attention straight from the token-major q, k, v (vsa_tile_pool + vsa_sparse_attn_direct, "
                         "no packed copies; slower) instead of pack + pool, attention on packed tiles, unpack")
    ap.add_argument("--fp8", action="store_true",
                    help="Q K^T from e4m3 tiles with per-tile scales (vsa_tile_pack_pool_fp8 + vsa_sparse_attn_fp8)")
    ap.add_argument("--teacher", action="store_true",
                    help="also time the teacher tile map and report the selection's tile recall")
    ap.add_argument("--dense-reference", action="store_true",
                    help="also time torch's dense scaled_dot_product_attention on the same Q, K, V (context only)")
    args = ap.parse_args()
    if args.sparsity is None:
        from vsa_synth import get_config
        args.sparsity = get_config(args.config).sparsity[0]
    return args


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------- ncu traffic ----

ATTN_SRC = os.path.join(ROOT, "tile_sparse_video_pack_b200", "csrc", "attn.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_kernel_traffic.txt")


def attn_source_sha1() -> str:
    import hashlib
    with open(ATTN_SRC, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()


def measured_traffic(config: str, sparsity: float, heads: int, path: str = "packed"):
    """DRAM bytes per attention launch from the committed ncu capture, if it is of this kernel source.

    The capture runs a smaller case (fewer heads) of the same workload; bytes grow
    in proportion to the heads, so they are scaled to the benchmarked head count.
    Returns None when the kernel changed after the capture.
    """
    if not os.path.exists(TRAFFIC_FILE):
        return None
    kv = {}
    with open(TRAFFIC_FILE) as f:
        for ln in f:
            if "=" in ln and not ln.startswith("#"):
                a, b = ln.split("=", 1)
                kv[a.strip()] = b.strip()
    if (kv.get("attn_source_sha1") != attn_source_sha1() or kv.get("config") != config
            or float(kv.get("sparsity", "nan")) != sparsity or kv.get("path", "packed") != path):
        return None
    per_head = (float(kv["dram_bytes_read"]) + float(kv["dram_bytes_write"])) / float(kv["heads"])
    return int(per_head * heads)


# --------------------------------------------------------------- work counts --

def k_list(cfg, s):
    from tile_sparse_video_pack_b200 import vsa
    return [vsa.k_from_sparsity(s, -(-cfg.T // pt) * -(-cfg.H // ph) * -(-cfg.W // pw))
            for (pt, ph, pw) in cfg.tile_shapes]


def attention_flops(cfg, ks):
    """4 * d * sum over query rows of their key count (full tiles: closed form).

    With reference segments (R2VA budgets) a video row sees the dense prefix tokens
    plus k_ref reference tiles of 64 tokens instead of the whole prefix.
    """
    n = cfg.n_tokens
    npre = cfg.n_prefix_tokens
    nv = cfg.n_video_tokens
    flags = tuple(getattr(cfg, "seg_ref", ())) or (0,) * len(cfg.segments)
    ref_tok = sum(length for length, f in zip(cfg.segments, flags) if f)
    video_prefix = npre - ref_tok + (64 * cfg.k_ref if ref_tok else 0)
    pairs = 0
    for kh in ks:
        pairs += npre * n + nv * (video_prefix + kh * 64)
    return 4 * cfg.head_dim * pairs * cfg.batch


def workload_config(cfg, sparsity, k0, world, split="layers"):
    """The `config` object of the bench line, shared by both arms."""
    ref = cfg.seg_ref and any(cfg.seg_ref)
    mb = cfg.batch * cfg.n_tokens * cfg.heads * cfg.head_dim * 2 / 1e6
    heads_split = split == "heads" and world > 1
    return {"workload": f"{cfg.name}: one layer, B={cfg.batch}, {cfg.heads} heads, d={cfg.head_dim}, "
                        f"grid {cfg.T}x{cfg.H}x{cfg.W} + prefix {list(cfg.segments)}, "
                        f"{cfg.score_mode}, sparsity {sparsity} (k={k0})"
                        + (f", reference segments {list(cfg.seg_ref)} with k_ref={cfg.k_ref}" if ref else ""),
            "tokens": cfg.n_tokens, "heads": cfg.heads, "head_dim": cfg.head_dim, "k": k0,
            "layers_per_step": 1 if heads_split else world,
            "parallelism": (f"heads of one layer split over {world} ranks" if heads_split
                            else f"independent layers x{world}"),
            "l2": (f"inputs larger than L2 (Q, K, V {mb:.0f} MB each)" if mb > 126 else
                   f"inputs {mb:.0f} MB each: L2-resident between steps")}


def attn_roofline(args, cfg, peaks, flops, attn_ms):
    """The `roofline` object for the attention kernel from its event-timed mean duration."""
    achieved = flops / (attn_ms * 1e-3) / 1e12
    # fp8: Q K^T (half the FLOPs) at the e4m3 rate, twice bf16's (nominal ratio), P V at bf16, so the
    # mixed peak is 1 / (0.5 / 2 + 0.5 / 1) = 4/3 of the measured bf16 peak
    mix = 4.0 / 3.0 if args.fp8 else 1.0
    # each launch is timed on its own (tens of ms), not a seconds-long loop: the burst peak
    peak = round(peaks["bf16_tflops"] * mix, 1)
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": None if args.fp8 else measured_traffic(args.config, args.sparsity, cfg.heads,
                                                              getattr(args, "path", "packed")),
            "kernel": "attn_kernel<128, fp8> (vsa_sparse_attn_fp8; e4m3 Q K^T, bf16 P V)" if args.fp8
                      else ("attn_kernel, tiles straight from token-major q, k, v (vsa_sparse_attn_direct)"
                            if getattr(args, "path", "packed") == "direct" else "attn_kernel (vsa_sparse_attn)"),
            "peak_kind": (f"half e4m3 (2x bf16, nominal ratio), half bf16: 4/3 x bf16 dense, burst, "
                          f"{peaks['source']}") if args.fp8 else f"bf16 dense, burst, {peaks['source']}",
            "frac_of_sustained_peak": round(achieved / (peaks["bf16_tflops_sustained"] * mix), 4),
            "algorithmic_flops_per_launch": flops}


def bench_line(args, cfg, world, ks, flops, ms_step, stages, roofline, e2e, clocks, stats, sweep,
               teacher=None):
    """The JSON line of the CUDA arm (rank 0 prints it). With the heads of one layer split over
    the ranks, `cfg`, `ks` and `flops` are the whole layer's and a step is that one layer."""
    ref = cfg.seg_ref and any(cfg.seg_ref)
    split = getattr(args, "split", "layers")
    heads_split = split == "heads" and world > 1
    line = {
        "metric": metric_for(cfg),
        "value": round(ms_step if heads_split else job_ms_per_layer(ms_step, 1, world), 3), "unit": "ms",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3), "higher_is_better": False,
        "scaling": "strong" if heads_split else "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": workload_config(cfg, args.sparsity, ks[0], world, split),
        "stages_ms": {a: round(b, 3) for a, b in stages.items()},
        "effective_tflops": {"attn_kernel": roofline["achieved"],
                             "layer": round(flops / (ms_step * 1e-3) / 1e12, 1)},
        "score_select_share": round((stages["score"] + stages["select"]) / sum(stages.values()), 4),
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": ((KERNELS_PER_STEP_DIRECT if getattr(args, "path", "packed") == "direct" else KERNELS_PER_STEP)
                         + (4 if ref else 0)) * args.steps,
        "path": getattr(args, "path", "packed"),
        "clocks": clocks,
        "attention_computed_pct": round(100.0 * stats["computed_pairs"] / stats["dense_pairs"], 2),
        "sweep": sweep,
    }
    if teacher is not None:
        line["teacher"] = teacher
    return line


# ------------------------------------------------------------------ clocks ----

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return summarize_clocks(lines)


def summarize_clocks(lines):
    """Median SM clock under load, the maximum clock and the throttle reasons seen, from
    `nvidia-smi --query-gpu=<ClockSampler.FIELDS> --format=csv,noheader,nounits` rows."""
    rows = []
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:9]))
        except ValueError:
            continue
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    load = [r for r in rows if r[2] > 300.0] or rows     # samples drawing over 300 W: the timed kernels
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in load for i in range(4) if r[3][i + 1].lower().startswith("active")})
    return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
            "samples": len(load), "power_w_max": max(r[2] for r in rows), "reasons": reasons}


# ------------------------------------------------------------- CPU oracle ----

class OracleSample:
    """The fp64 oracle, as it stands, timed on a fixed bounded sample of one layer.

    One sample: scores and top-k of head 0 in full, then attention (the same two
    oracle calls run_layer makes per query tile) of a fixed, evenly spaced set of
    head 0's query tiles -- n_video video tiles and n_prefix prefix tiles. Each
    kind's mean time per tile is extrapolated to every query tile of every head.
    Both bench arms use this class with the same sample, so their estimates agree.
    """

    N_VIDEO, N_PREFIX = 48, 16

    def __init__(self, cfg, sparsity):
        import numpy as np
        import oracle.vsa_oracle as O
        from vsa_synth import bf16_bits_to_f32, make_layer_inputs
        self.np, self.O = np, O
        self.cfg = cfg
        self.sub = cfg.with_(heads=1, tile_shapes=cfg.tile_shapes[:1])
        self.inp = make_layer_inputs(self.sub)
        f = lambda b: bf16_bits_to_f32(b).astype(np.float64)
        self.q, self.k, self.v = f(self.inp.q), f(self.inp.k), f(self.inp.v)
        self.ks = [O.k_from_sparsity(sparsity, -(-cfg.T // pt) * -(-cfg.H // ph) * -(-cfg.W // pw))
                   for (pt, ph, pw) in self.sub.tile_shapes]
        self.til = O.head_tiling(self.sub, 0)
        til = self.til
        pick = lambda n, m: sorted({int(x) for x in np.linspace(0, n - 1, min(n, m))}) if n else []
        self.video_tiles = [til.n_prefix + i for i in pick(til.n_video, self.N_VIDEO)]
        self.prefix_tiles = pick(til.n_prefix, self.N_PREFIX)

    def run(self):
        """One sample; returns the extrapolated ms per layer and what was timed."""
        np, O, sub, til, inp = self.np, self.O, self.sub, self.til, self.inp
        t0 = time.perf_counter()
        s = O.tile_scores(self.q[0, :, 0], self.k[0, :, 0], til, sub, 0, inp.gate, inp.w_q, inp.w_k)
        kept = np.stack([O.topk_row(s[i], self.ks[0]) for i in range(til.n_video)])
        t_select = time.perf_counter() - t0
        scale = 1.0 / math.sqrt(sub.head_dim)
        q, k, v = self.q[0, :, 0], self.k[0, :, 0], self.v[0, :, 0]
        spent = {}
        for kind, tiles in (("video", self.video_tiles), ("prefix", self.prefix_tiles)):
            t1 = time.perf_counter()
            for t in tiles:
                kv = O.query_key_tokens(til, t, None if t < til.n_prefix else kept[t - til.n_prefix])
                O.softmax_attention(q[til.all[t]], k[kv], v[kv], scale)
            spent[kind] = time.perf_counter() - t1
        per_head = t_select
        per_head += spent["video"] / max(1, len(self.video_tiles)) * til.n_video
        per_head += spent["prefix"] / max(1, len(self.prefix_tiles)) * til.n_prefix
        ms = per_head * self.cfg.heads * self.cfg.batch * 1e3
        try:
            cores = len(os.sched_getaffinity(0))
        except AttributeError:
            cores = os.cpu_count()
        sample = (f"head 0 of {self.cfg.heads}: scores + top-k of all {til.n_video} video query tiles, attention "
                  f"of a fixed set of {len(self.video_tiles)} video and {len(self.prefix_tiles)} prefix query "
                  f"tiles (fp64 numpy; BLAS on all cores); extrapolated to {self.cfg.heads} heads x "
                  f"({til.n_video} video + {til.n_prefix} prefix) query tiles")
        return {"value": round(ms, 1), "unit": "ms", "cores": cores, "kind": "oracle", "sample": sample,
                "extrapolated": True, "sample_s": round(time.perf_counter() - t0, 5)}


def oracle_full_layer_ms(cfg, sparsity):
    """The fp64 oracle's whole layer (every head and query tile), timed once: for workloads small
    enough to run in full (the medium one takes seconds to tens of seconds)."""
    import numpy as np
    import oracle.vsa_oracle as O
    from vsa_synth import bf16_bits_to_f32, make_layer_inputs
    inp = make_layer_inputs(cfg)
    f = lambda b: bf16_bits_to_f32(b).astype(np.float64)
    q, k, v = f(inp.q), f(inp.k), f(inp.v)
    ks = [O.k_from_sparsity(sparsity, -(-cfg.T // pt) * -(-cfg.H // ph) * -(-cfg.W // pw))
          for (pt, ph, pw) in cfg.tile_shapes]
    t0 = time.perf_counter()
    O.run_layer(cfg, q, k, v, ks, gate=inp.gate, w_q=inp.w_q, w_k=inp.w_k)
    return (time.perf_counter() - t0) * 1e3


def cpu_baseline(cfg, sparsity):
    """The oracle on the host: one warm-up sample and one timed sample of this workload."""
    s = OracleSample(cfg, sparsity)
    s.run()
    return s.run()



# ---------------------------------------------------------------- ranks ------

def max_over_ranks_on(x: float, device, world: int) -> float:
    """The largest of every rank's x (each rank runs the same number of steps)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_ranks_sum(x: float, device, world: int) -> float:
    """The sum of every rank's x (the head blocks of one layer add up to the layer)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_ms_per_layer(ms_step_max: float, layers_per_rank: int, world: int) -> float:
    """Whole-job time per layer: the slowest rank's step time over all layers processed in a step."""
    return ms_step_max / (layers_per_rank * world)


# ---------------------------------------------------------------- GPU arm ----

def e2e_measure(args, layer, q, k, v, out, stream, world, barrier, max_over_ranks, layers=None):
    """The same layer through the public API from pinned host buffers, copies inside the timing.

    Every step copies its q, k, v in from pinned host memory, runs the layer and copies o
    back. The copies run on their own streams (host-to-device and device-to-host), double
    buffered, so step i+1's inputs and step i-1's output cross PCIe while step i computes.
    The timed window holds as many steps as the device-timed loop; it includes the first
    step's inputs (nothing to overlap them with) and the last step's output, which the
    steps in between amortise.
    """
    import torch
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    ho = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    dev_in = [[torch.empty_like(x) for x in (q, k, v)] for _ in range(2)]
    dev_out = [torch.empty_like(out) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, consumed, out_ready, out_copied = ([ev(), ev()] for _ in range(4))
    steps = max(3, args.steps)

    def load(i):                       # inputs of step i into slot i % 2, once step i-2 is done with it
        s = i & 1
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(consumed[s])
            for dst, src in zip(dev_in[s], (hq, hk, hv)):
                dst.copy_(src, non_blocking=True)
            in_ready[s].record(h2d)

    def run(i):                        # step i on the compute stream, then its output back
        s = i & 1
        stream.wait_event(in_ready[s])
        if i >= 2:
            stream.wait_event(out_copied[s])
        layer.forward(*dev_in[s], dev_out[s])
        consumed[s].record(stream)
        out_ready[s].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(out_ready[s])
            ho[s].copy_(dev_out[s], non_blocking=True)
            out_copied[s].record(d2h)

    def window(n):
        load(0)
        for i in range(n):
            if i + 1 < n:
                load(i + 1)
            run(i)
        stream.wait_event(out_copied[(n - 1) & 1])

    window(2)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d)
    stream.wait_event(e0)
    window(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    # the layer is deterministic: what came back equals the device-timed run's output
    if not torch.equal(ho[(steps - 1) & 1].view(torch.int16), out.cpu().view(torch.int16)):
        raise RuntimeError("end-to-end output differs from the device-timed run")
    ms = max_over_ranks(e0.elapsed_time(e1) / steps) / (world if layers is None else layers)
    return {"value": round(ms, 3), "unit": "ms", "h2d_bytes_per_step": 3 * q.numel() * q.element_size() * world,
            "d2h_bytes_per_step": out.numel() * out.element_size() * world, "steps": steps,
            "overlap": "h2d of step i+1 and d2h of step i-1 run on copy streams during step i; the first step's "
                       "h2d and the last step's d2h are inside the window too"}


def gpu_layer_ms(cfg, sparsity, steps=10, warmup=3):
    """Mean device time of one whole layer (vsa_layer_forward) of `cfg` on the current GPU."""
    import numpy as np
    import torch
    import tile_sparse_video_pack_b200 as T
    from vsa_synth import make_layer_inputs
    inp = make_layer_inputs(cfg)
    to_dev = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    if cfg.score_mode == "meanpool_gate":
        pq = pk = torch.from_numpy(inp.gate).cuda()
    else:
        pq, pk = torch.from_numpy(inp.w_q).cuda(), torch.from_numpy(inp.w_k).cuda()
    layer = T.TileSparseAttention.from_config(cfg, sparsity, pq, pk)
    out = torch.empty_like(q)
    for _ in range(warmup):
        layer(q, k, v, out)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        layer(q, k, v, out)
    e1.record()
    torch.cuda.synchronize()
    layer.plan.check()
    return e0.elapsed_time(e1) / steps


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import tile_sparse_video_pack_b200 as T
    from tile_sparse_video_pack_b200.build import build
    from vsa_synth import get_config, make_layer_inputs

    from tile_sparse_video_pack_b200.shard import partition_heads, shard_config, shard_heads_of

    build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = get_config(args.config)
    if args.heads:
        cfg = cfg.with_(heads=args.heads, tile_shapes=cfg.tile_shapes[:args.heads])
    inp = make_layer_inputs(cfg)
    layer_cfg = cfg                              # the whole layer (for the FLOP count and the line)
    heads_split = args.split == "heads" and world > 1
    h0, h1 = partition_heads(cfg.heads, world, rank) if heads_split else (0, cfg.heads)
    if heads_split:                              # this rank's block of the layer's heads
        cfg = shard_config(cfg, h0, h1)
    pick = lambda x: shard_heads_of(x, h0, h1, 2) if heads_split else x
    to_dev = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = to_dev(pick(inp.q)), to_dev(pick(inp.k)), to_dev(pick(inp.v))
    if cfg.score_mode == "meanpool_gate":        # the gate is shared by all heads: replicated
        pq = pk = torch.from_numpy(inp.gate).to(dev)
    else:                                        # per-head projections: this rank's heads
        w = lambda x: shard_heads_of(x, h0, h1, 0) if heads_split else x
        pq, pk = torch.from_numpy(w(inp.w_q)).to(dev), torch.from_numpy(w(inp.w_k)).to(dev)
    peaks = measured_peaks()
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return max_over_ranks_on(x, dev, world)

    def timed_layer(sparsity, steps, warmup, sample_clocks):
        layer = T.TileSparseAttention.from_config(cfg, sparsity, pq, pk, direct=args.direct and not args.fp8)
        args.path = "direct" if layer.direct else "packed"
        out = torch.empty_like(q)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
        for _ in range(warmup):
            layer.stages(q, k, v, out)
        layer.plan.check()
        barrier()
        torch.cuda.synchronize()
        clk = ClockSampler(local_rank) if sample_clocks else None
        if clk:
            clk.start()
        barrier()
        torch.cuda.synchronize()
        b, p = layer.bufs, layer.plan
        f8 = p.allocate_fp8() if args.fp8 else None
        direct = layer.direct and f8 is None
        for i in range(steps):
            e = ev[i]
            e[0].record(stream)
            if direct:                      # no packed copies: tiles straight from q, k, v; o written directly
                p.tile_pool(q, k, b["workspace"])
                e[1].record(stream)
                p.tile_score_pooled(pq, pk, b["scores"], b["workspace"])
                e[2].record(stream)
                p.topk_select(b["scores"], b["idx"])
                e[3].record(stream)
                p.sparse_attn_direct(q, k, v, b["idx"], out)
                e[4].record(stream)
                e[5].record(stream)
                continue
            if f8 is not None:
                p.tile_pack_pool_fp8(q, k, v, b["qp"], b["kp"], b["vp"], f8["qp8"], f8["kp8"], f8["q_scale"],
                                     f8["k_scale"], b["workspace"])
            else:
                p.tile_pack_pool(q, k, v, b["qp"], b["kp"], b["vp"], b["workspace"])
            e[1].record(stream)
            p.tile_score_pooled(pq, pk, b["scores"], b["workspace"])
            e[2].record(stream)
            p.topk_select(b["scores"], b["idx"])
            if p.info.n_ref_tiles:          # R2VA budgets: reference tiles scored and selected too
                p.ref_score(b["kp"], pk, b["scores_ref"], b["workspace"])
                p.topk_select_ref(b["scores_ref"], b["idx_ref"])
            e[3].record(stream)
            if f8 is not None:
                p.sparse_attn_fp8(f8["qp8"], f8["kp8"], f8["q_scale"], f8["k_scale"], b["vp"], b["idx"], b["op"])
            elif p.info.n_ref_tiles:
                p.sparse_attn_ref(b["qp"], b["kp"], b["vp"], b["idx"], b["idx_ref"], b["op"], None)
            else:
                p.sparse_attn(b["qp"], b["kp"], b["vp"], b["idx"], b["op"], None)
            e[4].record(stream)
            p.tile_unpack(b["op"], out)
            e[5].record(stream)
        torch.cuda.synchronize()
        barrier()
        clocks = clk.stop() if clk else None
        layer.plan.check()
        total = sum(ev[i][0].elapsed_time(ev[i][5]) for i in range(steps))
        names = ("pool", "score", "select", "attn") if direct else ("pack_pool", "score", "select", "attn", "unpack")
        stages = {name: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(steps)) / steps
                  for j, name in enumerate(names)}
        ms_step = max_over_ranks(total / steps)
        stats = layer.plan.stats()
        return layer, out, ms_step, stages, clocks, stats

    def teacher_measure(layer, ks):
        """The teacher tile map of this workload and the tile recall of the layer's selection.

        A dense plan (k = every video tile) runs the layer once for the rows' full
        log-sum-exp; the teacher kernel is then timed on its own; its top-k (same k as
        the layer) is overlapped with the layer's selection.
        """
        ntv = [layer.plan.info.ntv[h] for h in range(cfg.heads)]
        dense = T.TileSparseAttention.from_config(cfg, 0.0, pq, pk, k_per_head=ntv)
        db = dense.bufs
        dp = dense.plan
        dp.tile_pack_pool(q, k, v, db["qp"], db["kp"], db["vp"], db["workspace"])
        dp.tile_score_pooled(pq, pk, db["scores"], db["workspace"])
        dp.topk_select(db["scores"], db["idx"])
        lse = torch.empty(dp.info.lse_elems, dtype=torch.float32, device=dev)
        dp.sparse_attn(db["qp"], db["kp"], db["vp"], db["idx"], db["op"], lse)
        teacher = torch.zeros_like(db["scores"])
        iters = 3
        dp.teacher_tiles(db["qp"], db["kp"], lse, teacher)            # warm-up
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            dp.teacher_tiles(db["qp"], db["kp"], lse, teacher)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / iters
        lp = layer.plan
        t_idx = torch.empty_like(layer.bufs["idx"])
        lp.topk_select(teacher, t_idx)
        counts = torch.empty(cfg.batch * cfg.heads * lp.info.ntv_max, dtype=torch.int32, device=dev)
        lp.index_overlap(layer.bufs["idx"], t_idx, counts)
        dp.check()
        lp.check()
        c = counts.view(cfg.batch, cfg.heads, lp.info.ntv_max).cpu().numpy()
        recall = float(np.mean([c[b, h, :ntv[h]].mean() / ks[h] for b in range(cfg.batch) for h in range(cfg.heads)]))
        flops = 2 * cfg.head_dim * cfg.batch * cfg.heads * cfg.n_video_tokens ** 2
        tf = flops / (ms * 1e-3) / 1e12
        return {"kernel": "teacher_kernel (vsa_teacher_tiles)", "ms": round(ms, 3), "tflops": round(tf, 1),
                "bound": "tensor", "peak": peaks["bf16_tflops"], "frac": round(tf / peaks["bf16_tflops"], 4),
                "peak_kind": f"bf16 dense, burst, {peaks['source']}", "algorithmic_flops": flops,
                "recall": round(recall, 4), "recall_of": f"{cfg.score_mode} selection, k={ks[0]}, vs the teacher's top-k"}

    ks = k_list(cfg, args.sparsity)
    layer, out, ms_step, stages, clocks, stats = timed_layer(args.sparsity, args.steps, args.warmup, True)
    if heads_split:                  # the whole layer's pairs: the sum over the ranks' head blocks
        stats = {key: int(all_ranks_sum(float(val), dev, world)) for key, val in stats.items()}
    flops = attention_flops(layer_cfg, k_list(layer_cfg, args.sparsity))
    roofline = attn_roofline(args, layer_cfg, peaks, flops, max_over_ranks(stages["attn"]))
    # every rank's stage times are its own; the line reports the slowest rank's
    stages = {name: max_over_ranks(val) for name, val in stages.items()}

    # end to end through host buffers: pinned H2D of q, k, v, the layer, D2H of o
    e2e = None if args.no_e2e else e2e_measure(args, layer, q, k, v, out, stream, world, barrier, max_over_ranks,
                                               layers=1 if heads_split else world)

    # the workload's other sparsity levels, measured in the same run
    sweep = []
    if not args.no_secondary:
        for s2 in [x for x in layer_cfg.sparsity if x != args.sparsity]:
            f2 = attention_flops(layer_cfg, k_list(layer_cfg, s2))
            _, _, ms2, st2, _, _ = timed_layer(s2, max(3, args.steps // 2), 2, False)
            st2 = {name: max_over_ranks(val) for name, val in st2.items()}
            sweep.append({"sparsity": s2, "k": k_list(layer_cfg, s2)[0],
                          "ms_per_layer": round(ms2 if heads_split else ms2 / world, 3),
                          "stages_ms": {a: round(b, 3) for a, b in st2.items()},
                          "attn_tflops": round(f2 / (st2["attn"] * 1e-3) / 1e12, 1),
                          "attn_frac_of_burst_peak": round(f2 / (st2["attn"] * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                          "layer_tflops": round(f2 / (ms2 * 1e-3) / 1e12, 1),
                          "algorithmic_flops": f2})

    teacher = teacher_measure(layer, ks) if args.teacher else None
    if args.dense_reference:                 # a library's dense attention on the same tensors, for context
        qh, kh, vh = (x.transpose(1, 2) for x in (q, k, v))   # [B, heads, N, d] views
        import torch.nn.functional as F
        for _ in range(2):
            F.scaled_dot_product_attention(qh, kh, vh)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            F.scaled_dot_product_attention(qh, kh, vh)
        e1.record(stream)
        torch.cuda.synchronize()
        dms = e0.elapsed_time(e1) / 3
        dflops = 4 * cfg.head_dim * cfg.batch * cfg.heads * cfg.n_tokens ** 2
        dense_ref = {"what": "torch.nn.functional.scaled_dot_product_attention (library), dense, same q, k, v",
                     "ms": round(dms, 3), "tflops": round(dflops / (dms * 1e-3) / 1e12, 1), "flops": dflops}
    else:
        dense_ref = None
    line = bench_line(args, layer_cfg, world, k_list(layer_cfg, args.sparsity), flops, ms_step, stages, roofline,
                      e2e, clocks, stats, sweep, teacher)
    if dense_ref is not None:
        line["dense_reference"] = dense_ref
    return line


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        import oracle.vsa_oracle as O
        from vsa_synth import get_config
        cfg = get_config(args.config)
        if args.heads:
            cfg = cfg.with_(heads=args.heads, tile_shapes=cfg.tile_shapes[:args.heads])
        pt, ph, pw = cfg.tile_shapes[0]
        k0 = O.k_from_sparsity(args.sparsity, -(-cfg.T // pt) * -(-cfg.H // ph) * -(-cfg.W // pw))
        sampler = OracleSample(cfg, args.sparsity)
        for _ in range(args.warmup):
            sampler.run()
        t0 = time.time()
        vals, walls, last = [], [], None
        for _ in range(args.steps):          # a step: one fixed sample of the layer, run in full
            last = sampler.run()
            vals.append(last["value"])
            walls.append(last["sample_s"])
        v = statistics.median(vals)
        line = {"impl": "reference", "metric": metric_for(cfg),
                "value": v, "unit": "ms", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                # what one step (sample) actually took; `value` is the layer time extrapolated from it
                "ms_per_step": round(1e3 * statistics.mean(walls), 3) if walls else 0.0,
                "extrapolated": True,
                "step": "one fixed sample of the layer (see cpu_baseline.sample), timed in full; value = the "
                        "median over steps of the whole-layer time extrapolated from each sample",
                "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic",
                "config": workload_config(cfg, args.sparsity, k0, world),
                "cpu_baseline": {**last, "value": v} if last else None,
                "e2e": {"value": v, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                "wall_s": round(time.time() - t0, 1)}
        print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        import torch
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            from vsa_synth import get_config
            cfg = get_config(args.config)
            if args.heads:
                cfg = cfg.with_(heads=args.heads, tile_shapes=cfg.tile_shapes[:args.heads])
            line["cpu_baseline"] = cpu_baseline(cfg, args.sparsity)
            # the medium workload, small enough for the oracle to run whole, beside the GPU's time for it
            med = get_config("medium")
            line["cpu_baseline"]["medium_full_layer"] = {
                "workload": "medium (24 heads, 7,680 video tokens, 75%)", "extrapolated": False,
                "oracle_ms": round(oracle_full_layer_ms(med, med.sparsity[0]), 1),
                "gpu_ms": round(gpu_layer_ms(med, med.sparsity[0]), 3)}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
