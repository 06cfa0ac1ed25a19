"""Counter-based normal draws, the synthetic 3D position embedding, and bf16 rounding."""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

# Stream identifiers: one independent SplitMix64 seed per tensor of a layer.
STREAM_Q, STREAM_K, STREAM_V, STREAM_GATE, STREAM_WQ, STREAM_WK = range(6)


def _stream_seed(seed: int, stream: int) -> np.uint64:
    # A distinct 64-bit starting state per (seed, tensor); distinct states give
    # disjoint windows of the SplitMix64 sequence for any practical length.
    return np.uint64(((seed & 0xFFFFFFFF) << 32) ^ ((stream & 0xFFFF) << 16) ^ 0x5EED)


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64_outputs(state: np.uint64, start: int, n: int) -> np.ndarray:
    """Outputs ``start .. start+n-1`` of SplitMix64 seeded with ``state``."""
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(state + i * GAMMA)


def uniform01(state: np.uint64, start: int, n: int) -> np.ndarray:
    """Uniform doubles in (0, 1]: top 53 bits of each output, plus one ulp."""
    u = splitmix64_outputs(state, start, n) >> np.uint64(11)
    return (u.astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)


def standard_normal(state: np.uint64, start: int, n: int) -> np.ndarray:
    """N(0,1) draws ``start .. start+n-1``; draw j uses outputs 2j and 2j+1."""
    out = np.empty(n, dtype=np.float64)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        u = uniform01(state, 2 * (start + c0), 2 * (c1 - c0))
        u1, u2 = u[0::2], u[1::2]
        out[c0:c1] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns the raw uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def position_embedding(T: int, H: int, W: int, d: int) -> np.ndarray:
    """Smooth sinusoidal 3D embedding, ``[T*H*W, d]`` in (t, h, w) raster order (w fastest).

    Channel c follows axis c mod 3 (t, h, w), wavelength 8 * 2**((c div 6) mod 4)
    tokens, and phase (c div 3 mod 2) * pi/2 (sine, or cosine).
    """
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    coords = np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1).astype(np.float64)
    c = np.arange(d)
    axis = c % 3
    lam = 8.0 * 2.0 ** ((c // 6) % 4)
    phase = ((c // 3) % 2) * (math.pi / 2)
    return np.sin(2.0 * math.pi * coords[:, axis] / lam[None, :] + phase[None, :])


@dataclasses.dataclass
class LayerInputs:
    """bf16 bit patterns of Q, K, V (``[B, N, heads, d]`` uint16) and the fp32 score weights."""

    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    gate: np.ndarray | None      # [d, d] fp32, mean-pool gate scoring
    w_q: np.ndarray | None       # [heads, 3d, p] fp32, TripPool scoring
    w_k: np.ndarray | None

    def as_f64(self, name: str) -> np.ndarray:
        return bf16_bits_to_f32(getattr(self, name)).astype(np.float64)


def _token_tensor(cfg, stream: int) -> np.ndarray:
    B, N, Hh, d = cfg.batch, cfg.n_tokens, cfg.heads, cfg.head_dim
    n_pre = cfg.n_prefix_tokens
    pe = position_embedding(cfg.T, cfg.H, cfg.W, d).astype(np.float32)   # [Nv, d]
    state = _stream_seed(cfg.seed, stream)
    out = np.empty((B, N, Hh, d), dtype=np.uint16)
    row = Hh * d
    flat = out.reshape(B, N, row)
    tok_block = max(1, _CHUNK // row)

    def fill(job):
        b, t0 = job
        t1 = min(N, t0 + tok_block)
        start = (b * N + t0) * row
        x = standard_normal(state, start, (t1 - t0) * row).reshape(t1 - t0, Hh, d)
        lo = max(t0, n_pre)
        if lo < t1:
            x[lo - t0:] += 0.5 * pe[lo - n_pre:t1 - n_pre][:, None, :]
        flat[b, t0:t1] = f32_to_bf16_bits(x.astype(np.float32).reshape(t1 - t0, row))

    jobs = [(b, t0) for b in range(B) for t0 in range(0, N, tok_block)]
    workers = max(1, min(len(jobs), len(os.sched_getaffinity(0))))
    if workers == 1:
        for j in jobs:
            fill(j)
    else:
        # numpy ufuncs release the GIL, so threads give a near-linear speed-up
        with concurrent.futures.ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, jobs))
    return out


def make_layer_inputs(cfg, with_qkv: bool = True) -> LayerInputs:
    """All tensors for one layer of ``cfg`` (a :class:`vsa_synth.configs.LayerConfig`)."""
    d = cfg.head_dim
    q = k = v = None
    if with_qkv:
        q = _token_tensor(cfg, STREAM_Q)
        k = _token_tensor(cfg, STREAM_K)
        v = _token_tensor(cfg, STREAM_V)
    gate = w_q = w_k = None
    if cfg.score_mode == "meanpool_gate":
        g = standard_normal(_stream_seed(cfg.seed, STREAM_GATE), 0, d * d) / math.sqrt(d)
        gate = g.astype(np.float32).reshape(d, d)
    else:
        p, three_d = cfg.proj_dim, 3 * d
        n = cfg.heads * three_d * p
        w_q = (standard_normal(_stream_seed(cfg.seed, STREAM_WQ), 0, n) / math.sqrt(three_d)).astype(np.float32)
        w_k = (standard_normal(_stream_seed(cfg.seed, STREAM_WK), 0, n) / math.sqrt(three_d)).astype(np.float32)
        w_q = w_q.reshape(cfg.heads, three_d, p)
        w_k = w_k.reshape(cfg.heads, three_d, p)
    return LayerInputs(q=q, k=k, v=v, gate=gate, w_q=w_q, w_k=w_k)
