"""The five layer workloads used by the tests and the benchmark.

Each one is a single attention layer of a video-diffusion transformer whose
sequence is a conditioning prefix (text, reference image, reference audio
segments, in that order) followed by a video latent grid T x H x W in
(t, h, w) raster order. Sizes follow the 1344x768, ~5 s clip class that the
Ref2VA VSA and Veda pages measure on (104k-token layers); the tiny and medium
cases exist so that the fp64 oracle finishes in seconds.
"""
from __future__ import annotations

import dataclasses

UNIFORM_444 = (4, 4, 4)
VEDA_HEAD_CYCLE = ((4, 4, 4), (1, 8, 8), (16, 2, 2), (2, 4, 8))


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    batch: int
    heads: int
    head_dim: int
    T: int
    H: int
    W: int
    segments: tuple            # prefix segment lengths, in sequence order
    tile_shapes: tuple         # one (pt, ph, pw) per head
    score_mode: str            # "meanpool_gate" or "tripool"
    proj_dim: int              # width of the projected pooled descriptors
    sparsity: tuple            # video-key sparsity levels this workload is run at
    seed: int
    note: str = ""
    # Reference segments (R2VA budget variant): seg_ref[s] = 1 marks prefix segment s as a
    # reference stream whose tiles each video query tile selects with its own budget k_ref;
    # the other segments stay dense. Empty: every prefix tile is kept (the default layer).
    seg_ref: tuple = ()
    k_ref: int = 0

    @property
    def n_prefix_tokens(self) -> int:
        return int(sum(self.segments))

    @property
    def n_video_tokens(self) -> int:
        return self.T * self.H * self.W

    @property
    def n_tokens(self) -> int:
        return self.n_prefix_tokens + self.n_video_tokens

    def with_(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


def _uniform(heads):
    return tuple(UNIFORM_444 for _ in range(heads))


def _veda(heads):
    return tuple(VEDA_HEAD_CYCLE[h % len(VEDA_HEAD_CYCLE)] for h in range(heads))


CONFIGS = {
    "tiny": LayerConfig(
        name="tiny", batch=1, heads=2, head_dim=64, T=4, H=8, W=8,
        segments=(64, 64), tile_shapes=_uniform(2), score_mode="meanpool_gate",
        proj_dim=64, sparsity=(0.5,), seed=0,
        note="4 video tiles, top-2; 2 prefix tiles"),
    "medium": LayerConfig(
        name="medium", batch=1, heads=24, head_dim=128, T=8, H=24, W=40,
        segments=(512, 960, 128), tile_shapes=_uniform(24), score_mode="meanpool_gate",
        proj_dim=128, sparsity=(0.75,), seed=1,
        note="120 video tiles, top-30; 25 prefix tiles"),
    "full": LayerConfig(
        name="full", batch=1, heads=24, head_dim=128, T=28, H=48, W=80,
        segments=(512, 3840, 640), tile_shapes=_uniform(24), score_mode="meanpool_gate",
        proj_dim=128, sparsity=(0.75, 0.9), seed=2,
        note="1344x768-like clip: 107,520 video tokens, 1,680 tiles; 78 prefix tiles"),
    "veda": LayerConfig(
        name="veda", batch=1, heads=24, head_dim=128, T=28, H=48, W=80,
        segments=(512, 3840, 640), tile_shapes=_veda(24), score_mode="tripool",
        proj_dim=64, sparsity=(0.9, 0.95), seed=3,
        note="head-aware tiling, TripPool scoring"),
    "r2va": LayerConfig(
        name="r2va", batch=1, heads=24, head_dim=128, T=28, H=48, W=80,
        segments=(512, 3840, 640), tile_shapes=_uniform(24), score_mode="meanpool_gate",
        proj_dim=128, sparsity=(1.0 - 32 / 1680,), seed=5, seg_ref=(0, 1, 0), k_ref=32,
        note="R2VA budgets: 32 of the 60 reference-image tiles + 32 of 1680 video tiles per query "
             "tile; text and audio tiles dense"),
    "long": LayerConfig(
        name="long", batch=1, heads=24, head_dim=128, T=60, H=48, W=80,
        segments=(512, 3840, 1280), tile_shapes=_uniform(24), score_mode="meanpool_gate",
        proj_dim=128, sparsity=(0.0, 0.5, 0.75, 0.9, 0.95), seed=4,
        note="long clip, 230,400 video tokens, sparsity sweep"),
}


def get_config(name: str) -> LayerConfig:
    return CONFIGS[name]
