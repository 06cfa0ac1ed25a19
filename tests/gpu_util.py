"""Helpers shared by the GPU parity tests: run the CUDA layer and check it against the oracle."""
from __future__ import annotations

import math

import numpy as np

import oracle.vsa_oracle as O
from vsa_synth import LayerConfig, bf16_bits_to_f32, make_layer_inputs

# tolerances on the attention output (bf16 inputs, fp32 accumulation)
ATOL_MAX = 2e-2
REL_L2 = 1e-2
# index parity: a kept set may differ from the oracle's only on tiles whose
# oracle score lies within this share of the row's score scale of the k-th score
TIE_REL = 1e-5
# scores: fp32 pooling and GEMMs against fp64
SCORE_REL = 1e-5


def ragged_gpu_config(d=128, score_mode="meanpool_gate", batch=1, seed=21):
    """Partial prefix tiles and per-head tile shapes with partial tiles at the grid edge."""
    return LayerConfig(
        name=f"ragged{d}", batch=batch, heads=4, head_dim=d, T=6, H=8, W=8,
        segments=(100, 30), tile_shapes=((4, 4, 4), (16, 2, 2), (2, 4, 8), (8, 4, 2)),
        score_mode=score_mode, proj_dim=d if score_mode == "meanpool_gate" else 64,
        sparsity=(0.5,), seed=seed)


def r2va_gpu_config(d=128, score_mode="meanpool_gate", k_ref=2, seed=23):
    """Text, a reference segment of 130 tokens (tiles of 64, 64 and 2 tokens), audio; the
    reference tiles are selected per video query tile with their own budget."""
    return ragged_gpu_config(d, score_mode, seed=seed).with_(
        name=f"r2va{d}", segments=(100, 130, 30), seg_ref=(0, 1, 0), k_ref=k_ref)


def no_prefix_config():
    return LayerConfig(name="noprefix", batch=1, heads=2, head_dim=128, T=8, H=8, W=8,
                       segments=(), tile_shapes=((4, 4, 4), (2, 4, 8)), score_mode="meanpool_gate",
                       proj_dim=128, sparsity=(0.75,), seed=31)


def n_video_tiles(cfg, h):
    pt, ph, pw = cfg.tile_shapes[h]
    return -(-cfg.T // pt) * -(-cfg.H // ph) * -(-cfg.W // pw)


def k_list(cfg, s):
    return [O.k_from_sparsity(s, n_video_tiles(cfg, h)) for h in range(cfg.heads)]


def to_device(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_f64(t) -> np.ndarray:
    import torch
    return bf16_bits_to_f32(t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


class LayerRun:
    """Inputs of one config on the device plus every intermediate of one GPU layer run."""

    def __init__(self, cfg, sparsity, k_per_head=None, inputs=None):
        import torch
        import tile_sparse_video_pack_b200 as T
        self.cfg = cfg
        self.inp = inputs if inputs is not None else make_layer_inputs(cfg)
        self.k = list(k_per_head) if k_per_head is not None else k_list(cfg, sparsity)
        self.plan = T.Plan.from_config(cfg, sparsity, k_per_head=self.k)
        self.bufs = self.plan.allocate(with_lse=True)
        self.bufs["op"].zero_()          # tiles past a head's own count are never written
        self.q, self.k_t, self.v = (to_device(getattr(self.inp, n)) for n in ("q", "k", "v"))
        if cfg.score_mode == "meanpool_gate":
            g = torch.from_numpy(self.inp.gate).cuda()
            self.proj_q = self.proj_k = g
        else:
            self.proj_q = torch.from_numpy(self.inp.w_q).cuda()
            self.proj_k = torch.from_numpy(self.inp.w_k).cuda()
        self.out = torch.empty_like(self.q)

    def run(self, stages=True, fused=False):
        """The layer as separate calls (fused: pack and pooling in one call), or as one
        vsa_layer_forward call (stages=False), which takes the fused path."""
        b, p = self.bufs, self.plan
        if stages:
            if fused:
                p.tile_pack_pool(self.q, self.k_t, self.v, b["qp"], b["kp"], b["vp"], b["workspace"])
                p.tile_score_pooled(self.proj_q, self.proj_k, b["scores"], b["workspace"])
            else:
                p.tile_pack(self.q, self.k_t, self.v, b["qp"], b["kp"], b["vp"])
                p.tile_score(b["qp"], b["kp"], self.proj_q, self.proj_k, b["scores"], b["workspace"])
            p.topk_select(b["scores"], b["idx"])
            if p.info.n_ref_tiles:       # R2VA budgets
                p.ref_score(b["kp"], self.proj_k, b["scores_ref"], b["workspace"])
                p.topk_select_ref(b["scores_ref"], b["idx_ref"])
                p.sparse_attn_ref(b["qp"], b["kp"], b["vp"], b["idx"], b["idx_ref"], b["op"], b["lse"])
            else:
                p.sparse_attn(b["qp"], b["kp"], b["vp"], b["idx"], b["op"], b["lse"])
            p.tile_unpack(b["op"], self.out)
        else:
            p.layer_forward(self.q, self.k_t, self.v, self.proj_q, self.proj_k, b, self.out)
        p.check()
        return self

    def ref_kept(self, b, h):
        ntv, kr = n_video_tiles(self.cfg, h), int(self.cfg.k_ref)
        return self.bufs["idx_ref"][b, h, :ntv, :kr].cpu().numpy().astype(np.int64)

    def ref_scores(self, b, h):
        ntv = n_video_tiles(self.cfg, h)
        return self.bufs["scores_ref"][b, h, :ntv, :].double().cpu().numpy()

    def kept(self, b, h):
        ntv, kh = n_video_tiles(self.cfg, h), self.k[h]
        return self.bufs["idx"][b, h, :ntv, :kh].cpu().numpy().astype(np.int64)

    def scores(self, b, h):
        ntv = n_video_tiles(self.cfg, h)
        return self.bufs["scores"][b, h, :ntv, :ntv].double().cpu().numpy()


def check_topk_rows(kept_gpu: np.ndarray, scores_oracle: np.ndarray, k: int, tie_rel=TIE_REL):
    """Every row: ascending, distinct, in range; equal to the oracle's set except on near-ties."""
    n = scores_oracle.shape[1]
    mismatched = 0
    for i in range(scores_oracle.shape[0]):
        row = kept_gpu[i]
        assert row.shape == (k,)
        assert np.all(np.diff(row) > 0) and row[0] >= 0 and row[-1] < n, (i, row)
        want = O.topk_row(scores_oracle[i], k)
        if np.array_equal(row, want):
            continue
        mismatched += 1
        s = scores_oracle[i]
        kth = np.sort(s)[::-1][k - 1]
        scale = np.max(np.abs(s))
        diff = np.setxor1d(row, want)
        assert np.all(np.abs(s[diff] - kth) <= tie_rel * scale), (i, diff, s[diff], kth)
    return mismatched


def check_close(got: np.ndarray, want: np.ndarray, atol=ATOL_MAX, rel_l2=REL_L2):
    err = np.abs(got - want)
    assert np.all(np.isfinite(got))
    mx = float(err.max()) if err.size else 0.0
    rl2 = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    assert mx <= atol and rl2 <= rel_l2, (mx, rl2)
    return mx, rl2


def oracle_inputs_f64(inp):
    return inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v")


def scale_of(cfg):
    return 1.0 / math.sqrt(cfg.head_dim)
