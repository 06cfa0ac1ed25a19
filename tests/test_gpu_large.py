"""GPU parity at full size, in the launch configuration the benchmark times.

The oracle cannot run a 112k-token layer in full, so it checks what it can one
by one: complete score rows and top-k sets for sampled heads, and attention
rows for sampled query tiles (prefix and video) of those heads. Properties that
hold at any size are checked on every row.
"""
import numpy as np
import pytest

import oracle.vsa_oracle as O
from gpu_util import (LayerRun, bf16_to_f64, check_close, check_topk_rows, n_video_tiles)
from vsa_synth import bf16_bits_to_f32, get_config

pytestmark = pytest.mark.gpu


def head_slice(cfg, inp, h):
    """Single-head config and fp64 inputs of head h (so the oracle handles one head at a time)."""
    sub = cfg.with_(heads=1, tile_shapes=(cfg.tile_shapes[h],))
    f = lambda bits: bf16_bits_to_f32(bits[:, :, h:h + 1]).astype(np.float64)
    wq = inp.w_q[h:h + 1] if inp.w_q is not None else None
    wk = inp.w_k[h:h + 1] if inp.w_k is not None else None
    return sub, f(inp.q), f(inp.k), f(inp.v), wq, wk


def all_rows_valid(r):
    import torch
    idx = r.bufs["idx"]
    for h in range(r.cfg.heads):
        ntv, kh = n_video_tiles(r.cfg, h), r.k[h]
        x = idx[:, h, :ntv, :kh]
        assert bool((x[..., 1:] > x[..., :-1]).all()) and int(x.min()) >= 0 and int(x.max()) < ntv
    assert bool(torch.isfinite(r.out.float()).all())


def sampled_parity(r, heads, n_video_samples=6, seed=0, out=None, qk_fp8=False):
    """Complete score rows and top-k sets of the sampled heads, and attention rows of sampled
    query tiles against the oracle (``out``: another output of the same run to check instead,
    ``qk_fp8``: against the oracle's fp8 model)."""
    rng = np.random.default_rng(seed)
    cfg = r.cfg
    got_all = None if out is None else bf16_to_f64(out)
    for h in heads:
        sub, q, k, v, wq, wk = head_slice(cfg, r.inp, h)
        til = O.head_tiling(sub, 0)
        s_or = O.tile_scores(q[0, :, 0], k[0, :, 0], til, sub, 0, r.inp.gate, wq, wk)
        kept = r.kept(0, h)
        check_topk_rows(kept, s_or, r.k[h])
        npre, nv = til.n_prefix, til.n_video
        qt = sorted({0, npre // 2, npre - 1} if npre else set())
        qt += sorted({npre, npre + 1, npre + nv - 1, *(npre + rng.integers(0, nv, n_video_samples))})
        kept_ref = {0: r.ref_kept(0, h)} if r.plan.info.n_ref_tiles else None
        res = O.run_layer(sub, q, k, v, [r.k[h]], gate=r.inp.gate, w_q=wq, w_k=wk,
                          query_tiles={0: qt}, kept={0: kept}, kept_ref=kept_ref, qk_fp8=qk_fp8)
        if got_all is None:
            got_all = bf16_to_f64(r.out)
        rows = np.concatenate([til.all[t] for t in qt])
        check_close(got_all[0, rows, h], res.out[0, rows, 0])


@pytest.mark.parametrize("sparsity", [0.75, 0.9])
def test_full_clip(sparsity):
    cfg = get_config("full")
    r = LayerRun(cfg, sparsity).run(fused=True)          # the bench's path: pack fused with pooling
    all_rows_valid(r)
    sampled_parity(r, heads=[0, 13])
    want_pairs = O.attention_flops(cfg, r.k) // (4 * cfg.head_dim)
    assert r.plan.stats()["computed_pairs"] == want_pairs


@pytest.mark.parametrize("sparsity", [0.9, 0.95])
def test_veda_head_aware(sparsity):
    cfg = get_config("veda")
    r = LayerRun(cfg, sparsity).run(fused=True)
    all_rows_valid(r)
    sampled_parity(r, heads=[0, 1, 2, 3])     # one head of each tile shape


def test_long_clip_dense_and_sparse():
    import torch
    import torch.nn.functional as F
    cfg = get_config("long")
    r = LayerRun(cfg, 0.0).run(fused=True)     # k = all tiles: dense attention
    all_rows_valid(r)
    sampled_parity(r, heads=[5], n_video_samples=3)
    # cross-check (not the oracle): torch dense attention on two heads
    for h in (0, 17):
        # [B, N, heads, d] -> [B, 1, N, d] for one head
        qh, kh, vh = (x[:, :, h].unsqueeze(1) for x in (r.q, r.k_t, r.v))
        ref = F.scaled_dot_product_attention(qh, kh, vh).float()
        got = r.out[:, :, h].unsqueeze(1).float()
        err = (got - ref).abs().max().item()
        assert err <= 2e-2, err
    r2 = LayerRun(cfg, 0.9, inputs=r.inp).run(fused=True)
    all_rows_valid(r2)
    sampled_parity(r2, heads=[3], n_video_samples=3)


_long_inputs = {}


@pytest.mark.parametrize("sparsity", [0.5, 0.75, 0.95])
def test_long_clip_sweep(sparsity):
    """The rest of the long clip's sparsity sweep (0 and 0.9 above), on sampled rows."""
    cfg = get_config("long")
    if "inp" not in _long_inputs:
        from vsa_synth import make_layer_inputs
        _long_inputs["inp"] = make_layer_inputs(cfg)
    r = LayerRun(cfg, sparsity, inputs=_long_inputs["inp"]).run(fused=True)
    all_rows_valid(r)
    sampled_parity(r, heads=[11], n_video_samples=3)
    want_pairs = O.attention_flops(cfg, r.k) // (4 * cfg.head_dim)
    assert r.plan.stats()["computed_pairs"] == want_pairs


def test_full_clip_fp8():
    """The fp8 Q K^T path at full size, against the oracle's fp8 model on sampled rows."""
    import torch
    cfg = get_config("full")
    r = LayerRun(cfg, 0.75).run(fused=True)
    f8 = r.plan.allocate_fp8()
    b = r.bufs
    r.plan.tile_pack_pool_fp8(r.q, r.k_t, r.v, b["qp"], b["kp"], b["vp"], f8["qp8"], f8["kp8"], f8["q_scale"],
                              f8["k_scale"], b["workspace"])
    op8 = torch.zeros_like(b["op"])
    r.plan.sparse_attn_fp8(f8["qp8"], f8["kp8"], f8["q_scale"], f8["k_scale"], b["vp"], b["idx"], op8)
    out8 = torch.empty_like(r.out)
    r.plan.tile_unpack(op8, out8)
    r.plan.check()
    assert bool(torch.isfinite(out8.float()).all())
    sampled_parity(r, heads=[7], out=out8, qk_fp8=True)


def test_r2va_full_clip():
    """R2VA budgets at full size: 32 of 60 reference tiles and 32 of 1680 video tiles."""
    cfg = get_config("r2va").with_(heads=4, tile_shapes=get_config("r2va").tile_shapes[:4])
    r = LayerRun(cfg, cfg.sparsity[0]).run(fused=True)
    all_rows_valid(r)
    for h in (0, 3):
        sub, q, k, v, wq, wk = head_slice(cfg, r.inp, h)
        til = O.head_tiling(sub, 0)
        ref = O.ref_tiles(sub)
        want = O.tile_scores(q[0, :, 0], k[0, :, 0], til, sub, 0, r.inp.gate, key_tiles=[til.prefix[t] for t in ref])
        check_topk_rows(r.ref_kept(0, h), want, cfg.k_ref)
    sampled_parity(r, heads=[0, 3], n_video_samples=4)
