"""GPU parity: every stage of the CUDA layer against the fp64 oracle on seeded inputs.

Sizes span several tiles, partial prefix tiles, head-specific partial video
tiles, a batch of two, no prefix, head_dim 64 and 128, both scorers.
"""
import numpy as np
import pytest

import oracle.vsa_oracle as O
from gpu_util import (LayerRun, bf16_to_f64, check_close, check_topk_rows, k_list, n_video_tiles,
                      no_prefix_config, oracle_inputs_f64, ragged_gpu_config, scale_of, SCORE_REL, to_device)
from vsa_synth import get_config

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": (lambda: get_config("tiny"), 0.5),
    "ragged128": (lambda: ragged_gpu_config(128), 0.5),
    "ragged64_tripool": (lambda: ragged_gpu_config(64, "tripool"), 0.5),
    "ragged128_batch2": (lambda: ragged_gpu_config(128, batch=2, seed=22), 0.75),
    "noprefix": (no_prefix_config, 0.75),
    "medium": (lambda: get_config("medium"), 0.75),
}

_runs = {}


def gpu_run(name, fused=False):
    if (name, fused) not in _runs:
        make, s = CASES[name]
        _runs[name, fused] = LayerRun(make(), s).run(fused=fused)
    return _runs[name, fused]


@pytest.mark.parametrize("fused", [False, True], ids=["pack", "pack_pool"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_pack_bit_exact(name, fused):
    r = gpu_run(name, fused)
    q, k, v = oracle_inputs_f64(r.inp)
    for src, packed in ((q, r.bufs["qp"]), (k, r.bufs["kp"]), (v, r.bufs["vp"])):
        want, counts = O.pack(src, r.cfg)
        got = bf16_to_f64(packed)
        assert got.shape == want.shape
        assert np.array_equal(got, want)
    # unpack(pack(x)) == x, bit for bit
    import torch
    back = torch.empty_like(r.q)
    r.plan.tile_unpack(r.bufs["qp"], back)
    r.plan.check()
    assert torch.equal(back.view(torch.int16), r.q.view(torch.int16))


@pytest.mark.parametrize("fused", [False, True], ids=["pool", "pack_pool"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_scores_and_topk(name, fused):
    r = gpu_run(name, fused)
    q, k, v = oracle_inputs_f64(r.inp)
    for b in range(r.cfg.batch):
        for h in range(r.cfg.heads):
            til = O.head_tiling(r.cfg, h)
            s_or = O.tile_scores(q[b, :, h], k[b, :, h], til, r.cfg, h, r.inp.gate, r.inp.w_q, r.inp.w_k)
            s_gpu = r.scores(b, h)
            scale = np.max(np.abs(s_or), axis=1, keepdims=True)
            assert np.all(np.abs(s_gpu - s_or) <= SCORE_REL * scale), (b, h)
            kept = r.kept(b, h)
            check_topk_rows(kept, s_or, r.k[h])
            # the same decision taken in the GPU's own precision is exact
            for i in range(kept.shape[0]):
                assert np.array_equal(kept[i], O.topk_row(s_gpu[i], r.k[h]))


@pytest.mark.parametrize("fused", [False, True], ids=["pack", "pack_pool"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_attention_matches_oracle(name, fused):
    r = gpu_run(name, fused)
    q, k, v = oracle_inputs_f64(r.inp)
    kept = {(b, h): r.kept(b, h) for b in range(r.cfg.batch) for h in range(r.cfg.heads)}
    res = O.run_layer(r.cfg, q, k, v, r.k, gate=r.inp.gate, w_q=r.inp.w_q, w_k=r.inp.w_k, kept=kept)
    got = bf16_to_f64(r.out)
    check_close(got, res.out)
    # log-sum-exp per row, compared in the packed layout over each head's own tiles
    # (padding slots are 0 on both sides; tiles past a head's tile count are not written)
    lse_want, counts = O.pack(res.lse[..., None], r.cfg)
    lse_want = lse_want[..., 0]                          # [B, heads, NT, 64]
    lse_got = r.bufs["lse"].double().cpu().numpy()
    exists = counts > 0                                  # [heads, NT]
    assert lse_got.shape == lse_want.shape
    assert np.max(np.abs(lse_got[:, exists] - lse_want[:, exists])) <= 1e-3
    # padding rows inside a head's tiles are zero
    op = bf16_to_f64(r.bufs["op"])
    slot = np.arange(64)[None, None, :]
    pad = (slot >= counts[:, :, None]) & exists[:, :, None]
    assert np.all(op[:, pad] == 0.0)
    # the pair count reported in the stats is the oracle's
    assert r.plan.stats()["computed_pairs"] == res.computed_pairs


@pytest.mark.parametrize("name", ["tiny", "ragged128", "ragged64_tripool", "noprefix"])
def test_dense_when_k_is_all(name):
    make, _ = CASES[name]
    cfg = make()
    r = LayerRun(cfg, 0.0, k_per_head=[n_video_tiles(cfg, h) for h in range(cfg.heads)]).run()
    q, k, v = oracle_inputs_f64(r.inp)
    want = O.dense_attention(q, k, v, scale_of(cfg))
    check_close(bf16_to_f64(r.out), want)


def test_layer_forward_equals_stages_and_is_deterministic():
    import torch
    r = gpu_run("ragged128_batch2", fused=True)
    first = r.out.clone()
    r.run(stages=False)                    # vsa_layer_forward takes the fused path
    assert torch.equal(first.view(torch.int16), r.out.view(torch.int16))
    r.run(stages=True, fused=True)
    assert torch.equal(first.view(torch.int16), r.out.view(torch.int16))


@pytest.mark.parametrize("name", sorted(CASES))
def test_pack_pool_descriptors_match_pool_stage(name):
    """The fused pass writes the score stage's pooled descriptors: same layout, values equal
    up to fp32 summation order (the separate pool sums rows in order, the fused one in a tree)."""
    import torch
    r0, r1 = gpu_run(name, False), gpu_run(name, True)
    n = r0.cfg.batch * r0.cfg.heads * r0.plan.info.ntv_max
    kd = 3 * r0.cfg.head_dim if r0.cfg.score_mode == "tripool" else r0.cfg.head_dim
    off = ((n * kd * 4 + 255) // 256) * 256
    for base in (0, off):                  # pooled Q, then pooled K
        a = r0.bufs["workspace"][base:base + n * kd * 4].view(torch.float32).view(n, kd)
        b = r1.bufs["workspace"][base:base + n * kd * 4].view(torch.float32).view(n, kd)
        for bh in range(r0.cfg.batch * r0.cfg.heads):
            h = bh % r0.cfg.heads
            rows = slice(bh * r0.plan.info.ntv_max, bh * r0.plan.info.ntv_max + n_video_tiles(r0.cfg, h))
            x, y = a[rows].double().cpu().numpy(), b[rows].double().cpu().numpy()
            assert np.max(np.abs(x - y)) <= 1e-5 * max(1.0, np.max(np.abs(x)))


def test_k_one_and_edges():
    cfg = ragged_gpu_config(128, seed=23)
    r = LayerRun(cfg, 1.0).run()          # k = 1 for every head
    assert r.k == [1] * cfg.heads
    q, k, v = oracle_inputs_f64(r.inp)
    kept = {h: r.kept(0, h) for h in range(cfg.heads)}
    res = O.run_layer(cfg, q, k, v, r.k, gate=r.inp.gate, kept=kept)
    check_close(bf16_to_f64(r.out), res.out)
    for h in range(cfg.heads):
        til = O.head_tiling(cfg, h)
        s_or = O.tile_scores(q[0, :, h], k[0, :, h], til, cfg, h, r.inp.gate)
        check_topk_rows(r.kept(0, h), s_or, 1)


def test_bad_index_is_latched_not_read():
    import tile_sparse_video_pack_b200 as T
    import torch
    r = LayerRun(get_config("tiny"), 0.5).run()
    idx = r.bufs["idx"].clone()
    idx[0, 0, 1, 0] = 99                 # out of range
    op = torch.zeros_like(r.bufs["op"])
    r.plan.sparse_attn(r.bufs["qp"], r.bufs["kp"], r.bufs["vp"], idx, op)
    with pytest.raises(T.VsaError) as e:
        r.plan.check()
    assert e.value.status == 5
    # the pair holding that query tile was skipped; the other blocks were written
    assert torch.count_nonzero(op[0, 1]) > 0
    r.plan.check()                       # the error was cleared


def test_argument_errors():
    import tile_sparse_video_pack_b200 as T
    import torch
    r = gpu_run("tiny")
    assert T.vsa.library().vsa_sparse_attn(r.plan._h, None, None, None, None, None, None, None, None) == 1
    with pytest.raises(TypeError):
        r.plan.tile_pack(r.q.float(), None, None, r.bufs["qp"], None, None)
    with pytest.raises(ValueError):
        r.plan.topk_select(r.bufs["scores"][:, :, :1].contiguous(), r.bufs["idx"])
    # misaligned device pointer is refused by the library itself
    bad = torch.empty(r.bufs["qp"].numel() + 8, dtype=torch.bfloat16, device="cuda")[1:]
    st = T.vsa.library().vsa_tile_unpack(r.plan._h, T.vsa.ctypes.c_void_p(bad.data_ptr()),
                                         T.vsa.ctypes.c_void_p(r.out.data_ptr()), None)
    assert st == 1


def test_running_max_jumps_late_in_the_row():
    """Keys of the last video frames scaled by 6: their scores exceed every earlier
    block's by far more than the lazy threshold, so the running max is raised late in
    the row and the partial outputs are rescaled (prefix rows see every key)."""
    import dataclasses
    from vsa_synth import bf16_bits_to_f32, f32_to_bf16_bits
    from vsa_synth.generate import make_layer_inputs
    cfg = ragged_gpu_config(128)
    inp = make_layer_inputs(cfg)
    k = bf16_bits_to_f32(inp.k).reshape(cfg.batch, -1, cfg.heads, cfg.head_dim)
    n_last = cfg.H * cfg.W * 2                       # tokens of the last two frames
    k[:, -n_last:] *= 6.0
    inp = dataclasses.replace(inp, k=f32_to_bf16_bits(k).reshape(inp.k.shape))
    r = LayerRun(cfg, 0.5, inputs=inp).run()
    q, kk, v = oracle_inputs_f64(r.inp)
    kept = {(b, h): r.kept(b, h) for b in range(cfg.batch) for h in range(cfg.heads)}
    res = O.run_layer(cfg, q, kk, v, r.k, gate=r.inp.gate, w_q=r.inp.w_q, w_k=r.inp.w_k, kept=kept)
    # the jump is real: some prefix row's largest logit comes from the scaled keys
    s = np.einsum("nd,md->nm", q[0, :64, 0], kk[0, :, 0]) * scale_of(cfg)
    assert np.any(np.argmax(s, axis=1) >= s.shape[1] - n_last)
    check_close(bf16_to_f64(r.out), res.out)
