"""The layer straight from token-major Q, K, V (no packed copies, the slower opt-in path) against
the packed path.

vsa_tile_pool + vsa_sparse_attn_direct load every tile with one multi-dimensional TMA box
(a prefix tile: 64 tokens of its segment; a video tile: its block of the (T, H, W) grid) and
write O token-major. Every other step is the packed path's, so the pooled scores, the output
and the log-sum-exp must equal those of vsa_tile_pack_pool + vsa_sparse_attn +
vsa_tile_unpack bit for bit; the packed path itself is checked against the oracle elsewhere
(tests/test_gpu_parity.py). The ragged configurations hold partial prefix tiles, video tiles
cut by the grid's far edge in t, four distinct head-aware tile shapes and head_dim 64.
"""
import pytest

from gpu_util import LayerRun, ragged_gpu_config
from vsa_synth import LayerConfig, get_config

pytestmark = pytest.mark.gpu


def _run_both(cfg, sparsity):
    import torch
    r = LayerRun(cfg, sparsity)
    p, b = r.plan, r.bufs
    assert p.info.direct_attn == 1
    b["lse"].zero_()
    # packed path
    p.tile_pack_pool(r.q, r.k_t, r.v, b["qp"], b["kp"], b["vp"], b["workspace"])
    p.tile_score_pooled(r.proj_q, r.proj_k, b["scores"], b["workspace"])
    p.topk_select(b["scores"], b["idx"])
    b["op"].zero_()
    p.sparse_attn(b["qp"], b["kp"], b["vp"], b["idx"], b["op"], b["lse"])
    o_packed = torch.zeros_like(r.q)
    p.tile_unpack(b["op"], o_packed)
    p.check()
    scores_packed, idx_packed, lse_packed = b["scores"].clone(), b["idx"].clone(), b["lse"].clone()
    # direct path on the same plan
    b["scores"].zero_()
    b["lse"].zero_()
    p.tile_pool(r.q, r.k_t, b["workspace"])
    p.tile_score_pooled(r.proj_q, r.proj_k, b["scores"], b["workspace"])
    p.topk_select(b["scores"], b["idx"])
    o_direct = torch.zeros_like(r.q)
    p.sparse_attn_direct(r.q, r.k_t, r.v, b["idx"], o_direct, b["lse"])
    p.check()
    return r, (scores_packed, idx_packed, lse_packed, o_packed), (b["scores"], b["idx"], b["lse"], o_direct)


@pytest.mark.parametrize("name", ["ragged128", "ragged64_tripool", "medium", "full_2heads"])
def test_direct_path_equals_packed_path_bit_for_bit(name):
    import torch
    cfg = {"ragged128": lambda: ragged_gpu_config(128),
           "ragged64_tripool": lambda: ragged_gpu_config(64, "tripool"),
           "medium": lambda: get_config("medium"),
           "full_2heads": lambda: get_config("full").with_(heads=2, tile_shapes=get_config("full").tile_shapes[:2]),
           }[name]()
    r, packed, direct = _run_both(cfg, 0.5 if cfg.n_video_tokens < 20000 else 0.75)
    sp, ip, lp, op = packed
    sd, idd, ld, od = direct
    assert torch.equal(sp.view(torch.int32), sd.view(torch.int32)), "pooled scores differ"
    assert torch.equal(ip, idd)
    assert torch.equal(op.view(torch.int16), od.view(torch.int16)), "outputs differ"
    assert torch.equal(lp.view(torch.int32), ld.view(torch.int32)), "log-sum-exp differs"


def test_direct_layer_allocates_no_packed_tiles_and_matches_the_packed_layer():
    import torch
    import tile_sparse_video_pack_b200 as T
    r = LayerRun(ragged_gpu_config(128), 0.5)
    layer = T.TileSparseAttention(r.plan, r.proj_q, r.proj_k, direct=True)
    assert layer.direct and layer.bufs["qp"] is None and layer.bufs["op"] is None
    out = layer(r.q, r.k_t, r.v)
    packed = T.TileSparseAttention(r.plan, r.proj_q, r.proj_k)
    assert not packed.direct and packed.bufs["qp"] is not None
    ref = packed(r.q, r.k_t, r.v)
    r.plan.check()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_plans_the_boxes_cannot_express_are_refused():
    import torch
    import tile_sparse_video_pack_b200 as T
    # W = 10 with pw = 4: the last tile along w is partial, so its tokens are not one box
    cfg = LayerConfig(name="partial_w", batch=1, heads=2, head_dim=64, T=4, H=8, W=10, segments=(64,),
                      tile_shapes=((4, 4, 4), (4, 4, 4)), score_mode="meanpool_gate", proj_dim=64,
                      sparsity=(0.5,), seed=9)
    r = LayerRun(cfg, 0.5)
    assert r.plan.info.direct_attn == 0
    with pytest.raises(T.VsaError) as e:
        r.plan.sparse_attn_direct(r.q, r.k_t, r.v, r.bufs["idx"], torch.zeros_like(r.q))
    assert e.value.status == 2                        # VSA_ERR_UNSUPPORTED
    with pytest.raises(T.VsaError) as e:
        r.plan.tile_pool(r.q, r.k_t, r.bufs["workspace"])
    assert e.value.status == 2
    # batch 2: one box map cannot span the batches
    r2 = LayerRun(ragged_gpu_config(128, batch=2), 0.5)
    assert r2.plan.info.direct_attn == 0
    with pytest.raises(ValueError):
        T.TileSparseAttention(r.plan, r.proj_q, r.proj_k, direct=True)
