"""GPU parity of the per-call k: one plan, created at its largest k, runs smaller sparsities.

vsa_topk_select, vsa_sparse_attn (and the fp8 / R2VA / overlap calls) take the kept
tiles per head of each call as a host array; NULL keeps the plan's own k. The index
table's row width stays the plan's k_max. Each call's selection and output must match
the oracle run at that call's k (Ref2VA VSA README: "75% video sparsity top-k";
BSAI VedaSparse README, "Nodes": keep_percent per run).
"""
import numpy as np
import pytest

import oracle.vsa_oracle as O
import tile_sparse_video_pack_b200 as T
from gpu_util import (LayerRun, bf16_to_f64, check_close, check_topk_rows, k_list, oracle_inputs_f64,
                      ragged_gpu_config)
from vsa_synth import get_config

pytestmark = pytest.mark.gpu


def run_at(r, ks):
    """The layer's calls on r's plan and buffers with this call's k per head."""
    b, p = r.bufs, r.plan
    b["op"].zero_()
    p.tile_pack_pool(r.q, r.k_t, r.v, b["qp"], b["kp"], b["vp"], b["workspace"])
    p.tile_score_pooled(r.proj_q, r.proj_k, b["scores"], b["workspace"])
    p.topk_select(b["scores"], b["idx"], k_per_head=ks)
    p.sparse_attn(b["qp"], b["kp"], b["vp"], b["idx"], b["op"], b["lse"], k_per_head=ks)
    p.tile_unpack(b["op"], r.out)
    p.check()


@pytest.mark.parametrize("cfg_name", ["ragged128", "ragged64_tripool", "medium"])
def test_one_plan_runs_several_sparsities(cfg_name):
    cfg = {"ragged128": lambda: ragged_gpu_config(128),
           "ragged64_tripool": lambda: ragged_gpu_config(64, "tripool"),
           "medium": lambda: get_config("medium")}[cfg_name]()
    r = LayerRun(cfg, 0.25)                      # the plan holds the largest k
    q, k, v = oracle_inputs_f64(r.inp)
    heads = range(cfg.heads) if cfg.heads <= 4 else (0, 7, 23)
    for s in (0.75, 0.9):
        ks = k_list(cfg, s)
        assert all(a <= b for a, b in zip(ks, r.k))
        run_at(r, ks)
        kept = {}
        for bb in range(cfg.batch):
            for h in range(cfg.heads):
                ntv = r.plan.info.ntv[h]
                kept[bb, h] = r.bufs["idx"][bb, h, :ntv, :ks[h]].cpu().numpy().astype(np.int64)
        for h in heads:
            til = O.head_tiling(cfg, h)
            s_or = O.tile_scores(q[0, :, h], k[0, :, h], til, cfg, h, r.inp.gate, r.inp.w_q, r.inp.w_k)
            check_topk_rows(kept[0, h], s_or, ks[h])
        res = O.run_layer(cfg, q, k, v, ks, gate=r.inp.gate, w_q=r.inp.w_q, w_k=r.inp.w_k, kept=kept,
                          heads=list(heads))
        got = bf16_to_f64(r.out)
        for h in heads:
            check_close(got[:, :, h], res.out[:, :, h])
        # the computed-pair count follows the call's k, not the plan's
        want = (res.computed_pairs if len(heads) == cfg.heads
                else O.attention_flops(cfg, ks) // (4 * cfg.head_dim))
        assert r.plan.stats()["computed_pairs"] == want


def test_null_k_is_the_plans_own():
    cfg = ragged_gpu_config(128)
    r = LayerRun(cfg, 0.5).run(fused=True)
    ref = r.out.clone()
    run_at(r, r.k)
    assert np.array_equal(bf16_to_f64(r.out), bf16_to_f64(ref))


def test_bad_k_is_rejected_before_launch():
    cfg = ragged_gpu_config(128)
    r = LayerRun(cfg, 0.5)
    b, p = r.bufs, r.plan
    kmax = r.plan.info.k_max      # the index tables' row width: no call may keep more
    for bad in ([0] + r.k[1:], [kmax + 1] + r.k[1:], r.k[:-1] + [r.plan.info.ntv[cfg.heads - 1] + 1],
                [-3] * cfg.heads):
        for call in (lambda: p.topk_select(b["scores"], b["idx"], k_per_head=bad),
                     lambda: p.sparse_attn(b["qp"], b["kp"], b["vp"], b["idx"], b["op"], k_per_head=bad)):
            with pytest.raises(T.VsaError) as e:
                call()
            assert e.value.status == 1
    with pytest.raises(ValueError):
        p.topk_select(b["scores"], b["idx"], k_per_head=r.k[:-1])
    p.check()
