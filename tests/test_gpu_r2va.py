"""GPU parity of the R2VA budget variant: reference tiles scored, selected with their own
top-k, and attended by each video query tile together with the dense prefix segments."""
import numpy as np
import pytest

import oracle.vsa_oracle as O
from gpu_util import (LayerRun, SCORE_REL, bf16_to_f64, check_close, check_topk_rows, oracle_inputs_f64,
                      r2va_gpu_config)
from vsa_synth import get_config

pytestmark = pytest.mark.gpu

CASES = {
    "r2va128": (lambda: r2va_gpu_config(128), 0.5),
    "r2va64_tripool": (lambda: r2va_gpu_config(64, "tripool", seed=24), 0.5),
    "medium_r2va": (lambda: get_config("medium").with_(name="medium_r2va", seg_ref=(0, 1, 0), k_ref=4,
                                                       heads=6, tile_shapes=get_config("medium").tile_shapes[:6]),
                    0.75),
}

_runs = {}


def run(name):
    if name not in _runs:
        make, s = CASES[name]
        _runs[name] = LayerRun(make(), s).run(fused=True)
    return _runs[name]


@pytest.mark.parametrize("name", sorted(CASES))
def test_reference_scores_and_selection(name):
    r = run(name)
    q, k, v = oracle_inputs_f64(r.inp)
    ref = O.ref_tiles(r.cfg)
    assert r.plan.info.n_ref_tiles == len(ref)
    for b in range(r.cfg.batch):
        for h in range(r.cfg.heads):
            til = O.head_tiling(r.cfg, h)
            want = O.tile_scores(q[b, :, h], k[b, :, h], til, r.cfg, h, r.inp.gate, r.inp.w_q, r.inp.w_k,
                                 key_tiles=[til.prefix[t] for t in ref])
            got = r.ref_scores(b, h)
            scale = np.max(np.abs(want), axis=1, keepdims=True)
            assert np.all(np.abs(got - want) <= SCORE_REL * scale), (b, h)
            kept = r.ref_kept(b, h)
            check_topk_rows(kept, want, r.cfg.k_ref)
            for i in range(kept.shape[0]):
                assert np.array_equal(kept[i], O.topk_row(got[i], r.cfg.k_ref))


@pytest.mark.parametrize("name", sorted(CASES))
def test_attention_with_reference_budget_matches_oracle(name):
    r = run(name)
    q, k, v = oracle_inputs_f64(r.inp)
    kept = {(b, h): r.kept(b, h) for b in range(r.cfg.batch) for h in range(r.cfg.heads)}
    kept_ref = {(b, h): r.ref_kept(b, h) for b in range(r.cfg.batch) for h in range(r.cfg.heads)}
    res = O.run_layer(r.cfg, q, k, v, r.k, gate=r.inp.gate, w_q=r.inp.w_q, w_k=r.inp.w_k, kept=kept,
                      kept_ref=kept_ref)
    check_close(bf16_to_f64(r.out), res.out)
    assert r.plan.stats()["computed_pairs"] == res.computed_pairs


def test_layer_forward_refuses_reference_plans():
    import tile_sparse_video_pack_b200 as T
    r = run("r2va128")
    with pytest.raises(T.vsa.VsaError, match="UNSUPPORTED"):
        r.plan.layer_forward(r.q, r.k_t, r.v, r.proj_q, r.proj_k, r.bufs, r.out)


def test_bad_reference_index_is_latched():
    import torch
    import tile_sparse_video_pack_b200 as T
    r = LayerRun(r2va_gpu_config(128), 0.5).run(fused=True)
    b = r.bufs
    b["idx_ref"][0, 0, 0, :] = torch.tensor([1, 0], dtype=torch.int32)   # not ascending
    r.plan.sparse_attn_ref(b["qp"], b["kp"], b["vp"], b["idx"], b["idx_ref"], b["op"], b["lse"])
    with pytest.raises(T.vsa.VsaError, match="BAD_INDEX"):
        r.plan.check()
