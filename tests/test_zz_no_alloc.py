"""vsa_tile_score_static: the tile-score stage without any caller workspace.

Some callers may not allocate device memory while they run the layer -- code
under another framework's memory planner or fixed arena, or a plugin that must
not call cudaMalloc. For them the library keeps the score stage's scratch in a
fixed 32 MiB device array. These tests check that this entry point returns the
same scores as vsa_tile_score with a caller workspace, on two calls in a row
with different inputs (the shared array keeps the previous call's contents),
and that a plan needing more scratch than the array holds is refused.

This file is collected last on purpose (its name sorts after the other tests):
the entry point is an addition beside the layer's own path, so if one of these
tests fails, a run that stops at the first failure (pytest -x) has already run
every test of the layer itself. The tests need no particular order otherwise and
pass alone in a fresh process too.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _check_same(got, want, rel):
    g = got.double().cpu().numpy()
    w = want.double().cpu().numpy()
    scale = np.max(np.abs(w), axis=-1, keepdims=True)
    assert np.all(np.isfinite(g))
    assert np.all(np.abs(g - w) <= rel * scale)


@pytest.mark.parametrize("scorer", ["meanpool_gate", "tripool"])
def test_static_scratch_scores_match_workspace_scores_twice(scorer):
    import torch
    from gpu_util import SCORE_REL, LayerRun
    from vsa_synth import get_config

    cfg = get_config("medium")
    if scorer == "tripool":     # avg, max and min per tile: wider pooled rows in the scratch
        cfg = cfg.with_(score_mode="tripool", proj_dim=64)
    r = LayerRun(cfg, 0.75)
    assert r.plan.info.workspace_bytes <= 32 << 20
    b, p = r.bufs, r.plan
    p.tile_pack(r.q, r.k_t, r.v, b["qp"], b["kp"], b["vp"])
    p.check()
    # two calls in a row on different inputs: (Q, K), then the roles swapped
    for qp, kp in ((b["qp"], b["kp"]), (b["kp"], b["qp"])):
        want = torch.empty_like(b["scores"])
        p.tile_score(qp, kp, r.proj_q, r.proj_k, want, b["workspace"])
        got = torch.full_like(b["scores"], float("nan"))
        p.tile_score_static(qp, kp, r.proj_q, r.proj_k, got)
        p.check()
        _check_same(got, want, SCORE_REL)
        # and the selections made from them agree
        idx_a = torch.empty_like(b["idx"])
        idx_b = torch.empty_like(b["idx"])
        p.topk_select(want, idx_a)
        p.topk_select(got, idx_b)
        p.check()
        assert torch.equal(idx_a, idx_b)


def test_static_scratch_refuses_plans_that_need_more():
    import tile_sparse_video_pack_b200 as T
    from vsa_synth import get_config

    plan = T.Plan.from_config(get_config("full"), 0.75)
    assert plan.info.workspace_bytes > 32 << 20
    st = T.vsa.library().vsa_tile_score_static(plan._h, *([T.vsa.ctypes.c_void_p(256)] * 5), None)
    assert st == 2   # VSA_ERR_UNSUPPORTED, returned before anything is launched


def test_static_scratch_refuses_reference_segment_plans():
    """R2VA plans continue with vsa_ref_score, which reads the projected pooled Q from the
    caller's workspace; the static call keeps it in the library's array, so it refuses them."""
    import tile_sparse_video_pack_b200 as T
    from gpu_util import r2va_gpu_config

    plan = T.Plan.from_config(r2va_gpu_config(128), 0.5)
    assert plan.info.n_ref_tiles > 0 and plan.info.workspace_bytes <= 32 << 20
    st = T.vsa.library().vsa_tile_score_static(plan._h, *([T.vsa.ctypes.c_void_p(256)] * 5), None)
    assert st == 2   # VSA_ERR_UNSUPPORTED
