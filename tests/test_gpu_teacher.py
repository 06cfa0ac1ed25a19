"""GPU parity of the teacher tile map and of the selection-overlap counts (tile recall).

The teacher map is compared with the fp64 oracle entry by entry; the overlap counts are
compared exactly with the oracle's recall rule applied to the GPU's own teacher values
(the top-k decision taken in the kernel's precision).
"""
import math

import numpy as np
import pytest

import oracle.vsa_oracle as O
from gpu_util import LayerRun, n_video_tiles, oracle_inputs_f64, ragged_gpu_config, scale_of
from vsa_synth import get_config

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": (lambda: get_config("tiny"), 0.5),
    "ragged128": (lambda: ragged_gpu_config(128), 0.5),
    "ragged64_tripool": (lambda: ragged_gpu_config(64, "tripool"), 0.5),
    "medium": (lambda: get_config("medium"), 0.75),
}


def teacher_run(name):
    import torch
    make, s = CASES[name]
    cfg = make()
    dense = LayerRun(cfg, 0.0, k_per_head=[n_video_tiles(cfg, h) for h in range(cfg.heads)]).run()
    sparse = LayerRun(cfg, s, inputs=dense.inp).run()
    teacher = torch.zeros_like(sparse.bufs["scores"])
    sparse.plan.teacher_tiles(dense.bufs["qp"], dense.bufs["kp"], dense.bufs["lse"], teacher)
    t_idx = torch.zeros_like(sparse.bufs["idx"])
    sparse.plan.topk_select(teacher, t_idx)
    counts = torch.zeros(cfg.batch * cfg.heads * sparse.plan.info.ntv_max, dtype=torch.int32, device="cuda")
    sparse.plan.index_overlap(sparse.bufs["idx"], t_idx, counts)
    sparse.plan.check()
    return cfg, sparse, teacher, counts


@pytest.mark.parametrize("name", sorted(CASES))
def test_teacher_and_recall_match_oracle(name):
    cfg, r, teacher, counts = teacher_run(name)
    q, k, v = oracle_inputs_f64(r.inp)
    ntv_max = r.plan.info.ntv_max
    T_gpu = teacher.view(cfg.batch, cfg.heads, ntv_max, ntv_max).double().cpu().numpy()
    cnt = counts.view(cfg.batch, cfg.heads, ntv_max).cpu().numpy()
    for b in range(cfg.batch):
        for h in range(cfg.heads):
            til = O.head_tiling(cfg, h)
            n = til.n_video
            want = O.teacher_tiles(q[b, :, h], k[b, :, h], til, scale_of(cfg))
            got = T_gpu[b, h, :n, :n]
            assert np.all(np.abs(got - want) <= 2e-3 * want + 1e-9), (b, h, np.max(np.abs(got - want) / want))
            kept = r.kept(b, h)
            for i in range(n):
                assert cnt[b, h, i] == round(O.tile_recall(kept[i], got[i], r.k[h]) * r.k[h]), (b, h, i)
