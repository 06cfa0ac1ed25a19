"""vsa_topk_select on crafted score rows, against the oracle's selection, index for index.

Selection keeps the k largest scores of each row, ties to the lower tile index, written
ascending (Veda news page, "Что делает Veda": head-aware top-k; ties by the lower index are
this build's reading). The rows below drive every path of the kernel: ordinary rows,
constant rows (no value range: a radix select over all keys), rows of a few repeated values
(equal keys straddle the cut), an outlier that squeezes every other score into one value bin
(more candidates than the counting path takes: a radix select inside the bin), +0 / -0 mixes,
infinite scores, and both the 16-byte and the scalar row loads (row strides that are and are
not multiples of four).
"""
import numpy as np
import pytest

import oracle.vsa_oracle as O
from vsa_synth import LayerConfig

pytestmark = pytest.mark.gpu


def _config(T, H, W, name):
    return LayerConfig(name=name, batch=1, heads=2, head_dim=64, T=T, H=H, W=W, segments=(64,),
                       tile_shapes=((4, 4, 4), (4, 4, 4)), score_mode="meanpool_gate", proj_dim=64,
                       sparsity=(0.0,), seed=5)


def _rows(n_rows, n, rng):
    rows = np.empty((n_rows, n), np.float32)
    for i in range(n_rows):
        kind = i % 8
        if kind == 0:
            r = rng.standard_normal(n)
        elif kind == 1:
            r = np.full(n, 0.5)
        elif kind == 2:
            r = rng.integers(0, 4, n).astype(np.float64)
        elif kind == 3:
            r = rng.standard_normal(n)
            r[rng.integers(0, n)] = 1e30
        elif kind == 4:
            r = np.where(rng.random(n) < 0.5, 0.0, -0.0) + np.where(rng.random(n) < 0.2, rng.standard_normal(n), 0.0)
        elif kind == 5:
            r = np.round(rng.standard_normal(n), 1)
        elif kind == 6:
            r = rng.standard_normal(n)
            r[rng.integers(0, n, 2)] = np.inf
        else:
            r = -np.abs(rng.standard_normal(n)) * 1e-3 - 5.0
        rows[i] = r
    return rows


@pytest.mark.parametrize("shape", [(16, 32, 40), (4, 12, 20)], ids=["n320_vector_loads", "n15_scalar_loads"])
def test_crafted_rows_match_the_oracle(shape):
    import torch
    import tile_sparse_video_pack_b200 as T
    cfg = _config(*shape, name="topk_edges")
    n = (shape[0] // 4) * (shape[1] // 4) * (shape[2] // 4)
    plan = T.Plan.from_config(cfg, 0.0)          # k = n: the index table holds any per-call k
    assert plan.info.ntv[0] == n and plan.info.ntv[1] == n
    bufs = plan.allocate()
    rng = np.random.default_rng(7)
    scores = np.stack([_rows(n, n, rng) for _ in range(cfg.heads)])[None]   # [1, heads, n, n]
    assert bufs["scores"].shape == scores.shape
    bufs["scores"].copy_(torch.from_numpy(scores))
    for ks in ([1, n], [n // 4, n - 1], [max(1, n // 10), max(1, n // 2)]):
        bufs["idx"].fill_(-1)
        plan.topk_select(bufs["scores"], bufs["idx"], k_per_head=ks)
        plan.check()
        got = bufs["idx"].cpu().numpy()
        for h in range(cfg.heads):
            for i in range(n):
                want = O.topk_row(scores[0, h, i].astype(np.float64), ks[h])
                assert np.array_equal(got[0, h, i, :ks[h]], want), (ks, h, i, i % 8)
