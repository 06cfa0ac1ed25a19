"""Pins for the fp64 oracle: checks against things other than the oracle itself.

* k = all tiles must reproduce brute-force dense attention (the BSAI VedaSparse
  README, "Correctness", reports keep=100% sparse equal to dense within 2.4e-7;
  the fp64 oracle must reach 1e-12).
* On tiny grids the selected tiles equal exhaustive enumeration of all
  k-subsets, and the tile loop equals one N x N softmax with an explicit mask.
* Closed forms: Q = 0 gives uniform weights; V = c gives c; a zero gate makes
  all scores tie so the k lowest tiles win; constant tiles pool to their
  constant; one-hot tiles fix which key tile wins and so the orientation of the
  score matrix; tiles with known avg, max and min pools fix the exact TripPool
  score matrices, and with them the descriptor's block order, which projection
  goes with queries and which with keys, and each head's own weights.
* The tile permutation matches a closed-form (tile, slot) formula.
* A printed figure: the share of full attention the Veda node reports for its
  1344x768 render at 90 % sparsity (tests/golden/veda_node_attention_share.txt).
* Mutation tests plant plausible mistakes in the oracle and check that a pin
  catches each of them.
"""
import math
import os

import numpy as np
import pytest

import oracle.vsa_oracle as O
from vsa_synth import get_config, make_layer_inputs, LayerConfig

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def ragged_config(batch=2):
    """Small grid with partial prefix tiles and partial, head-specific video tiles."""
    return LayerConfig(
        name="ragged", batch=batch, heads=4, head_dim=16, T=6, H=8, W=8,
        segments=(100, 30), tile_shapes=((4, 4, 4), (16, 2, 2), (2, 4, 8), (8, 4, 2)),
        score_mode="meanpool_gate", proj_dim=16, sparsity=(0.5,), seed=11)


def ragged_tripool_config():
    return ragged_config(batch=1).with_(name="ragged_tp", score_mode="tripool", proj_dim=8, seed=12)


def inputs_f64(cfg):
    inp = make_layer_inputs(cfg)
    return inp, inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v")


def n_video_tiles(cfg, h):
    pt, ph, pw = cfg.tile_shapes[h]
    return -(-cfg.T // pt) * -(-cfg.H // ph) * -(-cfg.W // pw)


def closed_form_tile_slot(cfg, h, r):
    """(tile index in the head's tile list, slot) of token r, from the tiling rules alone."""
    n_pre = cfg.n_prefix_tokens
    if r < n_pre:
        base_tok, base_tile = 0, 0
        for length in cfg.segments:
            if r < base_tok + length:
                j = r - base_tok
                return base_tile + j // 64, j % 64
            base_tok += length
            base_tile += -(-length // 64)
    n_pre_tiles = sum(-(-length // 64) for length in cfg.segments)
    pt, ph, pw = cfg.tile_shapes[h]
    v = r - n_pre
    t, y, x = v // (cfg.H * cfg.W), (v // cfg.W) % cfg.H, v % cfg.W
    nY, nX = -(-cfg.H // ph), -(-cfg.W // pw)
    ti, yi, xi = t // pt, y // ph, x // pw
    t0, y0, x0 = ti * pt, yi * ph, xi * pw
    eh, ew = min(ph, cfg.H - y0), min(pw, cfg.W - x0)
    return n_pre_tiles + (ti * nY + yi) * nX + xi, ((t - t0) * eh + (y - y0)) * ew + (x - x0)


def video_tile_of_token(cfg, h, v):
    """Video tile index of video token v (0-based within the grid), closed form."""
    pt, ph, pw = cfg.tile_shapes[h]
    t, y, x = v // (cfg.H * cfg.W), (v // cfg.W) % cfg.H, v % cfg.W
    nY, nX = -(-cfg.H // ph), -(-cfg.W // pw)
    return ((t // pt) * nY + y // ph) * nX + x // pw


def k_list(cfg, s):
    return [O.k_from_sparsity(s, n_video_tiles(cfg, h)) for h in range(cfg.heads)]


# ---------------------------------------------------------------- pins ------

def pin_dense_when_k_is_all(cfg):
    inp, q, k, v = inputs_f64(cfg)
    kk = [n_video_tiles(cfg, h) for h in range(cfg.heads)]
    res = O.run_layer(cfg, q, k, v, kk, gate=inp.gate, w_q=inp.w_q, w_k=inp.w_k)
    ref = O.dense_attention(q, k, v, 1.0 / math.sqrt(cfg.head_dim))
    err = np.max(np.abs(res.out - ref))
    assert err <= 1e-12, err
    assert np.max(np.abs(res.row_sum - 1.0)) <= 1e-12


def pin_gate_zero_keeps_lowest(cfg):
    inp, q, k, v = inputs_f64(cfg)
    kk = k_list(cfg, 0.5)
    res = O.run_layer(cfg, q, k, v, kk, gate=np.zeros_like(inp.gate), query_tiles={})
    for h in range(cfg.heads):
        assert np.all(res.scores[h] == 0.0)
        want = np.arange(kk[h])
        assert all(np.array_equal(row, want) for row in res.kept[h]), h


def pin_one_hot_orientation():
    """Query tile i pools to e_i, key tile j to e_{(j+3) mod 8}: row i must keep tile (i-3) mod 8."""
    cfg = LayerConfig(name="onehot", batch=1, heads=1, head_dim=16, T=4, H=8, W=16,
                      segments=(64,), tile_shapes=((4, 4, 4),), score_mode="meanpool_gate",
                      proj_dim=16, sparsity=(0.875,), seed=0)
    n_pre = 64
    N = cfg.n_tokens
    q = np.zeros((1, N, 1, 16))
    k = np.zeros((1, N, 1, 16))
    for v_tok in range(cfg.n_video_tokens):
        j = video_tile_of_token(cfg, 0, v_tok)
        q[0, n_pre + v_tok, 0, j] = 1.0
        k[0, n_pre + v_tok, 0, (j + 3) % 8] = 1.0
    kk = [O.k_from_sparsity(0.875, 8)]
    assert kk == [1]
    res = O.run_layer(cfg, q, k, q.copy(), kk, gate=np.eye(16), query_tiles={})
    got = res.kept[0][:, 0]
    assert np.array_equal(got, (np.arange(8) - 3) % 8), got
    # pooled features are exactly e_i and e_{(j+3) mod 8}: the scaled dot product over the
    # 16 gate outputs is 1/sqrt(16) on the matching pair and 0 elsewhere
    i = np.arange(8)[:, None]
    j = np.arange(8)[None, :]
    assert np.array_equal(res.scores[0], np.where(i == (j + 3) % 8, 0.25, 0.0))


def pin_constant_tiles_pool(cfg):
    """Token value = 1 + its slot: a tile of n tokens pools to avg (n+1)/2, max n, min 1."""
    for h in range(cfg.heads):
        til = O.head_tiling(cfg, h)
        x = np.zeros((cfg.n_tokens, 3))
        for r in range(cfg.n_tokens):
            x[r] = 1 + closed_form_tile_slot(cfg, h, r)[1]
        for tok in til.video:
            n = len(tok)
            assert np.allclose(O.mean_pool(x[tok]), (n + 1) / 2, rtol=0, atol=1e-14)
            tp = O.tripool(x[tok])
            assert np.allclose(tp, np.r_[[(n + 1) / 2] * 3, [n] * 3, [1] * 3], rtol=0, atol=1e-14)


def pin_tripool_projection_orientation():
    """TripPool scores on an 8-tile grid whose avg, max and min pools are all known.

    Video query tile i: every token e_i, one token also 100 at coordinate
    (i+1) mod 8, so avg = e_i + (100/64) e_{i+1}, max = e_i + 100 e_{i+1}, min = e_i.
    Video key tile j: every token e_{(j+3) mod 8}, one token also 100 at (j+6) mod 8.
    Head 0 projects the query's max block and the key's min block; head 1 the query's
    min block and the key's max block (identity on the chosen block, zero elsewhere).
    So S_0[i, j] = (1[j = i-3] + 100 * 1[j = i-2]) / 4 and
    S_1[i, j] = (1[j = i-3] + 100 * 1[j = i-6]) / 4 (indices mod 8), exactly in fp64.
    The block order of the descriptor, which projection goes with which side, and
    which head's weights are used all change these matrices.
    """
    d = 16
    cfg = LayerConfig(name="tp_onehot", batch=1, heads=2, head_dim=d, T=4, H=8, W=16,
                      segments=(64,), tile_shapes=((4, 4, 4), (4, 4, 4)), score_mode="tripool",
                      proj_dim=d, sparsity=(0.75,), seed=0)
    q = np.zeros((1, cfg.n_tokens, 2, d))
    k = np.zeros((1, cfg.n_tokens, 2, d))
    for h in range(2):
        for t, tok in enumerate(O.head_tiling(cfg, h).video):
            q[0, tok, h, t] = 1.0
            k[0, tok, h, (t + 3) % 8] = 1.0
            first = min(tok)                               # one token of the tile
            q[0, first, h, (t + 1) % 8] = 100.0
            k[0, first, h, (t + 6) % 8] = 100.0

    def block(b):                                          # identity on block b of [avg; max; min]
        w = np.zeros((3 * d, d))
        w[b * d:(b + 1) * d] = np.eye(d)
        return w

    AVG, MAX, MIN = 0, 1, 2
    w_q = np.stack([block(MAX), block(MIN)])
    w_k = np.stack([block(MIN), block(MAX)])
    kk = [2, 2]
    res = O.run_layer(cfg, q, k, q.copy(), kk, w_q=w_q, w_k=w_k, query_tiles={})
    i = np.arange(8)[:, None]
    j = np.arange(8)[None, :]
    want0 = (np.where(j == (i - 3) % 8, 1.0, 0.0) + np.where(j == (i - 2) % 8, 100.0, 0.0)) / 4
    want1 = (np.where(j == (i - 3) % 8, 1.0, 0.0) + np.where(j == (i - 6) % 8, 100.0, 0.0)) / 4
    assert np.array_equal(res.scores[0], want0), res.scores[0]
    assert np.array_equal(res.scores[1], want1), res.scores[1]
    r = np.arange(8)
    assert np.array_equal(res.kept[0], np.sort(np.stack([(r - 3) % 8, (r - 2) % 8], 1), 1))
    assert np.array_equal(res.kept[1], np.sort(np.stack([(r - 3) % 8, (r - 6) % 8], 1), 1))


# ---------------------------------------------------------------- tests -----

@pytest.mark.parametrize("name", ["tiny", "ragged", "ragged_tp"])
def test_dense_when_k_is_all(name):
    cfg = {"tiny": get_config("tiny"), "ragged": ragged_config(),
           "ragged_tp": ragged_tripool_config()}[name]
    pin_dense_when_k_is_all(cfg)


def test_exhaustive_selection_tiny():
    cfg = get_config("tiny")
    inp, q, k, v = inputs_f64(cfg)
    kk = k_list(cfg, 0.5)
    res = O.run_layer(cfg, q, k, v, kk, gate=inp.gate, query_tiles={})
    for h in range(cfg.heads):
        for i in range(4):
            assert np.array_equal(res.kept[h][i], O.exhaustive_topk(res.scores[h][i], kk[h]))


def pin_exhaustive_with_ties():
    rng = np.random.default_rng(5)
    for _ in range(200):
        row = rng.integers(0, 3, size=7).astype(np.float64)
        kk = int(rng.integers(1, 7))
        assert np.array_equal(O.topk_row(row, kk), O.exhaustive_topk(row, kk))


def test_exhaustive_with_ties():
    pin_exhaustive_with_ties()


def pin_tile_loop_equals_explicit_mask(cfg):
    inp, q, k, v = inputs_f64(cfg)
    kk = k_list(cfg, 0.5)
    res = O.run_layer(cfg, q, k, v, kk, gate=inp.gate, w_q=inp.w_q, w_k=inp.w_k)
    N, n_pre = cfg.n_tokens, cfg.n_prefix_tokens
    for h in range(cfg.heads):
        vt = np.array([video_tile_of_token(cfg, h, x) for x in range(cfg.n_video_tokens)])
        allowed = np.zeros((N, N), dtype=bool)
        allowed[:n_pre, :] = True                 # prefix rows: every key
        allowed[:, :n_pre] = True                 # every row: every prefix key
        for r in range(n_pre, N):
            kept = res.kept[h][vt[r - n_pre]]
            allowed[r, n_pre:] = np.isin(vt, kept)
        ref = O.masked_dense_attention(q[0, :, h], k[0, :, h], v[0, :, h], allowed,
                                       1.0 / math.sqrt(cfg.head_dim))
        assert np.max(np.abs(ref - res.out[0, :, h])) <= 1e-12


@pytest.mark.parametrize("name", ["tiny", "ragged", "ragged_tp"])
def test_tile_loop_equals_explicit_mask(name):
    pin_tile_loop_equals_explicit_mask({"tiny": get_config("tiny"), "ragged": ragged_config(batch=1),
                                        "ragged_tp": ragged_tripool_config()}[name])


def test_invariants_ragged():
    cfg = ragged_config()
    inp, q, k, v = inputs_f64(cfg)
    kk = k_list(cfg, 0.5)
    res = O.run_layer(cfg, q, k, v, kk, gate=inp.gate)
    for h in range(cfg.heads):
        nv = n_video_tiles(cfg, h)
        assert res.kept[h].shape == (nv, kk[h])
        for row in res.kept[h]:
            assert len(set(row.tolist())) == kk[h]
            assert np.all(np.diff(row) > 0) and row.min() >= 0 and row.max() < nv
    assert np.max(np.abs(res.row_sum - 1.0)) <= 1e-12
    assert np.all(np.isfinite(res.out))


def test_q_zero_gives_uniform_mean():
    cfg = ragged_config(batch=1)
    inp, q, k, v = inputs_f64(cfg)
    q[:] = 0.0
    kk = k_list(cfg, 0.5)
    res = O.run_layer(cfg, q, k, v, kk, gate=inp.gate)
    n_pre = cfg.n_prefix_tokens
    for h in range(cfg.heads):
        vt = np.array([video_tile_of_token(cfg, h, x) for x in range(cfg.n_video_tokens)])
        keys = np.r_[np.arange(n_pre), n_pre + np.nonzero(vt < kk[h])[0]]   # ties: lowest k tiles
        want_video = v[0, keys, h].mean(axis=0)
        want_prefix = v[0, :, h].mean(axis=0)
        assert np.max(np.abs(res.out[0, n_pre:, h] - want_video)) <= 1e-12
        assert np.max(np.abs(res.out[0, :n_pre, h] - want_prefix)) <= 1e-12


def test_v_constant_gives_constant():
    cfg = ragged_tripool_config()
    inp, q, k, v = inputs_f64(cfg)
    v[:] = 0.375
    res = O.run_layer(cfg, q, k, v, k_list(cfg, 0.5), w_q=inp.w_q, w_k=inp.w_k)
    assert np.max(np.abs(res.out - 0.375)) <= 1e-13


def test_gate_zero_keeps_lowest():
    pin_gate_zero_keeps_lowest(ragged_config(batch=1))


def test_one_hot_orientation():
    pin_one_hot_orientation()


def test_constant_tiles_pool():
    pin_constant_tiles_pool(ragged_config(batch=1))


def test_tripool_projection_orientation():
    pin_tripool_projection_orientation()


def pin_permutation_closed_form():
    cfg = ragged_config()
    inp, q, k, v = inputs_f64(cfg)
    packed, counts = O.pack(q, cfg)
    seen = np.zeros(packed.shape[1:4], dtype=bool)
    for h in range(cfg.heads):
        for r in range(cfg.n_tokens):
            n, s = closed_form_tile_slot(cfg, h, r)
            assert np.array_equal(packed[:, h, n, s], q[:, r, h])
            assert s < counts[h, n]
            seen[h, n, s] = True
    assert np.all(packed[:, ~seen] == 0.0)          # padding slots are zero
    assert seen.sum() == cfg.heads * cfg.n_tokens
    assert np.array_equal(O.unpack(packed, cfg), q)


def test_permutation_closed_form():
    pin_permutation_closed_form()


def pin_custom_tiling_golden_partitions_grid():
    with open(os.path.join(GOLDEN, "custom_tiling.txt")) as f:
        line = [x for x in f.read().splitlines() if x and not x.startswith("#")][0]
    shapes = [tuple(int(a) for a in part.split(",")) for part in line.split(";")]
    assert shapes == [(4, 4, 4), (8, 4, 2), (2, 4, 8), (4, 8, 2)]
    T, H, W = 28, 48, 80
    for shp in shapes:
        assert shp[0] * shp[1] * shp[2] == 64
        tiles = O.video_tiles(T, H, W, shp, 0)
        assert len(tiles) == -(-T // shp[0]) * -(-H // shp[1]) * -(-W // shp[2])
        allt = np.concatenate(tiles)
        assert np.array_equal(np.sort(allt), np.arange(T * H * W))


def test_custom_tiling_golden_partitions_grid():
    pin_custom_tiling_golden_partitions_grid()


def pin_head_aware_tile_counts():
    # (16,2,2) on 28 frames: 2 x 24 x 40 tiles, the second temporal row holds 12 frames
    tiles = O.video_tiles(28, 48, 80, (16, 2, 2), 0)
    sizes = np.array([len(t) for t in tiles])
    assert len(tiles) == 1920 and np.sum(sizes == 48) == 960 and np.sum(sizes == 64) == 960
    assert len(O.prefix_tiles((512, 3840, 640))) == 78
    assert [len(t) for t in O.prefix_tiles((100, 30))] == [64, 36, 30]


def test_head_aware_tile_counts():
    pin_head_aware_tile_counts()


def pin_k_from_sparsity():
    with open(os.path.join(GOLDEN, "sparsity_levels.txt")) as f:
        levels = [float(x.split()[0]) for x in f.read().splitlines() if x and not x.startswith("#")]
    for s in levels:
        for n in (4, 120, 1680, 1920, 3600):
            k = O.k_from_sparsity(s, n)
            if abs(s * n - round(s * n)) < 1e-9:        # s*n integral: exactly (1-s)*n kept
                assert k == n - round(s * n), (s, n, k)
            assert 1 <= k <= n
    assert O.k_from_sparsity(0.95, 1680) == 84          # not 85: (1-s)*n is 84.00000000000007
    assert O.k_from_sparsity(0.0, 1680) == 1680
    assert O.k_from_sparsity(1.0, 1680) == 1
    assert [O.k_from_sparsity(s, 3600) for s in (0, .5, .75, .9, .95)] == [3600, 1800, 900, 360, 180]


def test_k_from_sparsity():
    pin_k_from_sparsity()


def test_flop_count_matches_run():
    cfg = get_config("tiny")
    inp, q, k, v = inputs_f64(cfg)
    kk = k_list(cfg, 0.5)
    res = O.run_layer(cfg, q, k, v, kk, gate=inp.gate)
    assert O.attention_flops(cfg, kk) == 4 * cfg.head_dim * res.computed_pairs
    full = get_config("full")
    f = O.attention_flops(full, [420] * 24)
    dense = 4 * 128 * 24 * full.n_tokens ** 2
    assert abs(f / dense - 0.3151) < 5e-4


def pin_veda_node_attention_share():
    """The share of full attention the Veda node reports for its 1344x768, 90 % render
    (tests/golden/veda_node_attention_share.txt), from the oracle's count of computed
    pairs (4 d per pair) over the dense count, rounded to one decimal as printed."""
    with open(os.path.join(GOLDEN, "veda_node_attention_share.txt")) as f:
        rows = [x.split() for x in f.read().splitlines() if x and not x.startswith("#")]
    for T, H, W, text, s, computed, skipped in rows:
        cfg = LayerConfig(name="veda_node", batch=1, heads=1, head_dim=128, T=int(T), H=int(H), W=int(W),
                          segments=(int(text),), tile_shapes=((4, 4, 4),), score_mode="meanpool_gate",
                          proj_dim=128, sparsity=(float(s),), seed=0)
        kk = k_list(cfg, float(s))
        share = 100.0 * O.attention_flops(cfg, kk) / (4 * cfg.head_dim * cfg.n_tokens ** 2)
        assert f"{share:.1f}" == computed, share
        assert f"{100.0 - share:.1f}" == skipped, share


def test_veda_node_attention_share():
    pin_veda_node_attention_share()


# ------------------------------------------------------- planted mistakes ---

def _expect_pin_failure(pin, *args):
    with pytest.raises(AssertionError):
        pin(*args)


def test_mutation_tie_rule(monkeypatch):
    def bad(row, k):                       # ties resolved toward the higher index
        j = np.arange(row.shape[0])
        return np.sort(np.lexsort((-j, -row))[:k])
    monkeypatch.setattr(O, "topk_row", bad)
    _expect_pin_failure(pin_gate_zero_keeps_lowest, ragged_config(batch=1))


def test_mutation_smallest_instead_of_largest(monkeypatch):
    monkeypatch.setattr(O, "topk_row", lambda row, k: np.sort(np.lexsort((np.arange(row.size), row))[:k]))
    _expect_pin_failure(pin_one_hot_orientation)


def test_mutation_transposed_scores(monkeypatch):
    good = O.tile_scores
    monkeypatch.setattr(O, "tile_scores", lambda *a, **kw: good(*a, **kw).T)
    _expect_pin_failure(pin_one_hot_orientation)


def test_mutation_wrong_scale(monkeypatch):
    good = O.softmax_attention
    monkeypatch.setattr(O, "softmax_attention", lambda q, k, v, s: good(q, k, v, 2 * s))
    _expect_pin_failure(pin_dense_when_k_is_all, get_config("tiny"))


def test_mutation_video_rows_lose_prefix(monkeypatch):
    def bad(til, tile_id, kept, ref=None, kept_ref=None):
        if tile_id < til.n_prefix:
            return np.concatenate(til.all)
        return np.concatenate([til.video[j] for j in kept])
    monkeypatch.setattr(O, "query_key_tokens", bad)
    _expect_pin_failure(pin_dense_when_k_is_all, get_config("tiny"))


def test_mutation_pool_over_64(monkeypatch):
    monkeypatch.setattr(O, "mean_pool", lambda x: x.sum(axis=0) / 64.0)
    _expect_pin_failure(pin_constant_tiles_pool, ragged_config(batch=1))


def test_mutation_sum_pool_in_scores(monkeypatch):
    monkeypatch.setattr(O, "mean_pool", lambda x: x.sum(axis=0))
    _expect_pin_failure(pin_one_hot_orientation)


@pytest.mark.parametrize("order", [(0, 2, 1), (1, 0, 2), (1, 2, 0), (2, 0, 1), (2, 1, 0)])
def test_mutation_tripool_block_order(monkeypatch, order):
    good = O.tripool

    def bad(x):
        d = x.shape[1]
        parts = [good(x)[b * d:(b + 1) * d] for b in range(3)]
        return np.concatenate([parts[b] for b in order])
    monkeypatch.setattr(O, "tripool", bad)
    _expect_pin_failure(pin_tripool_projection_orientation)


def test_mutation_tripool_projections_swapped(monkeypatch):
    good = O.tile_scores

    def bad(q_h, k_h, til, cfg, h, gate=None, w_q=None, w_k=None, key_tiles=None):
        return good(q_h, k_h, til, cfg, h, gate, w_k, w_q, key_tiles)
    monkeypatch.setattr(O, "tile_scores", bad)
    _expect_pin_failure(pin_tripool_projection_orientation)


def test_mutation_tripool_first_head_weights(monkeypatch):
    good = O.tile_scores

    def bad(q_h, k_h, til, cfg, h, *a, **kw):
        return good(q_h, k_h, til, cfg, 0, *a, **kw)
    monkeypatch.setattr(O, "tile_scores", bad)
    _expect_pin_failure(pin_tripool_projection_orientation)


def test_mutation_unscaled_scores(monkeypatch):
    good = O.tile_scores
    monkeypatch.setattr(O, "tile_scores", lambda *a, **kw: 4.0 * good(*a, **kw))
    _expect_pin_failure(pin_one_hot_orientation)


def test_mutation_prefix_rows_sparse_in_count(monkeypatch):
    """Counting prefix query rows like video rows (prefix keys plus k video tiles)
    moves the share off the printed figure."""
    def bad(cfg, k_per_head):
        n_pre, n = cfg.n_prefix_tokens, cfg.n_tokens
        return sum(4 * cfg.head_dim * n * (n_pre + 64 * kh) for kh in k_per_head)
    monkeypatch.setattr(O, "attention_flops", bad)
    _expect_pin_failure(pin_veda_node_attention_share)


def test_mutation_video_rows_without_prefix_keys_in_count(monkeypatch):
    def bad(cfg, k_per_head):
        n_pre, nv, n = cfg.n_prefix_tokens, cfg.n_video_tokens, cfg.n_tokens
        return sum(4 * cfg.head_dim * (n_pre * n + nv * 64 * kh) for kh in k_per_head)
    monkeypatch.setattr(O, "attention_flops", bad)
    _expect_pin_failure(pin_veda_node_attention_share)


# ------------------------------------------------ teacher map and recall ---

def _teacher_case(h=1):
    cfg = ragged_config(batch=1)
    inp, q, k, v = inputs_f64(cfg)
    return cfg, O.head_tiling(cfg, h), q[0, :, h], k[0, :, h]


def pin_teacher_uniform_when_q_zero():
    """Q = 0: every row attends uniformly to all N tokens, prefix included, so every
    entry of the teacher map is exactly 1 / N."""
    cfg, til, q, k = _teacher_case()
    T = O.teacher_tiles(np.zeros_like(q), k, til, 1 / math.sqrt(cfg.head_dim))
    assert T.shape == (til.n_video, til.n_video)
    assert np.max(np.abs(T - 1.0 / cfg.n_tokens)) <= 1e-15


def test_teacher_uniform_when_q_zero():
    pin_teacher_uniform_when_q_zero()


def pin_teacher_dominant_token():
    """One query token r0 of video tile i0 aligned with one key token c0 of tile j0 (far
    larger logit than anything else): T[i0, j0] ~ 1 and j0 is the teacher's top tile of
    row i0, while a row-mean pooling would give about 1/64. Rows of other tiles are
    unaffected."""
    cfg, til, q, k = _teacher_case()
    i0, j0 = 2, 5
    r0, c0 = til.video[i0][7], til.video[j0][11]
    q, k = q.copy() * 0.1, k.copy() * 0.1
    q[r0] = 0.0
    q[r0, 3] = 40.0
    k[c0] = 0.0
    k[c0, 3] = 40.0
    scale = 1 / math.sqrt(cfg.head_dim)
    T = O.teacher_tiles(q, k, til, scale)
    assert T[i0, j0] > 0.999
    assert list(O.topk_row(T[i0], 1)) == [j0]
    # the same rows without the planted pair stay far below
    assert np.max(np.delete(T[i0], j0)) < 0.05


def test_teacher_dominant_token():
    pin_teacher_dominant_token()


def test_teacher_is_a_max_of_probabilities():
    cfg, til, q, k = _teacher_case(h=3)
    T = O.teacher_tiles(q, k, til, 1 / math.sqrt(cfg.head_dim))
    assert np.all(T > 0) and np.all(T <= 1)   # softmax weights


def pin_recall_identities():
    rng = np.random.default_rng(5)
    T = rng.random((6, 12))
    for i in range(6):
        best = O.topk_row(T[i], 4)
        assert O.tile_recall(best, T[i], 4) == 1.0
        rest = np.setdiff1d(np.arange(12), best)[:4]
        assert O.tile_recall(rest, T[i], 4) == 0.0
        assert O.tile_recall(np.arange(12), T[i], 12) == 1.0
        assert O.tile_recall(np.sort(np.r_[best[:2], rest[:2]]), T[i], 4) == 0.5


def test_recall_identities():
    pin_recall_identities()


def test_mutation_teacher_mean_over_rows(monkeypatch):
    def bad(q_h, k_h, til, scale):         # pools rows by their mean instead of the max
        keys = np.concatenate(til.all)
        start = np.cumsum([0] + [len(t) for t in til.all])
        T = np.zeros((til.n_video, til.n_video))
        for i, rows in enumerate(til.video):
            x = scale * (q_h[rows] @ k_h[keys].T)
            a = np.exp(x - x.max(axis=1, keepdims=True))
            a /= a.sum(axis=1, keepdims=True)
            for j in range(til.n_video):
                T[i, j] = a[:, start[til.n_prefix + j]:start[til.n_prefix + j + 1]].max(axis=1).mean()
        return T
    monkeypatch.setattr(O, "teacher_tiles", bad)
    _expect_pin_failure(pin_teacher_dominant_token)


def test_mutation_teacher_softmax_over_video_keys_only(monkeypatch):
    def bad(q_h, k_h, til, scale):         # normalises each row over video keys only
        keys = np.concatenate(til.video)
        start = np.cumsum([0] + [len(t) for t in til.video])
        T = np.zeros((til.n_video, til.n_video))
        for i, rows in enumerate(til.video):
            x = scale * (q_h[rows] @ k_h[keys].T)
            a = np.exp(x - x.max(axis=1, keepdims=True))
            a /= a.sum(axis=1, keepdims=True)
            for j in range(til.n_video):
                T[i, j] = a[:, start[j]:start[j + 1]].max()
        return T
    monkeypatch.setattr(O, "teacher_tiles", bad)
    _expect_pin_failure(pin_teacher_uniform_when_q_zero)


# ------------------------------------- R2VA budgets: reference tiles pruned ---

def ragged_r2va_config(score_mode="meanpool_gate"):
    """Text, a reference segment of 130 tokens (tiles of 64, 64 and 2 tokens), audio."""
    cfg = ragged_config(batch=1).with_(name="ragged_r2va", segments=(100, 130, 30), seg_ref=(0, 1, 0),
                                       k_ref=2, seed=13)
    if score_mode == "tripool":
        cfg = cfg.with_(name="ragged_r2va_tp", score_mode="tripool", proj_dim=8, seed=14)
    return cfg


def prefix_tile_of_token(cfg, x):
    t, base = 0, 0
    for length in cfg.segments:
        if x < base + length:
            return t + (x - base) // 64
        t += -(-length // 64)
        base += length
    raise ValueError(x)


def pin_r2va_explicit_mask(cfg):
    """Video rows see the dense prefix segments, their k_ref kept reference tiles and
    their k kept video tiles; prefix rows see everything: one N x N masked softmax."""
    inp, q, k, v = inputs_f64(cfg)
    kk = k_list(cfg, 0.5)
    res = O.run_layer(cfg, q, k, v, kk, gate=inp.gate, w_q=inp.w_q, w_k=inp.w_k)
    ref = O.ref_tiles(cfg)
    assert list(ref) == [2, 3, 4]
    N, n_pre = cfg.n_tokens, cfg.n_prefix_tokens
    pt = np.array([prefix_tile_of_token(cfg, x) for x in range(n_pre)])
    for h in range(cfg.heads):
        vt = np.array([video_tile_of_token(cfg, h, x) for x in range(cfg.n_video_tokens)])
        allowed = np.zeros((N, N), dtype=bool)
        allowed[:n_pre, :] = True
        for r in range(n_pre, N):
            i = vt[r - n_pre]
            kept_pre = [t for t in range(pt.max() + 1) if t not in ref] + [int(ref[j]) for j in res.ref_kept[h][i]]
            allowed[r, :n_pre] = np.isin(pt, kept_pre)
            allowed[r, n_pre:] = np.isin(vt, res.kept[h][i])
            assert len(res.ref_kept[h][i]) == cfg.k_ref
        want = O.masked_dense_attention(q[0, :, h], k[0, :, h], v[0, :, h], allowed, 1.0 / math.sqrt(cfg.head_dim))
        assert np.max(np.abs(want - res.out[0, :, h])) <= 1e-12


@pytest.mark.parametrize("mode", ["meanpool_gate", "tripool"])
def test_r2va_equals_explicit_mask(mode):
    pin_r2va_explicit_mask(ragged_r2va_config(mode))


def test_r2va_all_reference_tiles_is_the_dense_prefix_layer():
    cfg = ragged_r2va_config().with_(k_ref=3)
    inp, q, k, v = inputs_f64(cfg)
    kk = k_list(cfg, 0.5)
    a = O.run_layer(cfg, q, k, v, kk, gate=inp.gate)
    b = O.run_layer(cfg.with_(seg_ref=(), k_ref=0), q, k, v, kk, gate=inp.gate)
    assert np.array_equal(a.out, b.out) and a.computed_pairs == b.computed_pairs


def test_r2va_zero_gate_keeps_lowest_reference_tiles():
    cfg = ragged_r2va_config()
    inp, q, k, v = inputs_f64(cfg)
    res = O.run_layer(cfg, q, k, v, k_list(cfg, 0.5), gate=np.zeros_like(inp.gate))
    for h in range(cfg.heads):
        assert np.all(res.ref_kept[h] == np.array([0, 1]))


def pin_r2va_reference_orientation():
    """Reference tiles are described by their K rows, like video key tiles. Video query
    tile i pools (Q) to e_i; reference tile r holds K = e_{2r} and, as a decoy, Q = e_{2r+1}.
    With the identity gate and k_ref = 1, even query tiles keep reference tile i/2 (score
    1/sqrt(16)) and odd ones see only zeros and keep tile 0 by the tie rule; pooling the
    reference tiles' Q would swap the two cases."""
    d = 16
    cfg = LayerConfig(name="r2va_onehot", batch=1, heads=1, head_dim=d, T=4, H=8, W=16,
                      segments=(64, 256, 64), tile_shapes=((4, 4, 4),), score_mode="meanpool_gate",
                      proj_dim=d, sparsity=(0.5,), seed=0, seg_ref=(0, 1, 0), k_ref=1)
    til = O.head_tiling(cfg, 0)
    ref = O.ref_tiles(cfg)
    assert list(ref) == [1, 2, 3, 4]
    q = np.zeros((1, cfg.n_tokens, 1, d))
    k = np.zeros((1, cfg.n_tokens, 1, d))
    for i, tok in enumerate(til.video):
        q[0, tok, 0, i] = 1.0
    for r, t in enumerate(ref):
        k[0, til.prefix[t], 0, 2 * r] = 1.0
        q[0, til.prefix[t], 0, 2 * r + 1] = 1.0
    res = O.run_layer(cfg, q, k, q.copy(), [4], gate=np.eye(d), query_tiles={})
    want = np.array([[i // 2] if i % 2 == 0 else [0] for i in range(8)])
    assert np.array_equal(res.ref_kept[0], want), res.ref_kept[0]
    i = np.arange(8)[:, None]
    r = np.arange(4)[None, :]
    assert np.array_equal(res.ref_scores[0], np.where(i == 2 * r, 0.25, 0.0))


def test_r2va_reference_orientation():
    pin_r2va_reference_orientation()


def test_mutation_r2va_reference_tiles_pooled_from_q(monkeypatch):
    good = O.tile_scores

    def bad(q_h, k_h, til, cfg, h, gate=None, w_q=None, w_k=None, key_tiles=None):
        return good(q_h, q_h if key_tiles is not None else k_h, til, cfg, h, gate, w_q, w_k, key_tiles)
    monkeypatch.setattr(O, "tile_scores", bad)
    _expect_pin_failure(pin_r2va_reference_orientation)


def test_mutation_r2va_drops_reference_tiles(monkeypatch):
    good = O.query_key_tokens
    monkeypatch.setattr(O, "query_key_tokens",
                        lambda til, t, kept, ref=None, kept_ref=None:
                        good(til, t, kept, ref, kept_ref[:0] if kept_ref is not None else None))
    _expect_pin_failure(pin_r2va_explicit_mask, ragged_r2va_config())


# ------------------------------------------- fp8 (e4m3) Q K^T per-tile scales ---

def pin_e4m3_round_matches_torch_float8():
    """Against torch's float8_e4m3fn conversion (round to nearest even), which is a
    library routine independent of the oracle: every finite code, every midpoint between
    neighbouring codes, and random values within the finite range."""
    import torch
    codes = torch.arange(256, dtype=torch.int16).to(torch.uint8).view(torch.float8_e4m3fn).float().double().numpy()
    finite = np.unique(codes[np.isfinite(codes)])
    mids = (finite[1:] + finite[:-1]) / 2
    rng = np.random.default_rng(3)
    xs = np.concatenate([finite, mids, rng.uniform(-448, 448, 20000), rng.normal(0, 1e-2, 20000)])
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(O.e4m3_round(xs), want)
    assert np.array_equal(O.e4m3_round(finite), finite)          # idempotent on the codes
    assert O.e4m3_round(np.array([500.0, -1e6]))[0] == 448.0      # saturates (torch would give NaN)


def test_e4m3_round_matches_torch_float8():
    pin_e4m3_round_matches_torch_float8()


def test_tile_quantisation_scale_and_range():
    rng = np.random.default_rng(4)
    x = rng.normal(0, 3, (64, 128)).astype(np.float32)
    codes, scale = O.quantize_tile_e4m3(x)
    assert np.float32(scale) == np.float32(np.max(np.abs(x)) / np.float32(448.0))
    assert np.max(np.abs(codes)) == 448.0
    rel = np.abs(codes * scale - x) / np.maximum(np.abs(x), 1e-30)
    assert np.max(rel[np.abs(x) > 2.0 ** -6 * scale]) <= 2.0 ** -4 + 1e-7   # half a mantissa step
    assert O.quantize_tile_e4m3(np.zeros((3, 8)))[1] == 1.0


def pin_fp8_codes_divide_by_the_scale():
    """A tile whose largest magnitude is 1.53125 = 49/32 has the scale 49/32 / 448 = 7/2048,
    exact in fp32. Its entry 0.341796875 = 175/512 divided by that scale is exactly 100, the
    midpoint between the e4m3 codes 96 and 104, so rounding to nearest even gives 96.
    Multiplying by the rounded reciprocal fl(448 / amax) instead lands just above 100 and
    gives 104, so this tile tells the two rules apart."""
    x = np.full((64, 128), 0.341796875, dtype=np.float32)
    x[0, 0] = 1.53125
    codes, scale = O.quantize_tile_e4m3(x)
    assert scale == 7 / 2048
    assert codes[0, 0] == 448.0
    assert np.all(codes.ravel()[1:] == 96.0), np.unique(codes)


def test_fp8_codes_divide_by_the_scale():
    pin_fp8_codes_divide_by_the_scale()
    # the other rule really does differ on this tile
    inv = np.float32(np.float32(448.0) / np.float32(1.53125))
    assert O.e4m3_round(np.float64(np.float32(0.341796875) * inv)) == 104.0


def test_mutation_fp8_reciprocal_multiply(monkeypatch):
    def bad(x):
        xf = np.asarray(x, dtype=np.float32)
        amax = np.float32(np.max(np.abs(xf)))
        inv = np.float32(np.float32(O.E4M3_MAX) / amax)
        return O.e4m3_round((xf * inv).astype(np.float64)), float(np.float32(amax / np.float32(O.E4M3_MAX)))
    monkeypatch.setattr(O, "quantize_tile_e4m3", bad)
    _expect_pin_failure(pin_fp8_codes_divide_by_the_scale)


def test_fp8_attention_is_exact_on_representable_inputs():
    """Q and K entries from {0, +-0.5, +-1, +-1.75} with a 1.75 in every tile: every scale
    is 1.75/448 = 2^-8 exactly and every entry divided by it (0, 128, 256, 448) is an e4m3
    value, so quantisation is exact and the fp8 layer equals the bf16 one."""
    cfg = ragged_config(batch=1)
    inp, q, k, v = inputs_f64(cfg)
    rng = np.random.default_rng(6)
    vals = [-1.75, -1.0, -0.5, 0.0, 0.5, 1.0, 1.75]
    q = rng.choice(vals, size=q.shape)
    k = rng.choice(vals, size=k.shape)
    q[..., 0] = k[..., 0] = 1.75       # every token, so every tile, holds the largest magnitude
    kk = k_list(cfg, 0.5)
    a = O.run_layer(cfg, q, k, v, kk, gate=inp.gate)
    b = O.run_layer(cfg, q, k, v, kk, gate=inp.gate, qk_fp8=True)
    assert np.array_equal(a.out, b.out)


def pin_fp8_scales_are_per_tile():
    """Tiles of different magnitudes: tile t holds c_t * v with c_t in {1, 3, 9}, v from
    {0, +-0.5, +-1, +-1.25}, and its first token also +-1.75 c_t at channel 0 (the sign
    alternates between tiles). Per tile the scale is c_t / 256 exactly and every entry maps
    to 0, 128, 256, 320 or 448, all e4m3 values, so the fp8 layer equals the bf16 one bit for
    bit. One scale for the whole tensor (a tile of c = 1 against 9/256: 0.5 maps to 14.2),
    one per token (a row whose largest entry is 1.25: 1 maps to 358.4) or a signed maximum
    (1.25 c_t in place of 1.75 c_t) leaves the e4m3 grid and changes the output."""
    cfg = ragged_config(batch=1)
    inp, q, k, v = inputs_f64(cfg)
    rng = np.random.default_rng(8)
    vals = [-1.25, -1.0, -0.5, 0.0, 0.5, 1.0, 1.25]
    q = rng.choice(vals, size=q.shape)
    k = rng.choice(vals, size=k.shape)
    for h in range(cfg.heads):
        for t, tok in enumerate(O.head_tiling(cfg, h).all):
            c = 3.0 ** (t % 3)
            sign = 1.0 if t % 2 == 0 else -1.0
            for x in (q, k):
                x[0, tok, h] *= c
                x[0, tok[0], h, 0] = sign * 1.75 * c
    kk = k_list(cfg, 0.5)
    a = O.run_layer(cfg, q, k, v, kk, gate=inp.gate)
    b = O.run_layer(cfg, q, k, v, kk, gate=inp.gate, qk_fp8=True)
    assert np.array_equal(a.out, b.out), np.max(np.abs(a.out - b.out))


def test_fp8_scales_are_per_tile():
    pin_fp8_scales_are_per_tile()


def test_mutation_fp8_one_scale_per_tensor(monkeypatch):
    def bad(x_h, til):
        codes, scale = O.quantize_tile_e4m3(np.asarray(x_h, dtype=np.float64))
        return codes * scale
    monkeypatch.setattr(O, "dequantized_tiles", bad)
    _expect_pin_failure(pin_fp8_scales_are_per_tile)


def test_mutation_fp8_one_scale_per_token(monkeypatch):
    def bad(x_h, til):
        out = np.array(x_h, dtype=np.float64)
        for r in range(out.shape[0]):
            codes, scale = O.quantize_tile_e4m3(out[r:r + 1])
            out[r:r + 1] = codes * scale
        return out
    monkeypatch.setattr(O, "dequantized_tiles", bad)
    _expect_pin_failure(pin_fp8_scales_are_per_tile)


def test_mutation_fp8_signed_max(monkeypatch):
    def bad(x):
        xf = np.asarray(x, dtype=np.float32)
        amax = np.float32(np.max(xf))
        inv = np.float32(np.float32(O.E4M3_MAX) / amax)
        return O.e4m3_round((xf * inv).astype(np.float64)), float(np.float32(amax / np.float32(O.E4M3_MAX)))
    monkeypatch.setattr(O, "quantize_tile_e4m3", bad)
    _expect_pin_failure(pin_fp8_scales_are_per_tile)


def test_fp8_attention_close_to_bf16_and_not_equal():
    cfg = ragged_config(batch=1)
    inp, q, k, v = inputs_f64(cfg)
    kk = k_list(cfg, 0.5)
    a = O.run_layer(cfg, q, k, v, kk, gate=inp.gate)
    b = O.run_layer(cfg, q, k, v, kk, gate=inp.gate, qk_fp8=True)
    d = np.abs(a.out - b.out)
    assert 0 < np.max(d) < 0.3 * np.max(np.abs(a.out))      # e4m3 keeps 3 mantissa bits
    assert all(np.array_equal(x, y) for x, y in zip(a.kept, b.kept))   # selection unchanged


def test_flop_count_with_reference_budgets_matches_run():
    """The closed-form count with reference budgets equals the pairs the tile loop computes
    (full reference tiles: a 128-token reference segment)."""
    cfg = ragged_config(batch=1).with_(name="r2va_full_tiles", segments=(100, 128, 30), seg_ref=(0, 1, 0),
                                       k_ref=1, tile_shapes=((2, 4, 8),) * 4, seed=15)
    inp, q, k, v = inputs_f64(cfg)
    kk = k_list(cfg, 0.5)
    res = O.run_layer(cfg, q, k, v, kk, gate=inp.gate)
    assert O.attention_flops(cfg, kk) == 4 * cfg.head_dim * res.computed_pairs


@pytest.mark.parametrize("name", ["full", "r2va", "long"])
def test_bench_flop_count_is_the_oracle_count(name):
    import bench
    cfg = get_config(name)
    ks = [O.k_from_sparsity(cfg.sparsity[-1], n_video_tiles(cfg, h)) for h in range(cfg.heads)]
    assert bench.attention_flops(cfg, ks) == O.attention_flops(cfg, ks)


# ------------------------------- planted mistakes in tiling, k, e4m3, recall ---

def _video_tiles_with(order="thw", inner="thw", edge="ceil"):
    """The oracle's video tiling with one rule changed: the tile order (``order``), the token
    order inside a tile (``inner``), or edge tiles dropped instead of kept partial (``edge``)."""
    def tiles(T, H, W, shape, n_prefix):
        pt, ph, pw = shape
        cnt = (lambda a, b: -(-a // b)) if edge == "ceil" else (lambda a, b: a // b)
        idx = [(ti, hi, wi) for ti in range(cnt(T, pt)) for hi in range(cnt(H, ph)) for wi in range(cnt(W, pw))]
        if order == "wht":
            idx.sort(key=lambda c: (c[2], c[1], c[0]))
        out = []
        for ti, hi, wi in idx:
            t = np.arange(ti * pt, min(T, (ti + 1) * pt))
            y = np.arange(hi * ph, min(H, (hi + 1) * ph))
            x = np.arange(wi * pw, min(W, (wi + 1) * pw))
            tok = (t[:, None, None] * H + y[None, :, None]) * W + x[None, None, :]
            if inner == "wht":
                tok = tok.transpose(2, 1, 0)
            out.append(n_prefix + tok.ravel().astype(np.int64))
        return out
    return tiles


def test_planted_tiling_reference_is_the_oracle():
    # the helper with no rule changed is the oracle's tiling, so each mutation below changes one rule only
    for shape in ((4, 4, 4), (16, 2, 2), (2, 4, 8), (8, 4, 2)):
        want = O.video_tiles(6, 8, 8, shape, 130)
        got = _video_tiles_with()(6, 8, 8, shape, 130)
        assert len(got) == len(want) and all(np.array_equal(a, b) for a, b in zip(got, want))


def test_mutation_video_tiles_w_major(monkeypatch):
    monkeypatch.setattr(O, "video_tiles", _video_tiles_with(order="wht"))
    _expect_pin_failure(pin_permutation_closed_form)


def test_mutation_tokens_w_major_inside_tile(monkeypatch):
    monkeypatch.setattr(O, "video_tiles", _video_tiles_with(inner="wht"))
    _expect_pin_failure(pin_permutation_closed_form)


def test_mutation_edge_tiles_dropped(monkeypatch):
    monkeypatch.setattr(O, "video_tiles", _video_tiles_with(edge="floor"))
    _expect_pin_failure(pin_head_aware_tile_counts)
    _expect_pin_failure(pin_custom_tiling_golden_partitions_grid)


def test_mutation_prefix_tiles_cross_segments(monkeypatch):
    def bad(segments):                      # 64-token chunks of the whole prefix, segments mixed
        n = int(sum(segments))
        return [np.arange(s0, min(n, s0 + O.TILE), dtype=np.int64) for s0 in range(0, n, O.TILE)]
    monkeypatch.setattr(O, "prefix_tiles", bad)
    _expect_pin_failure(pin_head_aware_tile_counts)


def _pack_with(padding="zero", one_tiling=False):
    def pack(x, cfg):
        B, N, Hh, d = x.shape
        tilings = [O.head_tiling(cfg, 0 if one_tiling else h) for h in range(Hh)]
        nt = max(len(t.all) for t in tilings)
        out = np.zeros((B, Hh, nt, O.TILE, d), dtype=x.dtype)
        counts = np.zeros((Hh, nt), dtype=np.int32)
        for h, til in enumerate(tilings):
            for n, tok in enumerate(til.all):
                out[:, h, n, :len(tok)] = x[:, tok, h]
                if padding == "repeat":
                    out[:, h, n, len(tok):] = x[:, tok[-1], h][:, None]
                counts[h, n] = len(tok)
        return out, counts
    return pack


def test_mutation_pack_padding_repeats_last_token(monkeypatch):
    monkeypatch.setattr(O, "pack", _pack_with(padding="repeat"))
    _expect_pin_failure(pin_permutation_closed_form)


def test_mutation_pack_first_heads_tiling_for_every_head(monkeypatch):
    monkeypatch.setattr(O, "pack", _pack_with(one_tiling=True))
    _expect_pin_failure(pin_permutation_closed_form)


def test_mutation_k_ceil_of_kept_share(monkeypatch):
    monkeypatch.setattr(O, "k_from_sparsity", lambda s, n: max(1, min(n, math.ceil((1.0 - s) * n))))
    _expect_pin_failure(pin_k_from_sparsity)


def test_mutation_k_not_clamped(monkeypatch):
    monkeypatch.setattr(O, "k_from_sparsity", lambda s, n: n - math.floor(s * n + 0.5))
    _expect_pin_failure(pin_k_from_sparsity)


def test_mutation_e4m3_ties_away_from_zero(monkeypatch):
    def bad(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.abs(x)
        step = 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -6))) - 3)
        return np.sign(x) * np.minimum(np.floor(a / step + 0.5) * step, O.E4M3_MAX)
    monkeypatch.setattr(O, "e4m3_round", bad)
    _expect_pin_failure(pin_e4m3_round_matches_torch_float8)


def test_mutation_e4m3_without_subnormals(monkeypatch):
    def bad(x):                             # every magnitude gets 3 mantissa bits, however small
        x = np.asarray(x, dtype=np.float64)
        a = np.abs(x)
        with np.errstate(divide="ignore", invalid="ignore"):
            step = 2.0 ** (np.floor(np.log2(a)) - 3)
            q = np.where(a > 0, np.round(a / step) * step, 0.0)
        return np.sign(x) * np.minimum(q, O.E4M3_MAX)
    monkeypatch.setattr(O, "e4m3_round", bad)
    _expect_pin_failure(pin_e4m3_round_matches_torch_float8)


def test_mutation_recall_against_the_teachers_weakest_tiles(monkeypatch):
    monkeypatch.setattr(O, "tile_recall", lambda kept, t, k: len(np.intersect1d(kept, np.argsort(t)[:k])) / k)
    _expect_pin_failure(pin_recall_identities)


def test_mutation_prefix_rows_see_only_the_prefix(monkeypatch):
    good = O.query_key_tokens

    def bad(til, tile_id, kept_video, ref=None, kept_ref=None):
        if tile_id < til.n_prefix:          # conditioning rows read as attending to the conditioning only
            return np.concatenate(til.prefix)
        return good(til, tile_id, kept_video, ref, kept_ref)
    monkeypatch.setattr(O, "query_key_tokens", bad)
    _expect_pin_failure(pin_tile_loop_equals_explicit_mask, ragged_config(batch=1))


def test_mutation_kept_tiles_in_score_order(monkeypatch):
    monkeypatch.setattr(O, "topk_row", lambda row, k: np.lexsort((np.arange(row.size), -row))[:k])
    _expect_pin_failure(pin_exhaustive_with_ties)


# ------------------------------------------------ the brute-force references ---

def pin_dense_attention_matches_torch():
    """The N x N references against torch's scaled_dot_product_attention in fp64 on the CPU (a
    library routine that shares nothing with the oracle), with and without a boolean mask."""
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((2, 50, 3, 16)) for _ in range(3))
    scale = 0.3
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(0, 2, 1, 3)   # [B, heads, N, d]
    want = F.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale).permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(O.dense_attention(q, k, v, scale) - want)) <= 1e-12
    allowed = rng.random((50, 50)) < 0.3
    allowed[np.arange(50), rng.integers(0, 50, 50)] = True          # every row keeps a key
    qh, kh, vh = (torch.from_numpy(np.ascontiguousarray(a[1, :, 2])) for a in (q, k, v))
    want = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=torch.from_numpy(allowed), scale=scale).numpy()
    got = O.masked_dense_attention(q[1, :, 2], k[1, :, 2], v[1, :, 2], allowed, scale)
    assert np.max(np.abs(got - want)) <= 1e-12


def test_dense_attention_matches_torch():
    pin_dense_attention_matches_torch()


def test_exhaustive_topk_hand_cases():
    # the best k-subset by score sum, worked by hand; equal sums go to the lower indices
    assert O.exhaustive_topk(np.array([1.0, 3.0, 2.0, 3.0]), 2).tolist() == [1, 3]
    assert O.exhaustive_topk(np.array([2.0, 2.0, 2.0]), 2).tolist() == [0, 1]
    assert O.exhaustive_topk(np.array([2.0, 1.0, 2.0]), 1).tolist() == [0]
    assert O.exhaustive_topk(np.array([-1.0, -5.0, 0.5, 0.5]), 3).tolist() == [0, 2, 3]
    assert O.exhaustive_topk(np.array([0.0, 4.0, 1.0, 3.0, 2.0]), 5).tolist() == [0, 1, 2, 3, 4]


def test_mutation_dense_softmax_over_queries(monkeypatch):
    def bad(q, k, v, scale):                 # weights normalised down each key's column
        out = np.empty_like(q)
        for b in range(q.shape[0]):
            for h in range(q.shape[2]):
                x = scale * (q[b, :, h] @ k[b, :, h].T)
                p = np.exp(x - x.max(axis=0, keepdims=True))
                out[b, :, h] = (p / p.sum(axis=0, keepdims=True)) @ v[b, :, h]
        return out
    monkeypatch.setattr(O, "dense_attention", bad)
    _expect_pin_failure(pin_dense_attention_matches_torch)
