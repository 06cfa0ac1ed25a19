"""Plain fp64 CPU oracle of one tile-sparse attention layer. TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import or call this module. It is slow on purpose: tiles are
lists of token indices, every score and every softmax is evaluated in fp64 with
numpy, and nothing is blocked, fused or reordered beyond what the method
states. It shares no code with the CUDA library.

What it computes, in the order the pages give it:

1. Tiling.  Video tokens on the (T, H, W) latent grid are grouped into 3D
   tiles of 64 tokens -- 4x4x4 for VSA (Ref2VA VSA README, "two-tier attention
   layout"; "From 650 s to 72 s", "The method"), or one (pt, ph, pw) per head
   with pt*ph*pw = 64 for head-aware tiling (BSAI VedaSparse README, "Core
   Technology: Head-Aware Tiling"; "Implementation": ``_tile_3d`` returns the
   tile and its key mask). The conditioning prefix (text, reference image,
   reference audio) is split into segment-pure tiles that never mix two
   segments (Ref2VA VSA news page, "Патч внимания с двумя уровнями", item 1).
2. Scoring of every (video query tile, video key tile) pair, either by the
   VSA gate on mean-pooled tiles (Ref2VA VSA README, gating projection
   ``to_gate_compress``), or by TripPool: the Avg+Max+Min descriptor of each
   tile with per-head Q/K projections (BSAI VedaSparse README, "Core
   Technology: TripPool"; "Scorer Modes"; Veda news page, "Что делает Veda").
3. Per head, each video query tile keeps its top-k video key tiles; prefix key
   tiles are never pruned and prefix query rows stay dense (BSAI VedaSparse
   README, "v3.4 Highlights": ``sink = exact_kv_and_rows``; Ref2VA README
   items 1-2).
4. Exact softmax attention over the kept tiles only (BSAI VedaSparse README,
   "Core Technology: Tile-Skipping"; "Implementation": ``_veda_sparse``).

Readings where the pages are silent:
* VSA score: S[i, j] = (qbar_i G) . (kbar_j G) / sqrt(d), one d x d gate G per
  layer shared by all heads; qbar/kbar are means over the tile's tokens.
* TripPool score: S = (desc_q W_q[h]) . (desc_k W_k[h]) / sqrt(p), desc = [avg;
  max; min] over the tile's tokens (3d wide), p the projection width.
* The query side pools Q tiles, the key side pools K tiles.
* k from a sparsity s over n tiles: n - floor(s*n + 0.5), clamped to [1, n].
* Ties in top-k: equal scores keep the lower key-tile index; the kept list is
  returned sorted ascending.
* Prefix query rows attend to every token; no mask other than tile pruning.
* A segment whose length is not a multiple of 64 ends in a partial tile; a
  video tile cut by the grid edge is partial too. Partial tiles hold only their
  valid tokens, in (t, h, w) raster order within the tile.
* Softmax scale 1/sqrt(head_dim).
"""
from __future__ import annotations

import dataclasses
import itertools
import math

import numpy as np

TILE = 64

# ---------------------------------------------------------------------------
# 1. tiling
# ---------------------------------------------------------------------------


def prefix_tiles(segments) -> list[np.ndarray]:
    """Segment-pure prefix tiles: 64 consecutive tokens of one segment each.

    Ref2VA VSA news page, "Патч внимания с двумя уровнями" item 1 (the geometry
    mapper keeps text / reference-image / reference-audio tokens in tiles that
    hold one segment only). The last tile of a segment may be partial.
    """
    tiles, base = [], 0
    for length in segments:
        for s0 in range(0, length, TILE):
            tiles.append(np.arange(base + s0, base + min(length, s0 + TILE), dtype=np.int64))
        base += length
    return tiles


def video_tiles(T: int, H: int, W: int, shape, n_prefix: int) -> list[np.ndarray]:
    """3D video tiles of shape (pt, ph, pw) over the latent grid, in (ti, hi, wi) raster order.

    Ref2VA VSA README, "two-tier attention layout" (4x4x4 spatial-temporal
    tiles); BSAI VedaSparse README, "Core Technology: Head-Aware Tiling"
    (per-head (pt, ph, pw), product 64). Tokens inside a tile are listed in
    (t, h, w) raster order; tiles at the grid's far edge keep only the tokens
    that exist.
    """
    pt, ph, pw = shape
    tiles = []
    for ti in range(-(-T // pt)):
        t = np.arange(ti * pt, min(T, (ti + 1) * pt))
        for hi in range(-(-H // ph)):
            y = np.arange(hi * ph, min(H, (hi + 1) * ph))
            for wi in range(-(-W // pw)):
                x = np.arange(wi * pw, min(W, (wi + 1) * pw))
                tok = (t[:, None, None] * H + y[None, :, None]) * W + x[None, None, :]
                tiles.append(n_prefix + tok.ravel().astype(np.int64))
    return tiles


@dataclasses.dataclass
class HeadTiling:
    prefix: list          # list of token-index arrays
    video: list           # list of token-index arrays

    @property
    def n_prefix(self) -> int:
        return len(self.prefix)

    @property
    def n_video(self) -> int:
        return len(self.video)

    @property
    def all(self) -> list:
        return self.prefix + self.video


def head_tiling(cfg, h: int) -> HeadTiling:
    if np.prod(cfg.tile_shapes[h]) != TILE:
        raise ValueError("tile shape must hold 64 tokens")
    return HeadTiling(prefix_tiles(cfg.segments),
                      video_tiles(cfg.T, cfg.H, cfg.W, cfg.tile_shapes[h], cfg.n_prefix_tokens))


def pack(x: np.ndarray, cfg) -> tuple[np.ndarray, np.ndarray]:
    """Token-major ``[B, N, heads, d]`` -> tile-major ``[B, heads, NT, 64, d]`` plus valid counts.

    A pure permutation of rows: slot s of tile n holds token ``tiles[n][s]``;
    slots past the tile's token count are zero. NT is the largest per-head tile
    count; a head with fewer tiles leaves its trailing tiles empty (count 0).
    """
    B, N, Hh, d = x.shape
    tilings = [head_tiling(cfg, h) for h in range(Hh)]
    nt = max(len(t.all) for t in tilings)
    out = np.zeros((B, Hh, nt, TILE, d), dtype=x.dtype)
    counts = np.zeros((Hh, nt), dtype=np.int32)
    for h, til in enumerate(tilings):
        for n, tok in enumerate(til.all):
            out[:, h, n, :len(tok)] = x[:, tok, h]
            counts[h, n] = len(tok)
    return out, counts


def unpack(xp: np.ndarray, cfg) -> np.ndarray:
    """Inverse of :func:`pack`: tile-major rows back to ``[B, N, heads, d]``."""
    B, Hh = xp.shape[:2]
    out = np.zeros((B, cfg.n_tokens, Hh, xp.shape[-1]), dtype=xp.dtype)
    for h in range(Hh):
        for n, tok in enumerate(head_tiling(cfg, h).all):
            out[:, tok, h] = xp[:, h, n, :len(tok)]
    return out


# ---------------------------------------------------------------------------
# 2. scoring
# ---------------------------------------------------------------------------


def k_from_sparsity(sparsity: float, n_tiles: int) -> int:
    """Kept video key tiles per query tile at a given sparsity.

    Sparsity is the pruned share of video key tiles (Ref2VA VSA README: "75%
    video sparsity top-k"; BSAI README node table: keep_percent 5 = 95%
    sparsity). k = n - round-half-up(s * n), clamped to [1, n].
    """
    k = n_tiles - math.floor(sparsity * n_tiles + 0.5)
    return max(1, min(n_tiles, k))


def mean_pool(x: np.ndarray) -> np.ndarray:
    """Mean over a tile's tokens (rows)."""
    return x.sum(axis=0) / x.shape[0]


def tripool(x: np.ndarray) -> np.ndarray:
    """TripPool descriptor of a tile: avg, max and min over its tokens, concatenated (3d).

    BSAI VedaSparse README, "Core Technology" (Avg+Max+Min), "Implementation"
    (``_tripool``, which the README ties to its eq. 5).
    """
    return np.concatenate([mean_pool(x), x.max(axis=0), x.min(axis=0)])


def tile_scores(q_h: np.ndarray, k_h: np.ndarray, til: HeadTiling, cfg, h: int,
                gate=None, w_q=None, w_k=None, key_tiles=None) -> np.ndarray:
    """Scores S[i, j] for video query tile i and video key tile j of head h (fp64).

    ``q_h``/``k_h`` are the head's token rows ``[N, d]``. Prefix tiles are not
    scored: they are never pruned. ``key_tiles`` (a list of token-index arrays)
    replaces the video key tiles on the key side: the reference tiles of the
    R2VA budget variant are scored this way, against the same video query tiles.
    """
    key_tiles = til.video if key_tiles is None else key_tiles
    if cfg.score_mode == "meanpool_gate":
        g = np.asarray(gate, dtype=np.float64)
        qd = np.stack([mean_pool(q_h[t]) for t in til.video]) @ g
        kd = np.stack([mean_pool(k_h[t]) for t in key_tiles]) @ g
        width = g.shape[1]
    elif cfg.score_mode == "tripool":
        wq = np.asarray(w_q[h], dtype=np.float64)
        wk = np.asarray(w_k[h], dtype=np.float64)
        qd = np.stack([tripool(q_h[t]) for t in til.video]) @ wq
        kd = np.stack([tripool(k_h[t]) for t in key_tiles]) @ wk
        width = wq.shape[1]
    else:
        raise ValueError(cfg.score_mode)
    return (qd @ kd.T) / math.sqrt(width)


def ref_tiles(cfg) -> np.ndarray:
    """Indices (into the prefix tile list) of the tiles of reference segments: the
    prefix streams that the R2VA budget variant prunes with their own top-k (BSAI
    VedaSparse README, v3.4.2 notes on the R2VA predictor: 32 reference tiles and 32
    video tiles per query, text / VLM / audio conditioning always dense). Empty when
    no segment is marked."""
    flags = tuple(cfg.seg_ref) or (0,) * len(cfg.segments)
    out, t = [], 0
    for length, f in zip(cfg.segments, flags):
        n = -(-length // TILE)
        if f:
            out.extend(range(t, t + n))
        t += n
    return np.asarray(out, dtype=np.int64)


# ---------------------------------------------------------------------------
# 3. top-k selection
# ---------------------------------------------------------------------------


def topk_row(scores_row: np.ndarray, k: int) -> np.ndarray:
    """The k best key tiles of one query tile: by score descending, lower index first on ties.

    Veda news page, "Что делает Veda" (head-aware top-k forms the tile mask);
    Ref2VA VSA README item 2 (top-k only over generated-video key tiles).
    Returned sorted ascending.
    """
    j = np.arange(scores_row.shape[0])
    order = np.lexsort((j, -scores_row))
    return np.sort(order[:k])


# ---------------------------------------------------------------------------
# 4. attention
# ---------------------------------------------------------------------------


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Exact softmax attention of query rows over key rows, fp64.

    Returns (out, lse, row_sum): lse is the natural-log sum of exp of the
    scaled logits; row_sum is the sum of the normalised weights (1 up to
    rounding).
    """
    x = scale * (q @ k.T)
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    s = e.sum(axis=1, keepdims=True)
    p = e / s
    return p @ v, (m + np.log(s))[:, 0], p.sum(axis=1)


def query_key_tokens(til: HeadTiling, tile_id: int, kept_video, ref=None, kept_ref=None) -> np.ndarray:
    """Key tokens that query tile ``tile_id`` (index into ``til.all``) attends to.

    Prefix query tiles see every token (BSAI README "cond rows always dense";
    Ref2VA README item 1). Video query tiles see every prefix tile plus their
    kept video tiles (Ref2VA README items 1-2). With reference tiles ``ref``
    (prefix tile indices) a video query tile sees, of those, only ``kept_ref``
    (positions into ``ref``); the other prefix tiles stay dense.
    """
    if tile_id < til.n_prefix:
        return np.concatenate(til.all)
    prefix = til.prefix
    if ref is not None and len(ref):
        drop = set(int(ref[r]) for r in range(len(ref))) - set(int(ref[r]) for r in kept_ref)
        prefix = [t for i, t in enumerate(til.prefix) if i not in drop]
    return np.concatenate(prefix + [til.video[j] for j in kept_video])


@dataclasses.dataclass
class LayerResult:
    scores: list                 # per head [NTv_h, NTv_h] fp64
    kept: list                   # per head [NTv_h, k_h] int64 (ascending)
    out: np.ndarray              # [B, N, heads, d] fp64 (rows not computed are NaN)
    lse: np.ndarray              # [B, N, heads] fp64
    row_sum: np.ndarray          # [B, N, heads] fp64
    computed_pairs: int          # sum over computed query rows of their key count
    ref_scores: list = None      # per head [NTv_h, n_ref] fp64 (reference tiles of the R2VA variant)
    ref_kept: list = None        # per head [NTv_h, k_ref] positions into ref_tiles(cfg), ascending


def run_layer(cfg, q: np.ndarray, k: np.ndarray, v: np.ndarray, k_per_head,
              gate=None, w_q=None, w_k=None, query_tiles=None,
              heads=None, kept=None, kept_ref=None, qk_fp8=False) -> LayerResult:
    """The whole layer, in fp64: tile, score, select, attend.

    ``q``, ``k``, ``v``: ``[B, N, heads, d]`` (any float dtype; widened to fp64).
    ``query_tiles``: optional {head: iterable of tile ids into the head's tile
    list (prefix first, then video)} restricting which query tiles get
    attention rows; the others stay NaN. ``heads`` restricts the heads computed.
    ``kept``: optional {head: [NTv_h, k_h] array} (or {(b, head): ...}) of kept
    video tiles to attend with instead of the oracle's own top-k (the scores
    are still computed and returned). With reference segments (``cfg.seg_ref``),
    each video query tile also keeps its ``cfg.k_ref`` best reference tiles by the
    same scorer; ``kept_ref`` overrides that choice like ``kept``. ``qk_fp8``: the
    attention logits use Q and K quantised per packed tile to e4m3 with one fp32 scale
    per tile (:func:`quantize_tile_e4m3`); scoring and selection still use the bf16 inputs.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, Hh, d = q.shape
    scale = 1.0 / math.sqrt(d)
    heads = range(Hh) if heads is None else heads
    out = np.full((B, N, Hh, d), np.nan)
    lse = np.full((B, N, Hh), np.nan)
    row_sum = np.full((B, N, Hh), np.nan)
    all_scores, all_kept = [None] * Hh, [None] * Hh
    all_rs, all_rk = [None] * Hh, [None] * Hh
    ref = ref_tiles(cfg)
    pairs = 0
    for h in heads:
        til = head_tiling(cfg, h)
        kh = int(k_per_head[h])
        tiles_h = range(len(til.all)) if query_tiles is None else query_tiles.get(h, ())
        for b in range(B):
            s = tile_scores(q[b, :, h], k[b, :, h], til, cfg, h, gate, w_q, w_k)
            if kept is not None:
                kept_bh = np.asarray(kept[(b, h)] if (b, h) in kept else kept[h])
            else:
                kept_bh = np.stack([topk_row(s[i], kh) for i in range(til.n_video)])
            rs = rk = None
            if len(ref):
                rs = tile_scores(q[b, :, h], k[b, :, h], til, cfg, h, gate, w_q, w_k,
                                 key_tiles=[til.prefix[r] for r in ref])
                if kept_ref is not None:
                    rk = np.asarray(kept_ref[(b, h)] if (b, h) in kept_ref else kept_ref[h])
                else:
                    rk = np.stack([topk_row(rs[i], int(cfg.k_ref)) for i in range(til.n_video)])
            if b == 0:
                all_scores[h], all_kept[h] = s, kept_bh
                all_rs[h], all_rk[h] = rs, rk
            qa, ka = q[b, :, h], k[b, :, h]
            if qk_fp8:
                qa, ka = dequantized_tiles(qa, til), dequantized_tiles(ka, til)
            for t in tiles_h:
                qt = til.all[t]
                if t < til.n_prefix:
                    kv = query_key_tokens(til, t, None)
                else:
                    kv = query_key_tokens(til, t, kept_bh[t - til.n_prefix], ref,
                                          None if rk is None else rk[t - til.n_prefix])
                o, l, rsum = softmax_attention(qa[qt], ka[kv], v[b, kv, h], scale)
                out[b, qt, h], lse[b, qt, h], row_sum[b, qt, h] = o, l, rsum
                pairs += len(qt) * len(kv)
    return LayerResult(all_scores, all_kept, out, lse, row_sum, pairs, all_rs, all_rk)


# ---------------------------------------------------------------------------
# independent checks used to pin the oracle
# ---------------------------------------------------------------------------


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Brute-force N x N softmax attention per (batch, head), no tiles at all."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, N, Hh, d = q.shape
    out = np.empty_like(q)
    for b in range(B):
        for h in range(Hh):
            x = scale * (q[b, :, h] @ k[b, :, h].T)
            x -= x.max(axis=1, keepdims=True)
            p = np.exp(x)
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, h] = p @ v[b, :, h]
    return out


def masked_dense_attention(q_h: np.ndarray, k_h: np.ndarray, v_h: np.ndarray,
                           allowed: np.ndarray, scale: float) -> np.ndarray:
    """N x N attention of one head with an explicit 0/-inf mask (``allowed`` is boolean N x N)."""
    x = scale * (q_h @ k_h.T)
    x = np.where(allowed, x, -np.inf)
    x -= x.max(axis=1, keepdims=True)
    p = np.exp(x)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v_h


def exhaustive_topk(scores_row: np.ndarray, k: int) -> np.ndarray:
    """The k-subset with the largest score sum, ties broken toward lower indices.

    Enumerates every subset, so only for tiny rows. Among subsets with equal
    sums the lexicographically smallest sorted index tuple wins, which is the
    lower-index tie rule.
    """
    best, best_sum = None, -np.inf
    for sub in itertools.combinations(range(scores_row.shape[0]), k):
        s = float(np.sum(scores_row[list(sub)]))
        if s > best_sum:
            best, best_sum = sub, s
    return np.array(best, dtype=np.int64)


def attention_flops(cfg, k_per_head) -> int:
    """Algorithmic attention FLOPs: 4 * d * sum over valid query rows of their key count.

    Counts QK^T and PV only; softmax and any work on padding are excluded.
    Mirrors the "Attention computed: X% of full attention" accounting of the
    Veda node (Veda news page, "Узел ComfyUI").
    """
    ref = ref_tiles(cfg)
    total_pairs = 0
    for h in range(cfg.heads):
        til = head_tiling(cfg, h)
        n_pre_tok = sum(len(t) for t in til.prefix)
        n_all = cfg.n_tokens
        total_pairs += n_pre_tok * n_all
        # every video tile keeps k tiles (and k_ref reference tiles); their sizes
        # depend on which tiles are kept only when tiles are partial, so this
        # closed form needs full tiles
        sizes = [len(t) for t in til.video]
        if min(sizes) != TILE or any(len(til.prefix[r]) != TILE for r in ref):
            raise ValueError("closed-form count needs full video and reference tiles")
        seen_prefix = n_pre_tok - TILE * len(ref) + (TILE * int(cfg.k_ref) if len(ref) else 0)
        kh = int(k_per_head[h])
        total_pairs += sum(sizes) * (seen_prefix + kh * TILE)
    return 4 * cfg.head_dim * total_pairs * cfg.batch


# ---------------------------------------------------------------------------
# teacher tile map and tile recall (the Veda method's first stage)
# ---------------------------------------------------------------------------


def teacher_tiles(q_h: np.ndarray, k_h: np.ndarray, til: HeadTiling, scale: float) -> np.ndarray:
    """Teacher map of one head, fp64: T[i, j] is the largest weight that any token of video
    tile i gives any token of video tile j in FULL softmax attention, i.e. over every token of
    the sequence, prefix included (Veda news page, "Что делает Veda": full attention,
    max-pooled per tile pair, is the tile-level teacher distribution that the scorer learns).
    """
    keys = np.concatenate(til.all)
    start = np.cumsum([0] + [len(t) for t in til.all])       # tile t occupies keys[start[t]:start[t+1]]
    n_pre, n_vid = til.n_prefix, til.n_video
    T = np.zeros((n_vid, n_vid))
    for i, rows in enumerate(til.video):
        x = scale * (q_h[rows] @ k_h[keys].T)
        a = np.exp(x - x.max(axis=1, keepdims=True))
        a /= a.sum(axis=1, keepdims=True)                     # each row: weights over every key
        for j in range(n_vid):
            T[i, j] = a[:, start[n_pre + j]:start[n_pre + j + 1]].max()
    return T


def tile_recall(kept_row: np.ndarray, teacher_row: np.ndarray, k: int) -> float:
    """Share of the teacher's k best key tiles (ranked by :func:`topk_row`) that a selection
    keeps: the tile recall by which the BSAI VedaSparse README ("Core Technology") compares
    TripPool with mean pooling."""
    return len(np.intersect1d(kept_row, topk_row(teacher_row, k))) / k


# ---------------------------------------------------------------------------
# fp8 (e4m3) Q K^T with per-tile scales
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_round(x) -> np.ndarray:
    """Nearest value of the e4m3 format (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
    bits, subnormals below 2^-6, no infinities, largest finite 448), ties to the even
    mantissa, magnitudes above 448 saturated to 448. fp64 in, fp64 out (every e4m3 value is
    exact in fp64)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))   # exponent; subnormals share 2^-6's spacing
    step = 2.0 ** (e - 3)                               # 8 steps per binade
    q = np.minimum(np.round(a / step) * step, E4M3_MAX)   # np.round: half to even
    return np.sign(x) * q


def quantize_tile_e4m3(x: np.ndarray):
    """Per-tile fp8 quantisation of one packed tile's rows (the tile-skipping kernels on the
    Veda page run their QK^T in 8-bit with per-tile scales; the plainest reading): the scale
    s is the tile's largest magnitude / 448 in fp32 (1 for an all-zero tile), and each value
    is divided by s in fp32 (one correctly rounded division per element) and rounded to
    e4m3. Returns (codes as fp64 values, scale)."""
    xf = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(xf))) if xf.size else np.float32(0)
    scale = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
    return e4m3_round((xf / scale).astype(np.float64)), float(scale)


def dequantized_tiles(x_h: np.ndarray, til: HeadTiling) -> np.ndarray:
    """One head's token rows with every tile replaced by its e4m3 codes times its scale."""
    out = np.array(x_h, dtype=np.float64)
    for t in til.all:
        codes, scale = quantize_tile_e4m3(out[t])
        out[t] = codes * scale
    return out
