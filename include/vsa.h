/*
 * vsa.h -- C ABI of libvsa: tile-sparse video attention with a dense-exempt
 * conditioning prefix, for NVIDIA B200 (sm_100a).
 *
 * One attention layer of a video-diffusion transformer runs as five calls on
 * one CUDA stream:
 *
 *   vsa_tile_pack   -> vsa_tile_score -> vsa_topk_select -> vsa_sparse_attn
 *                                                       -> vsa_tile_unpack
 *
 * The method (tiles of 64 tokens; a prefix of text / reference-image /
 * reference-audio tokens in segment-pure tiles that are never pruned; per-head
 * top-k selection of video key tiles; exact softmax over the kept tiles) is
 * described on the Ref2VA VSA pages ("Патч внимания с двумя уровнями"; README
 * "two-tier attention layout") and the Veda / BSAI VedaSparse pages ("Что
 * делает Veda"; README "Core Technology", "Implementation").
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *    16-byte aligned, and stay valid until the stream reaches the call.
 *  - Q/K/V/O are bf16 (raw 16-bit patterns, passed as void*). There is no
 *    other dtype and no implicit conversion: anything else is rejected, as the
 *    Ref2VA VSA node rejects non-bf16 inputs instead of falling back
 *    ("From 650 s to 72 s", "The method" / "What transfers": fail loudly).
 *  - Calls are asynchronous on `stream` (a cudaStream_t, passed as void*; NULL
 *    is the legacy default stream). Argument errors are returned before
 *    anything is launched. Errors raised on the device are latched in the plan
 *    and returned by vsa_plan_check().
 *  - The library allocates only the plan's small tables and its error word.
 *    There is no CPU path and no fallback kernel.
 *  - A plan may be used by one stream at a time; calls on the same plan that
 *    overlap on the GPU share the attention kernel's work counter and race.
 *  - A plan belongs to the device that was current when it was created. Every
 *    call that launches work, and vsa_plan_check(), must be made with that
 *    device current; otherwise it returns VSA_ERR_INVALID_ARG and launches
 *    nothing.
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define VSA_API __attribute__((visibility("default")))
#else
#define VSA_API
#endif

#define VSA_TILE 64          /* tokens per tile */
#define VSA_MAX_HEADS 64
#define VSA_MAX_SEGMENTS 8

typedef enum {
  VSA_OK = 0,
  VSA_ERR_INVALID_ARG = 1,     /* bad pointer, size, shape or alignment */
  VSA_ERR_UNSUPPORTED = 2,     /* valid request these kernels do not handle */
  VSA_ERR_CUDA = 3,            /* a CUDA runtime or driver call failed */
  VSA_ERR_DEVICE_TIMEOUT = 4,  /* a device-side wait ran past its limit */
  VSA_ERR_BAD_INDEX = 5,       /* a kept-tile list holds an out-of-range or repeated tile */
  VSA_ERR_NO_MEMORY = 6        /* host or device allocation failed */
} vsa_status;

typedef enum {
  VSA_SCORE_MEANPOOL_GATE = 0, /* VSA: (mean(Q tile) G) . (mean(K tile) G) / sqrt(d) */
  VSA_SCORE_TRIPPOOL = 1       /* Veda: ([avg;max;min](Q) Wq[h]) . ([avg;max;min](K) Wk[h]) / sqrt(p) */
} vsa_score_mode;

/* Layer description. Sequence = prefix segments in order, then the video grid
 * T x H x W in (t, h, w) raster order (w fastest). Token-major tensors are
 * [batch, n_tokens, heads, head_dim]. */
typedef struct {
  int32_t batch;
  int32_t heads;                        /* 1 .. VSA_MAX_HEADS */
  int32_t head_dim;                     /* 64 or 128 */
  int32_t T, H, W;                      /* video latent grid, each >= 1 */
  int32_t n_segments;                   /* 0 .. VSA_MAX_SEGMENTS */
  int32_t seg_len[VSA_MAX_SEGMENTS];    /* prefix segment lengths (>= 1); any length: a
                                           segment's last tile may be partial */
  int32_t tile_shape[VSA_MAX_HEADS][3]; /* (pt, ph, pw) per head, pt*ph*pw == 64 */
  int32_t k_per_head[VSA_MAX_HEADS];    /* kept video key tiles per video query tile,
                                           1 .. number of video tiles of that head */
  int32_t score_mode;                   /* vsa_score_mode */
  int32_t proj_dim;                     /* mean-pool gate: == head_dim; TripPool: 8..256, a multiple of 8 */
  float softmax_scale;                  /* 0 -> 1/sqrt(head_dim) */
  /* R2VA budget variant (BSAI VedaSparse README, v3.4.2 notes on the R2VA
   * predictor: per query, 32 reference tiles and 32 video tiles; text / VLM /
   * audio conditioning stays dense). seg_ref[s] = 1 marks prefix segment s as
   * a reference stream: each video query tile keeps only k_ref_per_head[h] of
   * the reference segments' tiles, chosen by the layer's scorer
   * (vsa_ref_score, vsa_topk_select_ref, vsa_sparse_attn_ref). All zero: every
   * prefix tile is kept by every query tile, as in the default layer. */
  int32_t seg_ref[VSA_MAX_SEGMENTS];    /* 0 or 1 per segment */
  int32_t k_ref_per_head[VSA_MAX_HEADS];/* 1 .. reference tiles, when any seg_ref is set */
} vsa_desc;

/* Sizes a caller needs to allocate buffers for a plan. */
typedef struct {
  int64_t n_tokens;                     /* prefix + video tokens */
  int32_t n_prefix_tiles;               /* segment-pure prefix tiles (shared by all heads) */
  int32_t nt_max;                       /* tiles per head in the packed layout (max over heads) */
  int32_t ntv_max;                      /* video tiles, max over heads */
  int32_t ntv[VSA_MAX_HEADS];           /* video tiles of each head */
  int32_t k_max;                        /* max over heads of k_per_head */
  int64_t packed_elems;                 /* batch*heads*nt_max*64*head_dim (bf16 elements) */
  int64_t score_elems;                  /* batch*heads*ntv_max*ntv_max (fp32) */
  int64_t index_elems;                  /* batch*heads*ntv_max*k_max (int32) */
  int64_t workspace_bytes;              /* scratch for vsa_tile_score */
  int64_t lse_elems;                    /* batch*heads*nt_max*64 (fp32) */
  int64_t attn_work_items;              /* 128-row blocks the attention kernel schedules */
  int32_t n_ref_tiles;                  /* tiles of the reference segments (0: none) */
  int32_t k_ref_max;                    /* max over heads of k_ref_per_head (0: none) */
  int64_t ref_score_elems;              /* batch*heads*ntv_max*n_ref_tiles (fp32) */
  int64_t ref_index_elems;              /* batch*heads*ntv_max*k_ref_max (int32) */
  int64_t tile_scale_elems;             /* batch*heads*nt_max: one fp32 scale per packed tile (fp8 path) */
  int32_t direct_attn;                  /* 1: vsa_tile_pool + vsa_sparse_attn_direct can run this plan (no
                                           packed copies, slower); see vsa_sparse_attn_direct */
  int32_t reserved0;
} vsa_plan_info;

typedef struct vsa_plan vsa_plan;

/* Per-plan counters (host-side, updated by the calls). */
typedef struct {
  int64_t calls_pack, calls_score, calls_select, calls_attn, calls_unpack;
  int64_t errors;                       /* non-OK statuses returned by any call */
  int64_t computed_pairs;               /* (query row, key row) pairs the last attention call
                                           computed, counting valid rows only: the
                                           "attention computed X% of full attention" figure
                                           of the Veda node (Veda page, "Узел ComfyUI") */
  int64_t dense_pairs;                  /* valid query rows x valid key rows, all heads */
} vsa_plan_stats;

/* Validates `desc`, builds the tiling tables and the attention work list on
 * the host, and uploads them to the current CUDA device (the plan is bound to
 * that device). Blocks until the upload finishes. On any error *out is NULL.
 * Returns VSA_ERR_INVALID_ARG for a malformed descriptor (checked before any
 * CUDA call), VSA_ERR_UNSUPPORTED for shapes the kernels do not handle,
 * VSA_ERR_CUDA / VSA_ERR_NO_MEMORY for device failures. */
VSA_API vsa_status vsa_plan_create(const vsa_desc* desc, vsa_plan** out);

/* Frees the plan's device tables. Synchronises the plan's device first (making
 * it current for the call and restoring the caller's device after). NULL is OK. */
VSA_API vsa_status vsa_plan_destroy(vsa_plan* plan);

VSA_API vsa_status vsa_plan_query(const vsa_plan* plan, vsa_plan_info* out);
VSA_API vsa_status vsa_plan_get_stats(const vsa_plan* plan, vsa_plan_stats* out);

/* Kept tiles for a sparsity s in [0, 1] over n video tiles:
 * n - floor(s*n + 0.5) clamped to [1, n] (the pruned share of video key tiles;
 * Ref2VA VSA README: "75% video sparsity top-k"). Returns 0 for bad input. */
VSA_API int32_t vsa_k_from_sparsity(double sparsity, int32_t n_tiles);

/* a1. Pack token-major Q, K, V ([B, N, heads, d] bf16) into tile-major
 * [B, heads, nt_max, 64, d] bf16. Slot s of tile n of head h holds that tile's
 * s-th token; prefix tiles come first (segment order, 64 consecutive tokens
 * of one segment each), then video tiles in (ti, hi, wi) raster order with
 * tokens in (t, h, w) raster order inside the tile; a partial tile's tokens
 * fill its first slots. Unused slots and unused trailing tiles are zero.
 * Tiling: Ref2VA VSA README (4x4x4 tiles, segment-pure prefix tiles); BSAI
 * VedaSparse README "Core Technology: Head-Aware Tiling" and "Implementation"
 * (_tile_3d returns tiles and their key mask). Any of q/k/v may be NULL to
 * skip it (its packed pointer is then ignored). */
VSA_API vsa_status vsa_tile_pack(vsa_plan* plan, const void* q, const void* k, const void* v,
                         void* qp, void* kp, void* vp, void* stream);

/* a2-a4. Pool every video tile of packed Q and K (mean, or avg/max/min for
 * TripPool) in fp32, project, and write the tile scores
 * scores[b][h][i][j] (fp32, [B, heads, ntv_max, ntv_max]; rows/cols past a
 * head's own ntv are left untouched) for video query tile i and video key tile
 * j. proj_q/proj_k are fp32 device arrays: mean-pool gate -> both point to G
 * [d][d] (row-major; q_hat = mean(Q) G); TripPool -> Wq, Wk [heads][3d][p].
 * workspace: >= workspace_bytes of device scratch, 256-byte aligned.
 * Ref2VA VSA README (gating projection to_gate_compress decides which tiles
 * each query attends to); BSAI VedaSparse README "Core Technology: TripPool",
 * "Scorer Modes" (eq. 5 descriptor, eq. 6 per-head projection score). */
VSA_API vsa_status vsa_tile_score(vsa_plan* plan, const void* qp, const void* kp,
                          const float* proj_q, const float* proj_k, float* scores,
                          void* workspace, void* stream);

/* a1 + a2 in one pass (the fused form of the first two steps): pack Q, K and V
 * exactly as vsa_tile_pack and, while each video tile's Q and K rows pass
 * through, pool them as vsa_tile_score does (fp32 mean over the tile's valid
 * tokens; TripPool adds max and min), writing the descriptors into
 * `workspace` (>= workspace_bytes, 256-byte aligned). Follow with
 * vsa_tile_score_pooled on the same workspace. q, k and v are all required.
 * This saves the score stage's second read of packed Q and K. Same sources as
 * vsa_tile_pack and vsa_tile_score (Ref2VA VSA README: mean-pooled gate score;
 * BSAI VedaSparse README "Core Technology: TripPool", eq. 5). */
VSA_API vsa_status vsa_tile_pack_pool(vsa_plan* plan, const void* q, const void* k, const void* v,
                              void* qp, void* kp, void* vp, void* workspace, void* stream);

/* a3-a4 of vsa_tile_score from the descriptors vsa_tile_pack_pool left in
 * `workspace`: projection and tile scores, same arguments (less qp, kp),
 * layout and results as vsa_tile_score. */
VSA_API vsa_status vsa_tile_score_pooled(vsa_plan* plan, const float* proj_q, const float* proj_k,
                                 float* scores, void* workspace, void* stream);

/* The a2-a4 score stage of vsa_tile_score with its scratch in a fixed device
 * array owned by the library instead of a caller workspace, for callers that
 * may not allocate device memory while they run the layer: code under another
 * framework's memory planner or fixed arena, plugins that must not call
 * cudaMalloc (it can synchronise the device, or fail part-way through a step),
 * latency-critical loops. The pages describe no such call; it has no
 * counterpart there.
 *  - The scratch is a 32 MiB array in device memory, held by every GPU that
 *    loads this library until the process exits. Plans whose workspace_bytes
 *    exceed 32 MiB are rejected with VSA_ERR_UNSUPPORTED.
 *  - The call allocates nothing. The array's device address is looked up
 *    (cudaGetSymbolAddress, with the device current) by every
 *    vsa_plan_create and kept per device; if no plan had been created on
 *    the device, the first call of this function looks it up instead, so
 *    make that first call before any stream capture. After a
 *    cudaDeviceReset, create new plans (old ones are invalid anyway): that
 *    refreshes the address.
 *  - Plans with reference segments (seg_ref) are rejected with
 *    VSA_ERR_UNSUPPORTED: vsa_ref_score needs the projected pooled Q in the
 *    caller's workspace, which this call does not write.
 *  - The current device must be the plan's device (else VSA_ERR_INVALID_ARG).
 *  - Every call on a device shares the one array, which keeps the last
 *    call's contents (each call writes every scratch element before reading
 *    it, so nothing needs clearing). Calls whose kernels overlap on the GPU --
 *    on different streams, plans or threads -- race on it.
 * Arguments, layout and results are those of vsa_tile_score without the
 * workspace argument. */
VSA_API vsa_status vsa_tile_score_static(vsa_plan* plan, const void* qp, const void* kp,
                                         const float* proj_q, const float* proj_k, float* scores,
                                         void* stream);

/* Per-call k. k_per_head, where the calls below take it, is a HOST array of
 * `heads` int32 values read during the call (the caller keeps ownership; it
 * may be reused as soon as the call returns): the kept video key tiles per
 * video query tile of each head for this call, each in 1 .. min(video tiles of
 * the head, k_max of the plan) -- k_max, the largest k_per_head of the plan's
 * descriptor, is the row width of the index tables. NULL means the plan's own
 * k_per_head. Any other value is rejected with VSA_ERR_INVALID_ARG before
 * anything is launched. One plan created at the largest k thus serves every
 * smaller sparsity (Ref2VA VSA README: "75% video sparsity top-k"; BSAI
 * VedaSparse README, "Nodes": keep_percent per run). The top-k and attention
 * calls of one layer must be given the same k. */

/* a5. For every (b, h, video query tile i) keep the k[h] video key tiles with
 * the largest scores (k from k_per_head, above); equal scores keep the lower
 * tile index. The kept tile indices (0-based video tile ids) are written
 * sorted ascending to idx[b][h][i][0 .. k[h]-1] (int32, [B, heads, ntv_max,
 * k_max]; entries past k[h] untouched). -0.0 and +0.0 compare equal; NaN
 * scores are rejected on the device (VSA_ERR_BAD_INDEX via vsa_plan_check).
 * Veda page "Что делает Veda" (head-aware top-k forms the tile mask); Ref2VA
 * VSA README item 2 (top-k only over video key tiles). */
VSA_API vsa_status vsa_topk_select(vsa_plan* plan, const float* scores, const int32_t* k_per_head, int32_t* idx,
                                   void* stream);

/* a6. Block-sparse exact attention on packed tiles. A prefix query tile
 * attends to every valid key of its head; a video query tile attends to every
 * prefix tile plus the video tiles listed in idx[b][h][i][0 .. k[h]-1] (k from
 * k_per_head, as for vsa_topk_select; ascending,
 * distinct, in range -- otherwise the rows are skipped and VSA_ERR_BAD_INDEX is
 * latched). o = softmax(scale * q k^T over the valid keys) v, fp32 accumulation,
 * written as bf16 to op ([B, heads, nt_max, 64, d]); rows of unused slots of
 * a head's tiles are zero, and tiles past a head's own tile count (heads with
 * fewer video tiles than ntv_max) are not written. lse (nullable, fp32
 * [B, heads, nt_max, 64]) gets the natural-log sum-exp of the scaled logits per
 * row (0 for unused slots, not written past a head's tiles).
 * BSAI VedaSparse README "Core Technology: Tile-Skipping", "v3.4 Highlights"
 * (sink = exact_kv_and_rows: conditioning rows and keys stay exact). */
VSA_API vsa_status vsa_sparse_attn(vsa_plan* plan, const void* qp, const void* kp, const void* vp,
                           const int32_t* idx, const int32_t* k_per_head, void* op, float* lse, void* stream);

/* a7. Inverse of the pack permutation: [B, heads, nt_max, 64, d] -> [B, N, heads, d]. */
VSA_API vsa_status vsa_tile_unpack(vsa_plan* plan, const void* op, void* o, void* stream);

/* The layer without packed copies (the other half of fusing a1 and a2: tiles
 * straight from the token-major tensors), for callers that cannot hold the
 * packed Q, K, V and O (four tensors the size of Q). It is the slower path:
 * a tile of the token-major layout is 64 rows 128 or 256 bytes long spread
 * over the tensor, which the TMA engine fetches several times more slowly
 * than one contiguous packed tile, so the attention takes about three times
 * as long as on packed tiles (full clip: 181 ms against 59 ms); the pack
 * pass costs 0.7 ms. For plans whose vsa_plan_info direct_attn is 1 --
 * batch 1, no reference segments (seg_ref), head_dim 64 or 128, every head's
 * video tiles whole along h and w (only tiles at the far end of t may be
 * partial), at most four distinct tile shapes -- the two calls below replace
 * vsa_tile_pack_pool, vsa_sparse_attn and vsa_tile_unpack; any other plan
 * gets VSA_ERR_UNSUPPORTED from them.
 *
 * vsa_tile_pool: a2 alone -- the score descriptors of every video tile, pooled
 * from the token-major q and k ([1, N, heads, d] bf16, 16-byte aligned) into
 * `workspace` exactly as vsa_tile_pack_pool pools them; follow with
 * vsa_tile_score_pooled on the same workspace. */
VSA_API vsa_status vsa_tile_pool(vsa_plan* plan, const void* q, const void* k, void* workspace, void* stream);

/* a6 + a7 without packed tiles: the attention of vsa_sparse_attn, reading each
 * tile of q, k, v ([1, N, heads, d] bf16, token-major, 16-byte aligned) with
 * one multi-dimensional TMA box (a prefix tile: 64 consecutive tokens of its
 * segment; a video tile: its (pt, ph, pw) block of the grid) and writing o
 * ([1, N, heads, d] bf16, token-major) directly -- the same values, bit for
 * bit, as vsa_sparse_attn followed by vsa_tile_unpack. idx, k_per_head and lse
 * (packed rows, [B, heads, nt_max, 64], may be NULL) as for vsa_sparse_attn. */
VSA_API vsa_status vsa_sparse_attn_direct(vsa_plan* plan, const void* q, const void* k, const void* v,
                                          const int32_t* idx, const int32_t* k_per_head, void* o, float* lse,
                                          void* stream);

/* R2VA budgets, scores of the reference tiles: for video query tile i and
 * reference tile r (the r-th tile of the segments marked in seg_ref, in
 * sequence order), scores_ref[b][h][i][r] = the layer's tile score of query
 * tile i against reference tile r (pooled K of tile r, projected with proj_k,
 * against the projected pooled Q of tile i), fp32 [B, heads, ntv_max,
 * n_ref_tiles]. `workspace` must hold the projected pooled Q that
 * vsa_tile_score or vsa_tile_score_pooled just wrote into it; this call adds
 * the reference tiles' pooled and projected K behind it (workspace_bytes
 * covers both). kp: packed K. Same scorer and sources as vsa_tile_score. */
VSA_API vsa_status vsa_ref_score(vsa_plan* plan, const void* kp, const float* proj_k, float* scores_ref,
                         void* workspace, void* stream);

/* R2VA budgets, a5 for the reference tiles: the k_ref_per_head[h] best
 * reference tiles of each video query tile, ties to the lower index, written
 * ascending into idx_ref [B, heads, ntv_max, k_ref_max] (positions 0 ..
 * n_ref_tiles - 1). As vsa_topk_select. */
VSA_API vsa_status vsa_topk_select_ref(vsa_plan* plan, const float* scores_ref, int32_t* idx_ref,
                               void* stream);

/* R2VA budgets, a6: vsa_sparse_attn in which a video query tile keeps, of the
 * reference segments' tiles, only those idx_ref lists for it; the other
 * prefix tiles stay dense and prefix query rows still see every key. Indices
 * out of range or not ascending are rejected as in vsa_sparse_attn. */
VSA_API vsa_status vsa_sparse_attn_ref(vsa_plan* plan, const void* qp, const void* kp, const void* vp,
                               const int32_t* idx, const int32_t* idx_ref, const int32_t* k_per_head, void* op,
                               float* lse, void* stream);

/* fp8 Q K^T (row f2; the tile-skipping kernels on the Veda page run Q K^T in
 * 8-bit with per-tile scales). vsa_tile_pack_pool, and besides: Q and K of
 * every packed tile as e4m3 bytes qp8, kp8 ([B, heads, nt_max, 64, head_dim]
 * bytes, packed_elems of them) with one fp32 scale per (tile, tensor) in
 * q_scale, k_scale ([B, heads, nt_max], tile_scale_elems): with amax the
 * tile's largest magnitude, scale = amax / 448 (fp32; 1 for an all-zero tile)
 * and code = e4m3(x / scale) (correctly rounded fp32 division, then round to
 * nearest even, saturating).
 * head_dim 128 only (VSA_ERR_UNSUPPORTED otherwise). */
VSA_API vsa_status vsa_tile_pack_pool_fp8(vsa_plan* plan, const void* q, const void* k, const void* v,
                                  void* qp, void* kp, void* vp, void* qp8, void* kp8, float* q_scale,
                                  float* k_scale, void* workspace, void* stream);

/* vsa_sparse_attn with the logits from the e4m3 tiles: s = (q8 . k8) *
 * q_scale[query tile] * k_scale[key tile] * softmax_scale, accumulated in
 * fp32 on the tensor cores; P and V stay bf16. qp8, kp8, q_scale, k_scale as
 * written by vsa_tile_pack_pool_fp8; vp the bf16 packed V. head_dim 128. */
VSA_API vsa_status vsa_sparse_attn_fp8(vsa_plan* plan, const void* qp8, const void* kp8, const float* q_scale,
                               const float* k_scale, const void* vp, const int32_t* idx, const int32_t* k_per_head,
                               void* op, float* lse, void* stream);

/* Teacher tile map (row f3; the first stage of the Veda method: full attention,
 * max-pooled per tile pair, is the teacher distribution at tile level -- Veda
 * news page, "Что делает Veda"). For video query tile i and video key tile j
 * of every (batch, head):
 *   teacher[b][h][i][j] = max over valid rows r of tile i and valid keys c of
 *                         tile j of exp(scale * q_r . k_c - lse[r]),
 * the largest full-attention weight a token of tile i puts on a token of tile
 * j. lse ([B, heads, nt_max, 64] fp32, natural log) must be the row
 * log-sum-exp over EVERY key: the lse output of vsa_sparse_attn on a plan
 * with k = every video tile. qp, kp: packed bf16 as from vsa_tile_pack.
 * teacher: fp32 [B, heads, ntv_max, ntv_max] (the layout of the scores of
 * vsa_tile_score, so vsa_topk_select ranks it); entries past a head's own
 * ntv are left untouched. Cost: a dense Q K^T over all video tile pairs. */
VSA_API vsa_status vsa_teacher_tiles(vsa_plan* plan, const void* qp, const void* kp, const float* lse,
                             float* teacher, void* stream);

/* For every (batch, head, video query tile) row of two index tables
 * ([B, heads, ntv_max, k_max] int32, ascending rows of k[h] entries, k from
 * k_per_head as for vsa_topk_select): the number of indices the rows share, in
 * counts [B, heads, ntv_max] (0 for rows past a head's ntv). With a = the
 * scorer's selection and b = the teacher's top-k, counts / k is the tile
 * recall of the scorer (BSAI VedaSparse README, "Core Technology": TripPool
 * tile recall against full attention). */
VSA_API vsa_status vsa_index_overlap(vsa_plan* plan, const int32_t* idx_a, const int32_t* idx_b,
                             const int32_t* k_per_head, int32_t* counts, void* stream);

/* The whole layer in order on one stream, on caller-provided buffers (sizes
 * from vsa_plan_query): vsa_tile_pack_pool, vsa_tile_score_pooled,
 * vsa_topk_select, vsa_sparse_attn, vsa_tile_unpack. Returns the first
 * failing call's status. Plans with reference segments (seg_ref) return
 * VSA_ERR_UNSUPPORTED: their layer adds vsa_ref_score and
 * vsa_topk_select_ref and attends with vsa_sparse_attn_ref. */
VSA_API vsa_status vsa_layer_forward(vsa_plan* plan, const void* q, const void* k, const void* v,
                             const float* proj_q, const float* proj_k,
                             void* qp, void* kp, void* vp, float* scores, int32_t* idx,
                             void* op, float* lse, void* workspace, void* o, void* stream);

/* Bound of every device-side wait of the plan's tcgen05 kernels (attention,
 * teacher map), in nanoseconds: 1,000 .. 60,000,000,000; 0 restores the
 * default of two seconds. A kernel whose wait runs past it stops: it latches
 * VSA_ERR_DEVICE_TIMEOUT (returned by vsa_plan_check), lets its own copies and
 * tensor-core work finish, frees its tensor memory and returns, leaving the
 * CUDA context usable (fail loudly, never hang: "From 650 s to 72 s", "What
 * transfers"). Host-side setting, read at each launch. */
VSA_API vsa_status vsa_plan_set_wait_limit(vsa_plan* plan, uint64_t limit_ns);

/* Test hook for the timeout path above; no counterpart on the pages. With
 * on = 1, every later attention launch of this plan has its softmax warps,
 * after their first block of scores, wait on a barrier that nothing arrives
 * on, so each CTA runs into the wait limit and takes the abort path with
 * copies and tensor-core work in flight. on = 0 (the default) turns it off.
 * Not for production use. */
VSA_API vsa_status vsa_plan_set_test_hold(vsa_plan* plan, int32_t on);

/* Waits for the plan's device (cudaDeviceSynchronize), then returns and clears
 * the latched device error (VSA_OK if none), or VSA_ERR_CUDA if the device
 * reports a CUDA error. */
VSA_API vsa_status vsa_plan_check(vsa_plan* plan);

VSA_API const char* vsa_status_string(vsa_status status);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H_ */
