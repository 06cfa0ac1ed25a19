// Internal declarations shared by the libvsa CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/vsa.h"

namespace vsa {

// Default bound of every device-side wait of the tcgen05 kernels (two seconds).
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

// Bits of the device error word.
enum : uint32_t {
  kErrTimeout = 1u << 0,
  kErrBadIndex = 1u << 1,
};

// Tiling of one layer, passed by value to the element-wise kernels.
struct Geometry {
  int32_t B, Hh, d;
  int32_t T, H, W;
  int32_t n_tokens, n_pre_tok, n_pre_tiles, nt_max, ntv_max, k_max;
  int32_t n_seg;
  int32_t seg_tok0[VSA_MAX_SEGMENTS + 1];   // first token of each segment (+ end)
  int32_t seg_tile0[VSA_MAX_SEGMENTS + 1];  // first prefix tile of each segment (+ end)
  int32_t seg_len[VSA_MAX_SEGMENTS];
  int32_t pt[VSA_MAX_HEADS], ph[VSA_MAX_HEADS], pw[VSA_MAX_HEADS];
  int32_t nY[VSA_MAX_HEADS], nX[VSA_MAX_HEADS], ntv[VSA_MAX_HEADS];
  int32_t k[VSA_MAX_HEADS];
  // reference tiles of the R2VA budget variant (0 when no segment is marked)
  int32_t n_ref, k_ref_max;
  int32_t k_ref[VSA_MAX_HEADS];
};

// One 128-row block of attention work: two query tiles of one (batch, head)
// that share a merged key list (qb < 0: a single query tile).
struct WorkItem {
  int32_t bh;      // b * heads + h
  int32_t qa, qb;  // packed tile ids (prefix tiles first)
  int32_t kind;    // 0: prefix query tiles (dense rows), 1: video query tiles
};

}  // namespace vsa

struct vsa_plan {
  vsa_desc desc;
  vsa_plan_info info;
  vsa_plan_stats stats;
  vsa::Geometry geo;
  int device;
  int num_sms;
  // device tables
  int32_t* d_tile_count;   // [heads][nt_max] valid tokens per packed tile
  vsa::WorkItem* d_items;  // attention work list, heaviest first
  int64_t n_items;
  uint32_t* d_state;       // [0] error word, [1] work counter
  uint32_t* d_lists;       // attention key lists and bitmaps, one slice per CTA
  int32_t* d_ref_tiles;    // [n_ref] prefix tile ids of the reference tiles, then
  int32_t* d_prefix_ref;   // [n_pre_tiles] each prefix tile's position among them, or -1
  int attn_smem_bytes;
  int list_cap;            // entries of one key-list buffer in the attention kernel
  uint64_t wait_ns;        // bound of every device-side wait of the tcgen05 kernels
  int32_t test_hold;       // test hook: the attention softmax waits for a release nothing gives
};

namespace vsa {

// Launchers (return cudaGetLastError()).
cudaError_t launch_pack(const vsa_plan* p, const void* q, const void* k, const void* v, void* qp,
                        void* kp, void* vp, cudaStream_t s);
// qp8 != null: also the e4m3 copies of Q and K and their per-tile scales (head_dim 128)
cudaError_t launch_pack_pool(const vsa_plan* p, const void* q, const void* k, const void* v, void* qp,
                             void* kp, void* vp, float* pooled_q, float* pooled_k, cudaStream_t s,
                             void* qp8 = nullptr, void* kp8 = nullptr, float* q_scale = nullptr,
                             float* k_scale = nullptr);
cudaError_t launch_unpack(const vsa_plan* p, const void* op, void* o, cudaStream_t s);
// The score descriptors (pooled Q, K of every video tile) straight from the token-major Q, K.
cudaError_t launch_pool(const vsa_plan* p, const void* q, const void* k, float* pooled_q, float* pooled_k,
                        cudaStream_t s);
// Attention with every tile loaded straight from the token-major Q, K, V and O written
// token-major (batch 1, no reference tiles, video tiles partial only along t).
bool direct_attn_supported(const vsa_plan* p);
cudaError_t launch_attn_direct(vsa_plan* p, const void* q, const void* k, const void* v, const int32_t* idx,
                               const int32_t* kk, void* o, float* lse, cudaStream_t s);
cudaError_t launch_score(const vsa_plan* p, const void* qp, const void* kp, const float* proj_q,
                         const float* proj_k, float* scores, void* workspace, cudaStream_t s);
int64_t score_workspace_bytes(const Geometry& g, int score_mode, int proj_dim);
// Where the score stage keeps the pooled Q and K descriptors in a workspace.
void score_pooled_ptrs(const vsa_plan* p, void* workspace, float** pooled_q, float** pooled_k);
// Looks up (with `dev` current) and caches the device address of the fixed scratch
// array of vsa_tile_score_static.
cudaError_t refresh_static_scratch_address(int dev);
cudaError_t launch_project_score(const vsa_plan* p, const float* proj_q, const float* proj_k, float* scores,
                                 void* workspace, cudaStream_t s);
// k: kept tiles per head for this call (host array of `heads` entries, validated)
cudaError_t launch_topk(const vsa_plan* p, const float* scores, int32_t* idx, cudaStream_t s, const int32_t* k);
cudaError_t launch_topk_ref(const vsa_plan* p, const float* scores_ref, int32_t* idx_ref, cudaStream_t s);
cudaError_t launch_ref_score(const vsa_plan* p, const void* kp, const float* proj_k, float* scores_ref,
                             void* workspace, cudaStream_t s);
// q_scale != null: qp, kp are e4m3 tiles (head_dim 128) with per-tile scales q_scale, k_scale
// k: kept video tiles per head for this call (host array of `heads` entries, validated)
cudaError_t launch_attn(vsa_plan* p, const void* qp, const void* kp, const void* vp,
                        const int32_t* idx, const int32_t* idx_ref, const int32_t* k, void* op, float* lse,
                        cudaStream_t s, const float* q_scale = nullptr, const float* k_scale = nullptr);
int attn_smem_bytes(int list_cap);
cudaError_t launch_teacher(vsa_plan* p, const void* qp, const void* kp, const float* lse, float* teacher,
                           cudaStream_t s);
cudaError_t launch_overlap(vsa_plan* p, const int32_t* a, const int32_t* b, int32_t* counts, cudaStream_t s,
                           const int32_t* k);

}  // namespace vsa
