// C ABI of libvsa: plan construction, argument validation and the entry points.
#include <cuda_runtime.h>
#include <math.h>
#include <nvtx3/nvToolsExt.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "vsa_internal.h"

using vsa::Geometry;
using vsa::WorkItem;

namespace {

inline int cdiv(int a, int b) { return (a + b - 1) / b; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// One NVTX range per entry point (named after the call), for timeline tools.
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
};

// The kept tiles per head of one call: the caller's host array (each entry
// 1 .. min(video tiles of the head, k_max), k_max being the plan's index row
// width) or, for NULL, the plan's own k_per_head.
bool resolve_k(const vsa_plan* p, const int32_t* k_per_head, int32_t* out) {
  for (int h = 0; h < p->geo.Hh; ++h) {
    const int32_t k = k_per_head ? k_per_head[h] : p->geo.k[h];
    if (k < 1 || k > p->geo.ntv[h] || k > p->geo.k_max) return false;
    out[h] = k;
  }
  return true;
}

vsa_status fail(vsa_plan* p, vsa_status s) {
  if (p && s != VSA_OK) p->stats.errors++;
  return s;
}

// Work is launched on the current device; a plan's tables live on the device
// that was current when it was created, so the two must agree.
bool on_plan_device(const vsa_plan* p) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return cur == p->device;
}

// Host-side validation of a descriptor; no CUDA call is made here.
vsa_status validate(const vsa_desc& d) {
  if (d.batch < 1 || d.heads < 1 || d.heads > VSA_MAX_HEADS) return VSA_ERR_INVALID_ARG;
  if (d.head_dim != 64 && d.head_dim != 128) return VSA_ERR_INVALID_ARG;
  if (d.T < 1 || d.H < 1 || d.W < 1) return VSA_ERR_INVALID_ARG;
  if (d.n_segments < 0 || d.n_segments > VSA_MAX_SEGMENTS) return VSA_ERR_INVALID_ARG;
  int64_t n_pre = 0;
  for (int i = 0; i < d.n_segments; ++i) {
    if (d.seg_len[i] < 1) return VSA_ERR_INVALID_ARG;
    n_pre += d.seg_len[i];
  }
  const int64_t n_video = int64_t(d.T) * d.H * d.W;
  const int64_t n_tok = n_pre + n_video;
  if (n_tok >= (int64_t(1) << 31)) return VSA_ERR_INVALID_ARG;
  for (int h = 0; h < d.heads; ++h) {
    const int32_t* s = d.tile_shape[h];
    if (s[0] < 1 || s[1] < 1 || s[2] < 1 || s[0] * s[1] * s[2] != VSA_TILE) return VSA_ERR_INVALID_ARG;
    const int64_t ntv = int64_t(cdiv(d.T, s[0])) * cdiv(d.H, s[1]) * cdiv(d.W, s[2]);
    if (d.k_per_head[h] < 1 || d.k_per_head[h] > ntv) return VSA_ERR_INVALID_ARG;
  }
  if (d.score_mode == VSA_SCORE_MEANPOOL_GATE) {
    if (d.proj_dim != d.head_dim) return VSA_ERR_INVALID_ARG;
  } else if (d.score_mode == VSA_SCORE_TRIPPOOL) {
    if (d.proj_dim < 8 || d.proj_dim > 256 || d.proj_dim % 8 != 0) return VSA_ERR_INVALID_ARG;
  } else {
    return VSA_ERR_INVALID_ARG;
  }
  if (!(d.softmax_scale >= 0.0f) || isinf(d.softmax_scale)) return VSA_ERR_INVALID_ARG;
  // reference segments (R2VA budgets): flags 0/1 on existing segments, a budget per head
  int64_t n_ref = 0;
  for (int i = 0; i < VSA_MAX_SEGMENTS; ++i) {
    if (d.seg_ref[i] != 0 && d.seg_ref[i] != 1) return VSA_ERR_INVALID_ARG;
    if (d.seg_ref[i] && i >= d.n_segments) return VSA_ERR_INVALID_ARG;
    if (d.seg_ref[i]) n_ref += cdiv(d.seg_len[i], VSA_TILE);
  }
  for (int h = 0; h < d.heads; ++h)
    if (n_ref ? (d.k_ref_per_head[h] < 1 || d.k_ref_per_head[h] > n_ref) : d.k_ref_per_head[h] != 0)
      return VSA_ERR_INVALID_ARG;
  return VSA_OK;
}

// Pairs the video query tiles of one head: tiles (ti, hi, wi) and (ti, hi+1, wi)
// share one 128-row block; a leftover row (odd tile count along h) pairs along w.
void video_pairs(int nT, int nY, int nX, std::vector<std::pair<int, int>>& out) {
  std::vector<char> used(size_t(nT) * nY * nX, 0);
  std::vector<int> singles;
  for (int t = 0; t < nT; ++t)
    for (int y = 0; y < nY; ++y)
      for (int x = 0; x < nX; ++x) {
        const int a = (t * nY + y) * nX + x;
        if (used[a]) continue;
        if (y % 2 == 0 && y + 1 < nY) {
          const int b = a + nX;
          used[a] = used[b] = 1;
          out.emplace_back(a, b);
        } else {
          used[a] = 1;
          singles.push_back(a);
        }
      }
  for (size_t i = 0; i < singles.size(); i += 2)
    out.emplace_back(singles[i], i + 1 < singles.size() ? singles[i + 1] : -1);
}

}  // namespace

extern "C" {

const char* vsa_status_string(vsa_status s) {
  switch (s) {
    case VSA_OK: return "VSA_OK";
    case VSA_ERR_INVALID_ARG: return "VSA_ERR_INVALID_ARG: invalid argument";
    case VSA_ERR_UNSUPPORTED: return "VSA_ERR_UNSUPPORTED: shape not supported by these kernels";
    case VSA_ERR_CUDA: return "VSA_ERR_CUDA: CUDA call failed";
    case VSA_ERR_DEVICE_TIMEOUT: return "VSA_ERR_DEVICE_TIMEOUT: device-side wait ran out";
    case VSA_ERR_BAD_INDEX: return "VSA_ERR_BAD_INDEX: invalid kept-tile index list or NaN score";
    case VSA_ERR_NO_MEMORY: return "VSA_ERR_NO_MEMORY: allocation failed";
  }
  return "unknown vsa_status";
}

int32_t vsa_k_from_sparsity(double s, int32_t n) {
  if (!(s >= 0.0 && s <= 1.0) || n < 1) return 0;
  int64_t k = int64_t(n) - int64_t(floor(s * double(n) + 0.5));
  if (k < 1) k = 1;
  if (k > n) k = n;
  return int32_t(k);
}

vsa_status vsa_plan_create(const vsa_desc* desc, vsa_plan** out) {
  if (!out) return VSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!desc) return VSA_ERR_INVALID_ARG;
  vsa_status st = validate(*desc);
  if (st != VSA_OK) return st;
  const vsa_desc& d = *desc;

  vsa_plan* p = new (std::nothrow) vsa_plan();
  if (!p) return VSA_ERR_NO_MEMORY;
  p->desc = d;
  if (p->desc.softmax_scale == 0.0f) p->desc.softmax_scale = 1.0f / sqrtf(float(d.head_dim));

  Geometry& g = p->geo;
  memset(&g, 0, sizeof(g));
  g.B = d.batch;
  g.Hh = d.heads;
  g.d = d.head_dim;
  g.T = d.T;
  g.H = d.H;
  g.W = d.W;
  g.n_seg = d.n_segments;
  int tok = 0, tile = 0;
  for (int i = 0; i < d.n_segments; ++i) {
    g.seg_tok0[i] = tok;
    g.seg_tile0[i] = tile;
    g.seg_len[i] = d.seg_len[i];
    tok += d.seg_len[i];
    tile += cdiv(d.seg_len[i], VSA_TILE);
  }
  g.seg_tok0[d.n_segments] = tok;
  g.seg_tile0[d.n_segments] = tile;
  g.n_pre_tok = tok;
  g.n_pre_tiles = tile;
  g.n_tokens = tok + d.T * d.H * d.W;
  g.ntv_max = 0;
  g.k_max = 0;
  for (int h = 0; h < d.heads; ++h) {
    g.pt[h] = d.tile_shape[h][0];
    g.ph[h] = d.tile_shape[h][1];
    g.pw[h] = d.tile_shape[h][2];
    g.nY[h] = cdiv(d.H, g.ph[h]);
    g.nX[h] = cdiv(d.W, g.pw[h]);
    g.ntv[h] = cdiv(d.T, g.pt[h]) * g.nY[h] * g.nX[h];
    g.k[h] = d.k_per_head[h];
    g.ntv_max = std::max(g.ntv_max, g.ntv[h]);
    g.k_max = std::max(g.k_max, g.k[h]);
  }
  g.nt_max = g.n_pre_tiles + g.ntv_max;
  std::vector<int32_t> ref_tiles, prefix_ref(size_t(g.n_pre_tiles), -1);
  for (int i = 0; i < d.n_segments; ++i)
    if (d.seg_ref[i])
      for (int t = g.seg_tile0[i]; t < g.seg_tile0[i + 1]; ++t) {
        prefix_ref[size_t(t)] = int32_t(ref_tiles.size());
        ref_tiles.push_back(t);
      }
  g.n_ref = int32_t(ref_tiles.size());
  g.k_ref_max = 0;
  for (int h = 0; h < d.heads; ++h) {
    g.k_ref[h] = g.n_ref ? d.k_ref_per_head[h] : 0;
    g.k_ref_max = std::max(g.k_ref_max, g.k_ref[h]);
  }

  // the attention kernel builds each item's merged key list (at most every
  // tile of a head, 16-bit tile ids) in a per-CTA slice of global memory
  p->list_cap = g.nt_max;
  p->attn_smem_bytes = vsa::attn_smem_bytes(p->list_cap);
  if (p->attn_smem_bytes > 227 * 1024 || g.nt_max >= 65536) {
    delete p;
    return VSA_ERR_UNSUPPORTED;
  }

  vsa_plan_info& info = p->info;
  memset(&info, 0, sizeof(info));
  info.n_tokens = g.n_tokens;
  info.n_prefix_tiles = g.n_pre_tiles;
  info.nt_max = g.nt_max;
  info.ntv_max = g.ntv_max;
  for (int h = 0; h < d.heads; ++h) info.ntv[h] = g.ntv[h];
  info.k_max = g.k_max;
  info.packed_elems = int64_t(g.B) * g.Hh * g.nt_max * VSA_TILE * g.d;
  info.score_elems = int64_t(g.B) * g.Hh * g.ntv_max * g.ntv_max;
  info.index_elems = int64_t(g.B) * g.Hh * g.ntv_max * g.k_max;
  info.workspace_bytes = vsa::score_workspace_bytes(g, d.score_mode, d.proj_dim);
  info.lse_elems = int64_t(g.B) * g.Hh * g.nt_max * VSA_TILE;
  info.n_ref_tiles = g.n_ref;
  info.k_ref_max = g.k_ref_max;
  info.ref_score_elems = int64_t(g.B) * g.Hh * g.ntv_max * g.n_ref;
  info.ref_index_elems = int64_t(g.B) * g.Hh * g.ntv_max * g.k_ref_max;
  info.tile_scale_elems = int64_t(g.B) * g.Hh * g.nt_max;

  // tile valid counts
  std::vector<int32_t> counts(size_t(g.Hh) * g.nt_max, 0);
  for (int h = 0; h < g.Hh; ++h) {
    int32_t* c = &counts[size_t(h) * g.nt_max];
    for (int s = 0; s < g.n_seg; ++s)
      for (int t = g.seg_tile0[s]; t < g.seg_tile0[s + 1]; ++t)
        c[t] = std::min(VSA_TILE, g.seg_len[s] - (t - g.seg_tile0[s]) * VSA_TILE);
    const int nT = cdiv(g.T, g.pt[h]);
    for (int ti = 0; ti < nT; ++ti)
      for (int yi = 0; yi < g.nY[h]; ++yi)
        for (int xi = 0; xi < g.nX[h]; ++xi) {
          const int et = std::min(g.pt[h], g.T - ti * g.pt[h]);
          const int eh = std::min(g.ph[h], g.H - yi * g.ph[h]);
          const int ew = std::min(g.pw[h], g.W - xi * g.pw[h]);
          c[g.n_pre_tiles + (ti * g.nY[h] + yi) * g.nX[h] + xi] = et * eh * ew;
        }
  }

  // attention work list: head by head, prefix query blocks (heaviest) first
  std::vector<WorkItem> items;
  std::vector<std::pair<int, int>> pairs;
  for (int b = 0; b < g.B; ++b)
    for (int h = 0; h < g.Hh; ++h) {
      const int bh = b * g.Hh + h;
      for (int t = 0; t < g.n_pre_tiles; t += 2)
        items.push_back({bh, t, t + 1 < g.n_pre_tiles ? t + 1 : -1, 0});
      pairs.clear();
      video_pairs(cdiv(g.T, g.pt[h]), g.nY[h], g.nX[h], pairs);
      for (auto& pr : pairs)
        items.push_back({bh, g.n_pre_tiles + pr.first,
                         pr.second >= 0 ? g.n_pre_tiles + pr.second : -1, 1});
    }
  p->n_items = int64_t(items.size());
  info.attn_work_items = p->n_items;
  info.direct_attn = vsa::direct_attn_supported(p) ? 1 : 0;
  p->wait_ns = vsa::kDefaultWaitNs;
  p->test_hold = 0;

  // dense pair count (valid rows x valid keys) for the stats
  p->stats.dense_pairs = int64_t(g.B) * g.Hh * int64_t(g.n_tokens) * g.n_tokens;

  // device tables
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device);
  if (e == cudaSuccess) e = cudaMalloc(&p->d_tile_count, counts.size() * sizeof(int32_t));
  if (e == cudaSuccess) e = cudaMalloc(&p->d_items, items.size() * sizeof(WorkItem));
  if (e == cudaSuccess) e = cudaMalloc(&p->d_state, 64);
  if (e == cudaSuccess) {
    const size_t words = size_t(p->num_sms) * 2 * (size_t(p->list_cap) + size_t(p->list_cap / 32 + 2));
    e = cudaMalloc(&p->d_lists, words * sizeof(uint32_t));
  }
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_tile_count, counts.data(), counts.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_items, items.data(), items.size() * sizeof(WorkItem), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemset(p->d_state, 0, 64);
  if (e == cudaSuccess && g.n_pre_tiles > 0) {
    std::vector<int32_t> ref_table(ref_tiles);
    ref_table.insert(ref_table.end(), prefix_ref.begin(), prefix_ref.end());
    e = cudaMalloc(&p->d_ref_tiles, ref_table.size() * sizeof(int32_t));
    if (e == cudaSuccess)
      e = cudaMemcpy(p->d_ref_tiles, ref_table.data(), ref_table.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
    p->d_prefix_ref = p->d_ref_tiles ? p->d_ref_tiles + g.n_ref : nullptr;
  }
  // (re)resolve this device's address of the fixed scratch of vsa_tile_score_static, so
  // that a plan made after a device reset never uses the address of a discarded module
  if (e == cudaSuccess) e = vsa::refresh_static_scratch_address(p->device);
  if (e != cudaSuccess) {
    cudaGetLastError();
    vsa_status r = (e == cudaErrorMemoryAllocation) ? VSA_ERR_NO_MEMORY : VSA_ERR_CUDA;
    vsa_plan_destroy(p);
    return r;
  }
  *out = p;
  return VSA_OK;
}

vsa_status vsa_plan_destroy(vsa_plan* p) {
  if (!p) return VSA_OK;
  if (p->d_tile_count || p->d_items || p->d_state || p->d_lists || p->d_ref_tiles) {
    // wait for the plan's own device, then put the caller's current device back
    int cur = -1;
    const bool switch_dev = cudaGetDevice(&cur) == cudaSuccess && cur != p->device;
    if (switch_dev) cudaSetDevice(p->device);
    cudaDeviceSynchronize();
    if (p->d_tile_count) cudaFree(p->d_tile_count);
    if (p->d_ref_tiles) cudaFree(p->d_ref_tiles);
    if (p->d_items) cudaFree(p->d_items);
    if (p->d_state) cudaFree(p->d_state);
    if (p->d_lists) cudaFree(p->d_lists);
    if (switch_dev) cudaSetDevice(cur);
    cudaGetLastError();
  }
  delete p;
  return VSA_OK;
}

vsa_status vsa_plan_query(const vsa_plan* p, vsa_plan_info* out) {
  if (!p || !out) return VSA_ERR_INVALID_ARG;
  *out = p->info;
  return VSA_OK;
}

vsa_status vsa_plan_get_stats(const vsa_plan* p, vsa_plan_stats* out) {
  if (!p || !out) return VSA_ERR_INVALID_ARG;
  *out = p->stats;
  uint64_t pairs = 0;
  if (cudaMemcpy(&pairs, reinterpret_cast<const char*>(p->d_state) + 8, 8, cudaMemcpyDeviceToHost) !=
      cudaSuccess) {
    cudaGetLastError();
    return VSA_ERR_CUDA;
  }
  out->computed_pairs = int64_t(pairs);
  return VSA_OK;
}

vsa_status vsa_tile_pack(vsa_plan* p, const void* q, const void* k, const void* v, void* qp, void* kp,
                         void* vp, void* stream) {
  Range r("vsa_tile_pack");
  if (!p) return VSA_ERR_INVALID_ARG;
  const void* src[3] = {q, k, v};
  void* dst[3] = {qp, kp, vp};
  int n = 0;
  for (int i = 0; i < 3; ++i) {
    if (!src[i]) continue;
    if (!dst[i] || !aligned16(src[i]) || !aligned16(dst[i])) return fail(p, VSA_ERR_INVALID_ARG);
    ++n;
  }
  if (n == 0) return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_pack++;
  if (vsa::launch_pack(p, q, k, v, qp, kp, vp, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_tile_pack_pool(vsa_plan* p, const void* q, const void* k, const void* v, void* qp, void* kp,
                              void* vp, void* ws, void* stream) {
  Range r("vsa_tile_pack_pool");
  if (!p || !q || !k || !v || !qp || !kp || !vp || !ws) return fail(p, VSA_ERR_INVALID_ARG);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(qp) || !aligned16(kp) || !aligned16(vp) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_pack++;
  float *pq, *pk;
  vsa::score_pooled_ptrs(p, ws, &pq, &pk);
  if (vsa::launch_pack_pool(p, q, k, v, qp, kp, vp, pq, pk, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_tile_pack_pool_fp8(vsa_plan* p, const void* q, const void* k, const void* v, void* qp, void* kp,
                                  void* vp, void* qp8, void* kp8, float* q_scale, float* k_scale, void* ws,
                                  void* stream) {
  Range r("vsa_tile_pack_pool_fp8");
  if (!p || !q || !k || !v || !qp || !kp || !vp || !qp8 || !kp8 || !q_scale || !k_scale || !ws)
    return fail(p, VSA_ERR_INVALID_ARG);
  if (p->geo.d != 128) return fail(p, VSA_ERR_UNSUPPORTED);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(qp) || !aligned16(kp) || !aligned16(vp) ||
      !aligned16(qp8) || !aligned16(kp8) || !aligned16(q_scale) || !aligned16(k_scale) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_pack++;
  float *pq, *pk;
  vsa::score_pooled_ptrs(p, ws, &pq, &pk);
  if (vsa::launch_pack_pool(p, q, k, v, qp, kp, vp, pq, pk, static_cast<cudaStream_t>(stream), qp8, kp8, q_scale,
                            k_scale) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_sparse_attn_fp8(vsa_plan* p, const void* qp8, const void* kp8, const float* q_scale,
                               const float* k_scale, const void* vp, const int32_t* idx, const int32_t* k_per_head,
                               void* op, float* lse, void* stream) {
  Range r("vsa_sparse_attn_fp8");
  if (!p || !qp8 || !kp8 || !q_scale || !k_scale || !vp || !idx || !op) return fail(p, VSA_ERR_INVALID_ARG);
  if (p->geo.d != 128) return fail(p, VSA_ERR_UNSUPPORTED);
  if (!aligned16(qp8) || !aligned16(kp8) || !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(vp) ||
      !aligned16(idx) || !aligned16(op) || (lse && !aligned16(lse)))
    return fail(p, VSA_ERR_INVALID_ARG);
  int32_t k[VSA_MAX_HEADS];
  if (!resolve_k(p, k_per_head, k)) return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_attn++;
  if (vsa::launch_attn(p, qp8, kp8, vp, idx, nullptr, k, op, lse, static_cast<cudaStream_t>(stream), q_scale,
                       k_scale) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_tile_score_pooled(vsa_plan* p, const float* proj_q, const float* proj_k, float* scores, void* ws,
                                 void* stream) {
  Range r("vsa_tile_score_pooled");
  if (!p || !proj_q || !proj_k || !scores || !ws) return fail(p, VSA_ERR_INVALID_ARG);
  if (!aligned16(proj_q) || !aligned16(proj_k) || !aligned16(scores) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_score++;
  if (vsa::launch_project_score(p, proj_q, proj_k, scores, ws, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_tile_unpack(vsa_plan* p, const void* op, void* o, void* stream) {
  Range r("vsa_tile_unpack");
  if (!p || !op || !o || !aligned16(op) || !aligned16(o)) return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_unpack++;
  if (vsa::launch_unpack(p, op, o, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_tile_score(vsa_plan* p, const void* qp, const void* kp, const float* proj_q,
                          const float* proj_k, float* scores, void* ws, void* stream) {
  Range r("vsa_tile_score");
  if (!p || !qp || !kp || !proj_q || !proj_k || !scores || !ws) return fail(p, VSA_ERR_INVALID_ARG);
  if (!aligned16(qp) || !aligned16(kp) || !aligned16(proj_q) || !aligned16(proj_k) ||
      !aligned16(scores) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_score++;
  if (vsa::launch_score(p, qp, kp, proj_q, proj_k, scores, ws, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_topk_select(vsa_plan* p, const float* scores, const int32_t* k_per_head, int32_t* idx,
                           void* stream) {
  Range r("vsa_topk_select");
  if (!p || !scores || !idx || !aligned16(scores) || !aligned16(idx)) return fail(p, VSA_ERR_INVALID_ARG);
  int32_t k[VSA_MAX_HEADS];
  if (!resolve_k(p, k_per_head, k)) return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_select++;
  if (vsa::launch_topk(p, scores, idx, static_cast<cudaStream_t>(stream), k) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_sparse_attn(vsa_plan* p, const void* qp, const void* kp, const void* vp,
                           const int32_t* idx, const int32_t* k_per_head, void* op, float* lse, void* stream) {
  Range r("vsa_sparse_attn");
  if (!p || !qp || !kp || !vp || !idx || !op) return fail(p, VSA_ERR_INVALID_ARG);
  if (!aligned16(qp) || !aligned16(kp) || !aligned16(vp) || !aligned16(idx) || !aligned16(op) ||
      (lse && !aligned16(lse)))
    return fail(p, VSA_ERR_INVALID_ARG);
  int32_t k[VSA_MAX_HEADS];
  if (!resolve_k(p, k_per_head, k)) return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_attn++;
  if (vsa::launch_attn(p, qp, kp, vp, idx, nullptr, k, op, lse, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_tile_pool(vsa_plan* p, const void* q, const void* k, void* ws, void* stream) {
  Range r("vsa_tile_pool");
  if (!p || !q || !k || !ws) return fail(p, VSA_ERR_INVALID_ARG);
  if (!p->info.direct_attn) return fail(p, VSA_ERR_UNSUPPORTED);
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_pack++;
  float *pq, *pk;
  vsa::score_pooled_ptrs(p, ws, &pq, &pk);
  if (vsa::launch_pool(p, q, k, pq, pk, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_sparse_attn_direct(vsa_plan* p, const void* q, const void* k, const void* v, const int32_t* idx,
                                  const int32_t* k_per_head, void* o, float* lse, void* stream) {
  Range r("vsa_sparse_attn_direct");
  if (!p || !q || !k || !v || !idx || !o) return fail(p, VSA_ERR_INVALID_ARG);
  if (!p->info.direct_attn) return fail(p, VSA_ERR_UNSUPPORTED);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(o) ||
      (lse && !aligned16(lse)))
    return fail(p, VSA_ERR_INVALID_ARG);
  int32_t kk[VSA_MAX_HEADS];
  if (!resolve_k(p, k_per_head, kk)) return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_attn++;
  if (vsa::launch_attn_direct(p, q, k, v, idx, kk, o, lse, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_ref_score(vsa_plan* p, const void* kp, const float* proj_k, float* scores_ref, void* ws,
                         void* stream) {
  Range r("vsa_ref_score");
  if (!p || !kp || !proj_k || !scores_ref || !ws) return fail(p, VSA_ERR_INVALID_ARG);
  if (p->geo.n_ref == 0) return fail(p, VSA_ERR_INVALID_ARG);
  if (!aligned16(kp) || !aligned16(proj_k) || !aligned16(scores_ref) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_score++;
  if (vsa::launch_ref_score(p, kp, proj_k, scores_ref, ws, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_topk_select_ref(vsa_plan* p, const float* scores_ref, int32_t* idx_ref, void* stream) {
  Range r("vsa_topk_select_ref");
  if (!p || !scores_ref || !idx_ref || p->geo.n_ref == 0 || !aligned16(scores_ref) || !aligned16(idx_ref))
    return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_select++;
  if (vsa::launch_topk_ref(p, scores_ref, idx_ref, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_sparse_attn_ref(vsa_plan* p, const void* qp, const void* kp, const void* vp, const int32_t* idx,
                               const int32_t* idx_ref, const int32_t* k_per_head, void* op, float* lse,
                               void* stream) {
  Range r("vsa_sparse_attn_ref");
  if (!p || !qp || !kp || !vp || !idx || !idx_ref || !op || p->geo.n_ref == 0) return fail(p, VSA_ERR_INVALID_ARG);
  if (!aligned16(qp) || !aligned16(kp) || !aligned16(vp) || !aligned16(idx) || !aligned16(idx_ref) ||
      !aligned16(op) || (lse && !aligned16(lse)))
    return fail(p, VSA_ERR_INVALID_ARG);
  int32_t k[VSA_MAX_HEADS];
  if (!resolve_k(p, k_per_head, k)) return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  p->stats.calls_attn++;
  if (vsa::launch_attn(p, qp, kp, vp, idx, idx_ref, k, op, lse, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_layer_forward(vsa_plan* p, const void* q, const void* k, const void* v,
                             const float* proj_q, const float* proj_k, void* qp, void* kp, void* vp,
                             float* scores, int32_t* idx, void* op, float* lse, void* ws, void* o,
                             void* stream) {
  Range r("vsa_layer_forward");
  if (p && p->geo.n_ref) return fail(p, VSA_ERR_UNSUPPORTED);
  vsa_status s = vsa_tile_pack_pool(p, q, k, v, qp, kp, vp, ws, stream);
  if (s == VSA_OK) s = vsa_tile_score_pooled(p, proj_q, proj_k, scores, ws, stream);
  if (s == VSA_OK) s = vsa_topk_select(p, scores, nullptr, idx, stream);
  if (s == VSA_OK) s = vsa_sparse_attn(p, qp, kp, vp, idx, nullptr, op, lse, stream);
  if (s == VSA_OK) s = vsa_tile_unpack(p, op, o, stream);
  return s;
}

vsa_status vsa_teacher_tiles(vsa_plan* p, const void* qp, const void* kp, const float* lse, float* teacher,
                             void* stream) {
  Range r("vsa_teacher_tiles");
  if (!p || !qp || !kp || !lse || !teacher || !aligned16(qp) || !aligned16(kp) || !aligned16(lse) ||
      !aligned16(teacher))
    return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  if (vsa::launch_teacher(p, qp, kp, lse, teacher, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_index_overlap(vsa_plan* p, const int32_t* idx_a, const int32_t* idx_b,
                             const int32_t* k_per_head, int32_t* counts, void* stream) {
  Range r("vsa_index_overlap");
  if (!p || !idx_a || !idx_b || !counts || !aligned16(idx_a) || !aligned16(idx_b) || !aligned16(counts))
    return fail(p, VSA_ERR_INVALID_ARG);
  int32_t k[VSA_MAX_HEADS];
  if (!resolve_k(p, k_per_head, k)) return fail(p, VSA_ERR_INVALID_ARG);
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  if (vsa::launch_overlap(p, idx_a, idx_b, counts, static_cast<cudaStream_t>(stream), k) != cudaSuccess)
    return fail(p, VSA_ERR_CUDA);
  return VSA_OK;
}

vsa_status vsa_plan_set_wait_limit(vsa_plan* p, uint64_t limit_ns) {
  if (!p) return VSA_ERR_INVALID_ARG;
  if (limit_ns == 0) limit_ns = vsa::kDefaultWaitNs;
  if (limit_ns < 1000ull || limit_ns > 60000000000ull) return fail(p, VSA_ERR_INVALID_ARG);
  p->wait_ns = limit_ns;
  return VSA_OK;
}

vsa_status vsa_plan_set_test_hold(vsa_plan* p, int32_t on) {
  if (!p || (on != 0 && on != 1)) return fail(p, VSA_ERR_INVALID_ARG);
  p->test_hold = on;
  return VSA_OK;
}

vsa_status vsa_plan_check(vsa_plan* p) {
  if (!p) return VSA_ERR_INVALID_ARG;
  if (!on_plan_device(p)) return fail(p, VSA_ERR_INVALID_ARG);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(p, VSA_ERR_CUDA);
  uint32_t err = 0;
  e = cudaMemcpy(&err, p->d_state, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(p, VSA_ERR_CUDA);
  if (err) {
    if (cudaMemset(p->d_state, 0, 4) != cudaSuccess) return fail(p, VSA_ERR_CUDA);
    if (err & vsa::kErrTimeout) return fail(p, VSA_ERR_DEVICE_TIMEOUT);
    return fail(p, VSA_ERR_BAD_INDEX);
  }
  return VSA_OK;
}

}  // extern "C"
