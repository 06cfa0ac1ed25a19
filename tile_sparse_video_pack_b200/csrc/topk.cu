// a5: per-head top-k tile selection -- a radix select over order-preserving keys.
//
// For every (b, h, video query tile i): keep the k video key tiles with the
// largest scores, ties to the lower tile index, written ascending (Veda page,
// "Что делает Veda": head-aware top-k forms the tile mask; Ref2VA VSA README
// item 2: only video key tiles are pruned). One CTA per row: the row's scores
// become uint32 keys whose unsigned order is the float order (-0 folded onto
// +0), four 8-bit radix passes find the k-th largest key, and one ordered
// compaction pass writes the kept indices in ascending order.
#include <cuda_runtime.h>

#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of one int per thread; *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    const int s = warp_sums[w];
    if (w < warp) before += s;
    all += s;
  }
  __syncthreads();
  *total = all;
  return before + x - v;
}

// ref = false: video key tiles (columns ntv[h], k[h]); ref = true: the
// reference tiles of the R2VA budget variant (columns n_ref, k_ref[h]).
__global__ void __launch_bounds__(kThreads) topk_kernel(Geometry g, const float* __restrict__ scores,
                                                        int32_t* __restrict__ idx, uint32_t* __restrict__ err,
                                                        bool ref) {
  extern __shared__ uint32_t keys[];
  __shared__ int hist[256];
  __shared__ int warp_sums[kThreads / 32];
  __shared__ uint32_t sel_bin;
  __shared__ int sel_above, nan_flag;

  const int64_t row = blockIdx.x;
  const int i = int(row % g.ntv_max);
  const int bh = int(row / g.ntv_max);
  const int h = bh % g.Hh;
  if (i >= g.ntv[h]) return;                   // no such query tile in this head
  const int n = ref ? g.n_ref : g.ntv[h];       // columns
  const int k = ref ? g.k_ref[h] : g.k[h];
  const float* srow = scores + row * (ref ? g.n_ref : g.ntv_max);
  int32_t* out = idx + row * (ref ? g.k_ref_max : g.k_max);
  const int tid = threadIdx.x;

  if (tid == 0) nan_flag = 0;
  __syncthreads();
  for (int j = tid; j < n; j += kThreads) {
    const float f = srow[j];
    if (f != f) nan_flag = 1;
    keys[j] = order_key(f);
  }
  __syncthreads();
  if (nan_flag) {
    if (tid == 0) atomicOr(err, kErrBadIndex);
    return;
  }

  // k-th largest key: 8 bits at a time from the top
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    hist[tid] = 0;  // kThreads == 256 bins
    __syncthreads();
    for (int j = tid; j < n; j += kThreads) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    // thread t looks at bin 255 - t; inclusive count of keys in bins >= that bin
    const int c = hist[255 - tid];
    int tot;
    const int above = block_excl_scan(c, warp_sums, &tot);
    if (above < remaining && above + c >= remaining) {
      sel_bin = uint32_t(255 - tid);
      sel_above = above;
    }
    __syncthreads();
    remaining -= sel_above;
    prefix |= sel_bin << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t thr = prefix;   // the k-th largest key
  const int take_eq = remaining; // how many keys equal to thr are kept (lowest indices first)

  int base_eq = 0, base_out = 0;
  for (int j0 = 0; j0 < n; j0 += kThreads) {
    const int j = j0 + tid;
    const uint32_t key = j < n ? keys[j] : 0u;
    const int is_eq = (j < n && key == thr) ? 1 : 0;
    const int is_gt = (j < n && key > thr) ? 1 : 0;
    int tot_eq;
    const int eq_rank = base_eq + block_excl_scan(is_eq, warp_sums, &tot_eq);
    const int take = is_gt | (is_eq & (eq_rank < take_eq ? 1 : 0));
    int tot_take;
    const int pos = base_out + block_excl_scan(take, warp_sums, &tot_take);
    if (take) out[pos] = j;
    base_eq += tot_eq;
    base_out += tot_take;
  }
}

}  // namespace

cudaError_t launch_topk(const vsa_plan* p, const float* scores, int32_t* idx, cudaStream_t s, const int32_t* k) {
  Geometry g = p->geo;   // by value: this call's k per head
  for (int h = 0; h < g.Hh; ++h) g.k[h] = k[h];
  const int64_t rows = int64_t(g.B) * g.Hh * g.ntv_max;
  const size_t smem = size_t(g.ntv_max) * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  topk_kernel<<<unsigned(rows), kThreads, smem, s>>>(g, scores, idx, p->d_state, false);
  return cudaGetLastError();
}

cudaError_t launch_topk_ref(const vsa_plan* p, const float* scores_ref, int32_t* idx_ref, cudaStream_t s) {
  const Geometry& g = p->geo;
  const int64_t rows = int64_t(g.B) * g.Hh * g.ntv_max;
  const size_t smem = size_t(g.n_ref) * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  topk_kernel<<<unsigned(rows), kThreads, smem, s>>>(g, scores_ref, idx_ref, p->d_state, true);
  return cudaGetLastError();
}

}  // namespace vsa
