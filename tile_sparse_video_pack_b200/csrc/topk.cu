// a5: per-head top-k tile selection -- one warp per row, two passes.
//
// For every (b, h, video query tile i): keep the k video key tiles with the
// largest scores, ties to the lower tile index, written ascending (Veda page,
// "Что делает Veda": head-aware top-k forms the tile mask; Ref2VA VSA README
// item 2: only video key tiles are pruned).
//
// One warp per row, several rows per CTA, no block-wide barriers. The row's
// scores become uint32 keys whose unsigned order is the float order (-0 folded
// onto +0) and stay in the warp's slice of shared memory. A histogram of 512
// value bins between the row's minimum and maximum (a monotone map in fp32:
// bin = (f - min) * (512 / (max - min)), truncated) finds the bin that holds
// the k-th largest score; the exact threshold key comes from that bin's few
// candidates by counting, or, when the bin holds more than 64 (many equal
// scores, or one outlier that makes the bins coarse), from an 8-bit radix
// select restricted to the bin. A last pass writes the kept indices in
// ascending order: every key above the threshold and the lowest-indexed keys
// equal to it.
#include <cuda_runtime.h>

#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int kBins = 512;        // value bins of the first pass
constexpr int kSmall = 64;        // candidates resolved by counting
constexpr int kMaxWarps = 4;      // rows (warps) per CTA
constexpr int kLoads = 16;        // score loads in flight per lane

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}
__device__ __forceinline__ int value_bin(uint32_t key, float lo, float inv) {
  const int b = int(__fmul_rn(__fsub_rn(key_value(key), lo), inv));   // >= 0, truncated
  return b < kBins - 1 ? b : kBins - 1;
}
__device__ __forceinline__ uint32_t lanes_below(int lane) { return (1u << lane) - 1u; }

// Bin b of nb (lanes own nb / 32 consecutive bins) such that the counts of
// the bins above it sum to fewer than need and, with its own count, to at
// least need. Returns the bin; *above gets the count above it.
__device__ __forceinline__ int find_bin(const int* hist, int nb, int need, int lane, int* above) {
  const int per = nb / 32;
  int own = 0;
  for (int t = 0; t < per; ++t) own += hist[lane * per + t];
  int suffix = own;   // counts of lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, suffix, o);
    if (lane + o < 32) suffix += y;
  }
  int run = suffix - own;  // counts of the bins above this lane's
  int bin = -1, run_at = 0;
  if (run < need && suffix >= need) {
    for (int t = per - 1; t >= 0; --t) {
      const int c = hist[lane * per + t];
      if (run + c >= need) {
        bin = lane * per + t;
        run_at = run;
        break;
      }
      run += c;
    }
  }
  const uint32_t who = __ballot_sync(0xffffffffu, bin >= 0);
  const int src = __ffs(who) - 1;   // exactly one lane: 1 <= need <= total
  *above = __shfl_sync(0xffffffffu, run_at, src);
  return __shfl_sync(0xffffffffu, bin, src);
}

// need-th largest key among the row's keys that pass `in` (8 bits at a time).
template <typename Pred>
__device__ uint32_t radix_select(const uint32_t* keys, int n, int need, int* hist, int lane, Pred in) {
  uint32_t prefix = 0, mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix && in(key)) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncwarp();
    int above;
    const int digit = find_bin(hist, 256, need, lane, &above);
    need -= above;
    prefix |= uint32_t(digit) << shift;
    mask |= 255u << shift;
    __syncwarp();   // the histogram is cleared next pass
  }
  return prefix;
}

// ref = false: video key tiles (columns ntv[h], k[h]); ref = true: the
// reference tiles of the R2VA budget variant (columns n_ref, k_ref[h]).
__global__ void __launch_bounds__(kMaxWarps * 32) topk_kernel(Geometry g, const float* __restrict__ scores,
                                                              int32_t* __restrict__ idx,
                                                              uint32_t* __restrict__ err, bool ref,
                                                              int key_stride) {
  extern __shared__ uint32_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  uint32_t* keys = smem + size_t(warp) * (key_stride + kBins);
  int* hist = reinterpret_cast<int*>(keys + key_stride);
  const int64_t rows = int64_t(g.B) * g.Hh * g.ntv_max;

  for (int64_t row = int64_t(blockIdx.x) * warps + warp; row < rows; row += int64_t(gridDim.x) * warps) {
    const int i = int(row % g.ntv_max);
    const int bh = int(row / g.ntv_max);
    const int h = bh % g.Hh;
    if (i >= g.ntv[h]) continue;                  // no such query tile in this head (warp-uniform)
    const int n = ref ? g.n_ref : g.ntv[h];       // columns
    const int k = ref ? g.k_ref[h] : g.k[h];
    const float* srow = scores + row * (ref ? g.n_ref : g.ntv_max);
    int32_t* out = idx + row * (ref ? g.k_ref_max : g.k_max);
    if (n < 1 || k < 1 || k > n) {               // the plan rules this out; never index past the row
      if (lane == 0) atomicOr(err, kErrBadIndex);
      continue;
    }

    // keys, range, NaN check; the row streams from memory, so each lane keeps
    // kLoads loads in flight before it uses any of them
    float lo = INFINITY, hi = -INFINITY;
    bool nan = false;
    for (int j0 = 0; j0 < n; j0 += 32 * kLoads) {
      float f[kLoads];
#pragma unroll
      for (int u = 0; u < kLoads; ++u) {
        const int j = j0 + 32 * u + lane;
        f[u] = j < n ? srow[j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kLoads; ++u) {
        const int j = j0 + 32 * u + lane;
        if (j < n) {
          const float x = f[u] + 0.0f;
          nan |= x != x;
          lo = fminf(lo, x);
          hi = fmaxf(hi, x);
          keys[j] = order_key(x);
        }
      }
    }
    if (__any_sync(0xffffffffu, nan)) {
      if (lane == 0) atomicOr(err, kErrBadIndex);
      continue;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    __syncwarp();

    // threshold: the k-th largest key
    uint32_t thr;
    const float range = __fsub_rn(hi, lo);
    const float inv = range > 0.f ? __fdiv_rn(float(kBins), range) : 0.f;
    if (range > 0.f && range < INFINITY && inv < INFINITY) {   // finite, non-degenerate bins
      for (int b = lane; b < kBins; b += 32) hist[b] = 0;
      __syncwarp();
      for (int j = lane; j < n; j += 32) atomicAdd(&hist[value_bin(keys[j], lo, inv)], 1);
      __syncwarp();
      int above;
      const int bin = find_bin(hist, kBins, k, lane, &above);
      const int c = hist[bin];
      const int need = k - above;
      __syncwarp();   // hist is reused below
      if (c <= kSmall) {
        // the bin's candidates, then the one whose rank among them brackets need
        uint32_t* cand = reinterpret_cast<uint32_t*>(hist);
        int base = 0;
        for (int j0 = 0; j0 < n; j0 += 32) {
          const int j = j0 + lane;
          const bool in = j < n && value_bin(keys[j], lo, inv) == bin;
          const uint32_t bal = __ballot_sync(0xffffffffu, in);
          if (in) cand[base + __popc(bal & lanes_below(lane))] = keys[j];
          base += __popc(bal);
        }
        __syncwarp();
        bool found = false;
        uint32_t mine = 0;
        for (int ci = lane; ci < c; ci += 32) {
          const uint32_t v = cand[ci];
          int gt = 0, ge = 0;
          for (int m = 0; m < c; ++m) {
            const uint32_t w = cand[m];
            gt += w > v ? 1 : 0;
            ge += w >= v ? 1 : 0;
          }
          if (gt < need && need <= ge) {
            found = true;
            mine = v;
          }
        }
        const uint32_t who = __ballot_sync(0xffffffffu, found);
        thr = __shfl_sync(0xffffffffu, mine, __ffs(who) - 1);   // equal keys agree
      } else {
        thr = radix_select(keys, n, need, hist, lane,
                           [&](uint32_t key) { return value_bin(key, lo, inv) == bin; });
      }
    } else {   // all scores equal, an infinite one, or a denormal range: select over the keys directly
      thr = radix_select(keys, n, k, hist, lane, [](uint32_t) { return true; });
    }

    // kept indices, ascending: keys above thr, then the lowest-indexed equal ones
    int n_gt = 0;
    for (int j = lane; j < n; j += 32) n_gt += keys[j] > thr ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
    const int take_eq = k - n_gt;
    int base_eq = 0, base_out = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < n ? keys[j] : 0u;
      const bool is_eq = j < n && key == thr;
      const bool is_gt = j < n && key > thr;
      const uint32_t eq = __ballot_sync(0xffffffffu, is_eq);
      const int eq_rank = base_eq + __popc(eq & lanes_below(lane));
      const bool take = is_gt || (is_eq && eq_rank < take_eq);
      const uint32_t tk = __ballot_sync(0xffffffffu, take);
      if (take) out[base_out + __popc(tk & lanes_below(lane))] = j;
      base_eq += __popc(eq);
      base_out += __popc(tk);
    }
    __syncwarp();   // keys and hist are rewritten for the next row
  }
}

cudaError_t launch(const vsa_plan* p, const Geometry& g, const float* scores, int32_t* idx, cudaStream_t s,
                   bool ref) {
  const int64_t rows = int64_t(g.B) * g.Hh * g.ntv_max;
  if (rows == 0) return cudaSuccess;
  const int cols = ref ? g.n_ref : g.ntv_max;
  const int key_stride = (cols + 3) & ~3;
  int max_smem = 0;
  cudaError_t e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, p->device);
  if (e != cudaSuccess) return e;
  int warps = kMaxWarps;
  size_t smem = 0;
  for (; warps >= 1; warps >>= 1) {
    smem = size_t(warps) * (key_stride + kBins) * sizeof(uint32_t);
    if (smem <= size_t(max_smem)) break;
  }
  if (warps < 1) return cudaErrorInvalidValue;   // a row does not fit shared memory
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_kernel, warps * 32, smem);
  if (e != cudaSuccess) return e;
  const int64_t want = (rows + warps - 1) / warps;
  const int64_t full = int64_t(p->num_sms) * (per_sm > 0 ? per_sm : 1);
  const unsigned grid = unsigned(want < full ? want : full);
  topk_kernel<<<grid, warps * 32, smem, s>>>(g, scores, idx, p->d_state, ref, key_stride);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk(const vsa_plan* p, const float* scores, int32_t* idx, cudaStream_t s, const int32_t* k) {
  Geometry g = p->geo;   // by value: this call's k per head
  for (int h = 0; h < g.Hh; ++h) g.k[h] = k[h];
  return launch(p, g, scores, idx, s, false);
}

cudaError_t launch_topk_ref(const vsa_plan* p, const float* scores_ref, int32_t* idx_ref, cudaStream_t s) {
  return launch(p, p->geo, scores_ref, idx_ref, s, true);
}

}  // namespace vsa
