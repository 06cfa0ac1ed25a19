// a5: per-head top-k tile selection -- one warp per row.
//
// For every (b, h, video query tile i): keep the k video key tiles with the
// largest scores, ties to the lower tile index, written ascending (Veda page,
// "Что делает Veda": head-aware top-k forms the tile mask; Ref2VA VSA README
// item 2: only video key tiles are pruned).
//
// One warp per row, several rows per CTA, no block-wide barriers. The row's
// scores become uint32 keys whose unsigned order is the float order (-0 folded
// onto +0) and stay in the warp's slice of shared memory, four to a lane per
// 16-byte access. A histogram of 256 value bins between the row's minimum and
// maximum (a monotone map in fp32: bin = (f - min) * (256 / (max - min)),
// truncated) finds the bin that holds the k-th largest score; each key's bin
// is kept as a byte, so the bin's candidates are gathered without recomputing
// it, and the exact threshold key comes from those few candidates by counting
// -- or, when the bin holds more than 64 (many equal scores, or one outlier
// that makes the bins coarse), from an 8-bit radix select restricted to the
// bin. The count above the threshold follows from the histogram and the
// candidates, so one more pass writes the kept indices in ascending order:
// every key above the threshold and the lowest-indexed keys equal to it (their
// ranks are counted only when equal keys straddle the cut).
#include <cuda_runtime.h>

#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int kBins = 256;        // value bins of the first pass (a byte per key)
constexpr int kSmall = 64;        // candidates resolved by counting
static_assert(kSmall < kBins - 1, "the candidates and their slot counter share the histogram's words");
constexpr int kMaxWarps = 4;      // rows (warps) per CTA

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

__device__ __forceinline__ int warp_excl_scan(int v, int lane, int* total) {
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  *total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

// Shared memory of one warp: keys [key_stride] | bin bytes [key_stride / 4 words] | histogram [kBins].
// key_stride is a multiple of 128, so every lane's 16-byte chunk of keys is in bounds.
__host__ __device__ constexpr int warp_words(int key_stride) { return key_stride + key_stride / 4 + kBins; }

// ref = false: video key tiles (columns ntv[h], k[h]); ref = true: the
// reference tiles of the R2VA budget variant (columns n_ref, k_ref[h]).
__global__ void __launch_bounds__(kMaxWarps * 32) topk_kernel(Geometry g, const float* __restrict__ scores,
                                                              int32_t* __restrict__ idx,
                                                              uint32_t* __restrict__ err, bool ref,
                                                              int key_stride) {
  extern __shared__ __align__(16) uint32_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  uint32_t* keys = smem + size_t(warp) * warp_words(key_stride);
  uint8_t* bins = reinterpret_cast<uint8_t*>(keys + key_stride);
  int* hist = reinterpret_cast<int*>(keys + key_stride + key_stride / 4);
  const int64_t rows = int64_t(g.B) * g.Hh * g.ntv_max;
  const int row_stride = ref ? g.n_ref : g.ntv_max;

  for (int64_t row = int64_t(blockIdx.x) * warps + warp; row < rows; row += int64_t(gridDim.x) * warps) {
    const int i = int(row % g.ntv_max);
    const int bh = int(row / g.ntv_max);
    const int h = bh % g.Hh;
    if (i >= g.ntv[h]) continue;                  // no such query tile in this head (warp-uniform)
    const int n = ref ? g.n_ref : g.ntv[h];       // columns
    const int k = ref ? g.k_ref[h] : g.k[h];
    const float* srow = scores + row * row_stride;
    int32_t* out = idx + row * (ref ? g.k_ref_max : g.k_max);
    if (n < 1 || k < 1 || k > n) {               // the plan rules this out; never index past the row
      if (lane == 0) atomicOr(err, kErrBadIndex);
      continue;
    }
    const int chunks = (n + 127) / 128;           // 128 keys: four per lane

    // keys, range, NaN check. Keys past n are 0 (below every real key) and never counted.
    float lo = INFINITY, hi = -INFINITY;
    bool nan = false;
    const bool vec = (row_stride & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
    for (int c0 = 0; c0 < chunks; c0 += 4) {
      float4 f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {              // up to four 16-byte loads in flight per lane
        const int j = 4 * ((c0 + u) * 32 + lane);
        if (vec && j + 3 < n) {
          f[u] = *reinterpret_cast<const float4*>(srow + j);
        } else {
          f[u].x = j < n ? srow[j] : 0.f;
          f[u].y = j + 1 < n ? srow[j + 1] : 0.f;
          f[u].z = j + 2 < n ? srow[j + 2] : 0.f;
          f[u].w = j + 3 < n ? srow[j + 3] : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = 4 * ((c0 + u) * 32 + lane);
        if (c0 + u < chunks) {
          const float x[4] = {f[u].x + 0.0f, f[u].y + 0.0f, f[u].z + 0.0f, f[u].w + 0.0f};
          uint32_t kk[4];
          if (j + 3 < n) {                          // four real scores: no per-key checks
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              nan |= x[t] != x[t];
              lo = fminf(lo, x[t]);
              hi = fmaxf(hi, x[t]);
              kk[t] = order_key(x[t]);
            }
          } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const bool in = j + t < n;
              nan |= in && x[t] != x[t];
              if (in) {
                lo = fminf(lo, x[t]);
                hi = fmaxf(hi, x[t]);
              }
              kk[t] = in ? order_key(x[t]) : 0u;
            }
          }
          *reinterpret_cast<uint4*>(keys + j) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
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

    // threshold: the k-th largest key; n_gt: keys above it
    uint32_t thr;
    int n_gt = -1;        // -1: not known from the histogram; counted below
    const float range = __fsub_rn(hi, lo);
    const float inv = range > 0.f ? __fdiv_rn(float(kBins), range) : 0.f;
    if (range > 0.f && range < INFINITY && inv < INFINITY) {   // finite, non-degenerate bins
      for (int b = lane; b < kBins; b += 32) hist[b] = 0;
      __syncwarp();
      for (int c = 0; c < chunks; ++c) {
        const int j = 4 * (c * 32 + lane);
        const uint4 kv = *reinterpret_cast<const uint4*>(keys + j);
        const uint32_t kk[4] = {kv.x, kv.y, kv.z, kv.w};
        uint32_t code = 0;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          // padding keys (0, past n) decode to NaN, whose bin is clamped to 0; they are taken off below
          const int b = max(value_bin(kk[t], lo, inv), 0);
          atomicAdd(&hist[b], 1);
          code |= uint32_t(b) << (8 * t);
        }
        reinterpret_cast<uint32_t*>(bins)[c * 32 + lane] = code;
      }
      __syncwarp();
      if (lane == 0) hist[0] -= chunks * 128 - n;
      __syncwarp();
      int above;
      const int bin = find_bin(hist, kBins, k, lane, &above);
      const int cnt = hist[bin];
      const int need = k - above;
      __syncwarp();   // hist is reused below
      if (cnt <= kSmall) {
        // the bin's candidates (any order), then the one whose rank among them brackets need
        uint32_t* cand = reinterpret_cast<uint32_t*>(hist);
        int* n_cand = hist + (kBins - 1);   // a slot counter past the (at most kSmall) candidates
        if (lane == 0) *n_cand = 0;
        __syncwarp();
        for (int c = 0; c < chunks; ++c) {
          const int j = 4 * (c * 32 + lane);
          const uint32_t code = reinterpret_cast<const uint32_t*>(bins)[c * 32 + lane];
#pragma unroll
          for (int t = 0; t < 4; ++t)
            if (int((code >> (8 * t)) & 255u) == bin && j + t < n) cand[atomicAdd(n_cand, 1)] = keys[j + t];
        }
        __syncwarp();
        bool found = false;
        uint32_t mine = 0;
        int mine_gt = 0;
        for (int ci = lane; ci < cnt; ci += 32) {
          const uint32_t v = cand[ci];
          int gt = 0, ge = 0;
          for (int m = 0; m < cnt; ++m) {
            const uint32_t w = cand[m];
            gt += w > v ? 1 : 0;
            ge += w >= v ? 1 : 0;
          }
          if (gt < need && need <= ge) {
            found = true;
            mine = v;
            mine_gt = gt;
          }
        }
        const uint32_t who = __ballot_sync(0xffffffffu, found);
        const int src = __ffs(who) - 1;   // equal keys agree
        thr = __shfl_sync(0xffffffffu, mine, src);
        n_gt = above + __shfl_sync(0xffffffffu, mine_gt, src);   // bins above, and the bin's keys above thr
      } else {
        thr = radix_select(keys, n, need, hist, lane,
                           [&](uint32_t key) { return value_bin(key, lo, inv) == bin; });
      }
    } else {   // all scores equal, an infinite one, or a denormal range: select over the keys directly
      thr = radix_select(keys, n, k, hist, lane, [](uint32_t) { return true; });
    }
    __syncwarp();
    if (n_gt < 0) {
      n_gt = 0;
      for (int j = lane; j < n; j += 32) n_gt += keys[j] > thr ? 1 : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
    }
    const int take_eq = k - n_gt;   // >= 1: thr itself is among the k largest

    // kept indices, ascending (lane-major within a chunk, then the lane's four)
    int base_eq = 0, base_out = 0;
    for (int c = 0; c < chunks; ++c) {
      const int j = 4 * (c * 32 + lane);
      const uint4 kv = *reinterpret_cast<const uint4*>(keys + j);
      const uint32_t kk[4] = {kv.x, kv.y, kv.z, kv.w};
      uint32_t gt4 = 0, eq4 = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        // padding keys are 0, below every real key, so neither above nor equal to thr
        gt4 |= kk[t] > thr ? (1u << t) : 0u;
        eq4 |= kk[t] == thr ? (1u << t) : 0u;
      }
      uint32_t take4 = gt4;
      if (__any_sync(0xffffffffu, eq4 != 0)) {
        // equal keys in this chunk: the lowest-indexed take_eq of all of them are kept
        int n_eq;
        const int r_eq = base_eq + warp_excl_scan(__popc(eq4), lane, &n_eq);
        int r = r_eq;
#pragma unroll
        for (int t = 0; t < 4; ++t)
          if (eq4 & (1u << t)) {
            if (r < take_eq) take4 |= 1u << t;
            ++r;
          }
        base_eq += n_eq;
      }
      // output slots: this lane's count (0..4) as three bit planes of ballots, no shuffle chain
      const uint32_t nt = __popc(take4);
      const uint32_t b0 = __ballot_sync(0xffffffffu, nt & 1u), b1 = __ballot_sync(0xffffffffu, nt & 2u),
                     b2 = __ballot_sync(0xffffffffu, nt & 4u);
      const uint32_t below = (1u << lane) - 1u;
      int pos = base_out + __popc(b0 & below) + 2 * __popc(b1 & below) + 4 * __popc(b2 & below);
      const int n_take = __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2);
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (take4 & (1u << t)) out[pos++] = j + t;
      base_out += n_take;
    }
    __syncwarp();   // keys, bins and hist are rewritten for the next row
  }
}

cudaError_t launch(const vsa_plan* p, const Geometry& g, const float* scores, int32_t* idx, cudaStream_t s,
                   bool ref) {
  const int64_t rows = int64_t(g.B) * g.Hh * g.ntv_max;
  if (rows == 0) return cudaSuccess;
  const int cols = ref ? g.n_ref : g.ntv_max;
  const int key_stride = (cols + 127) & ~127;
  int max_smem = 0;
  cudaError_t e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, p->device);
  if (e != cudaSuccess) return e;
  int warps = kMaxWarps;
  size_t smem = 0;
  for (; warps >= 1; warps >>= 1) {
    smem = size_t(warps) * warp_words(key_stride) * sizeof(uint32_t);
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
