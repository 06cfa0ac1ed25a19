// Teacher tile map and selection overlap (the Veda method's first stage and
// the tile-recall figure that measures a selection against it).
//
// What it computes (Veda news page, "Что делает Veda": full attention,
// max-pooled per tile pair, is the teacher distribution at tile level; BSAI
// VedaSparse README, "Core Technology": tile recall of a scorer against full
// attention): for head h, video query tile i and video key tile j,
//
//   T[i, j] = max over valid rows r of tile i and valid keys c of tile j of
//             exp(scale * q_r . k_c - lse_r),
//
// the largest full-attention weight a token of tile i puts on a token of tile
// j, where lse_r is row r's log-sum-exp over every key (prefix and video) --
// the lse output of a dense vsa_sparse_attn call (k = every video tile).
//
// How: one CTA per block of 128 query rows (two video query tiles of one
// (batch, head)). A producer thread loads the Q pair once and streams K tile
// pairs (2 stages) by TMA; one thread issues S = Q K^T for 128 keys at a time
// (tcgen05, both operands in shared memory, accumulator in one of two TMEM
// buffers); four warps (one per TMEM lane quarter, thread = row) read S,
// subtract the row's lse, take the max over each 64-key tile, and reduce it
// over the 32 rows of the warp and the two warps of a query tile.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "tc_sm100.h"
#include "vsa_internal.h"

namespace vsa {
namespace {

using namespace tc;

constexpr int kTThreads = 192;            // warp 0 producer, warp 1 MMA, warps 2-5 reduce
constexpr uint32_t kTTileBytes = 64 * 64 * 2;

template <int D>
struct TSmem {
  static constexpr uint32_t kPairBytes = (D / 64) * 128 * 128;   // 128 rows x D bf16, K-major
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + kPairBytes;                // two stages
  static constexpr uint32_t oBar = oK + 2 * kPairBytes;
  static constexpr uint32_t oMisc = oBar + 16 * 8;               // tmem base, abort flag
  static constexpr uint32_t oRed = oMisc + 16;   // [2 blocks][2 warps of a tile][2 key tiles][2 query tiles]
  static constexpr uint32_t oEnd = oRed + 2 * 2 * 2 * 2 * 4;
};

enum {
  T_QFULL = 0, T_KFULL0, T_KFULL1, T_KEMPTY0, T_KEMPTY1, T_SFULL0, T_SFULL1, T_SEMPTY0, T_SEMPTY1, T_RED0, T_RED1,
  T_DRAIN
};

struct TeacherParams {
  const float* lse;        // [B, heads, nt_max, 64] natural log, dense rows
  const int32_t* counts;   // [heads, nt_max] valid tokens per packed tile
  float* teacher;          // [B, heads, ntv_max, ntv_max]
  uint32_t* state;         // [0] error word
  int32_t heads, nt_max, ntv_max, n_pre, pairs_max;   // pairs_max = ceil(ntv_max / 2)
  float scale_log2;
  uint64_t wait_ns;        // bound of every mbarrier wait
  int32_t ntv[VSA_MAX_HEADS];
};

template <int D>
__global__ void __launch_bounds__(kTThreads, 1)
    teacher_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ TeacherParams prm) {
  using L = TSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + L::oBar + 8u * uint32_t(i); };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::oMisc);
  volatile uint32_t* abort_flag = misc + 1;
  float* red = reinterpret_cast<float*>(smem + L::oRed);
  uint32_t* gerr = prm.state;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // the block: query tiles (2p, 2p + 1) of video tiles of (batch, head) bh
  const int bh = int(blockIdx.x / prm.pairs_max);
  const int p = int(blockIdx.x % prm.pairs_max);
  const int h = bh % prm.heads;
  const int ntv = prm.ntv[h];
  const int va = 2 * p, vb = 2 * p + 1 < ntv ? 2 * p + 1 : -1;
  if (va >= ntv) return;                          // uniform over the CTA
  const int nblk = (ntv + 1) >> 1;                // key blocks of two video tiles
  const int row_base = bh * prm.nt_max + prm.n_pre;   // packed tile index of video tile 0

  if (threadIdx.x == 0) {
    mbar_init(bar(T_QFULL), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(T_KFULL0 + i), 1);
      mbar_init(bar(T_KEMPTY0 + i), 1);
      mbar_init(bar(T_SFULL0 + i), 1);
      mbar_init(bar(T_SEMPTY0 + i), 4);           // one arrival per reducing warp
      mbar_init(bar(T_RED0 + i), 4);
    }
    mbar_init(bar(T_DRAIN), 1);
    misc[1] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(sbase + L::oMisc));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];                  // S buffers at columns [0,128) and [128,256)

  if (warp == 0) {
    // ---------------------------------------------------------- producer ---
    if (lane == 0) {
      uint32_t issued = 0;
      bool ok = true;
      mbar_expect_tx(bar(T_QFULL), 2 * (D / 64) * kTTileBytes);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_2d(sbase + L::oQ + c * 16384, &tq, 64 * c, (row_base + va) * 64, bar(T_QFULL));
        tma_load_2d(sbase + L::oQ + c * 16384 + 8192, &tq, 64 * c, (row_base + (vb >= 0 ? vb : va)) * 64,
                    bar(T_QFULL));
      }
      for (int j = 0; j < nblk && ok; ++j) {
        const int st = j & 1;
        if (!(ok = wait_bar(bar(T_KEMPTY0 + st), ((j >> 1) & 1) ^ 1, abort_flag, gerr, prm.wait_ns))) break;
        const int ta = 2 * j, tb = 2 * j + 1 < ntv ? 2 * j + 1 : 2 * j;
        mbar_expect_tx(bar(T_KFULL0 + st), 2 * (D / 64) * kTTileBytes);
        const uint32_t sk = sbase + L::oK + st * L::kPairBytes;
        for (int c = 0; c < D / 64; ++c) {
          tma_load_2d(sk + c * 16384, &tk, 64 * c, (row_base + ta) * 64, bar(T_KFULL0 + st));
          tma_load_2d(sk + c * 16384 + 8192, &tk, 64 * c, (row_base + tb) * 64, bar(T_KFULL0 + st));
        }
        ++issued;
      }
      if (*abort_flag) {   // let this thread's copies land before shared memory is released
        drain_wait(bar(T_QFULL), 0);
        for (uint32_t j = issued >= 2 ? issued - 2 : 0; j < issued; ++j)
          drain_wait(bar(T_KFULL0 + int(j & 1)), (j >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ S MMA ---
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
      const uint64_t dq = sw128_desc(sbase + L::oQ, 16, 1024);
      const uint64_t dk0 = sw128_desc(sbase + L::oK, 16, 1024);
      bool ok = wait_bar(bar(T_QFULL), 0, abort_flag, gerr, prm.wait_ns);
      for (int j = 0; j < nblk && ok; ++j) {
        const int st = j & 1;                     // K stage and S buffer of block j
        if (!(ok = wait_bar(bar(T_KFULL0 + st), (j >> 1) & 1, abort_flag, gerr, prm.wait_ns))) break;
        if (!(ok = wait_bar(bar(T_SEMPTY0 + st), ((j >> 1) & 1) ^ 1, abort_flag, gerr, prm.wait_ns))) break;
        tc_fence_after();
        const uint64_t dk = dk0 + ((st * L::kPairBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {     // 16 channels per step
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          tc_mma(tmem + st * 128, dq + off, dk + off, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(T_SFULL0 + st));
        tc_commit(bar(T_KEMPTY0 + st));
      }
      tc_commit(bar(T_DRAIN));                    // nothing of ours may run when TMEM is freed
      drain_wait(bar(T_DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ reduce ---
    // Warp w reads TMEM lanes 32 (w mod 4) .. +31: row r of the block; rows
    // 0-63 belong to query tile va, rows 64-127 to vb.
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int qt = r >> 6;                        // 0: tile va, 1: tile vb
    const int vq = qt ? vb : va;
    const uint32_t lane_off = uint32_t(q4 * 32) << 16;
    const float* lse = prm.lse + (size_t(bh) * prm.nt_max + prm.n_pre + (vq >= 0 ? vq : va)) * 64;
    const int rows = vq >= 0 ? prm.counts[h * prm.nt_max + prm.n_pre + vq] : 0;
    // x = s * scale - lse in log2 units; rows past the tile's valid count give -inf
    const float off = (r & 63) < rows ? lse[r & 63] * 1.4426950408889634f : INFINITY;
    float* out_row = prm.teacher + (size_t(bh) * prm.ntv_max + (vq >= 0 ? vq : 0)) * prm.ntv_max;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int st = j & 1;
      ok = wait_bar(bar(T_SFULL0 + st), (j >> 1) & 1, abort_flag, gerr, prm.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      float mx[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {               // key tile 2j + t: columns [64 t, 64 t + 64)
        const int vk = 2 * j + t;
        const int keys = vk < ntv ? prm.counts[h * prm.nt_max + prm.n_pre + vk] : 0;
        uint32_t s0[32], s1[32];
        tmem_ld32(tmem + st * 128 + lane_off + 64 * t, s0);
        tmem_ld32(tmem + st * 128 + lane_off + 64 * t + 32, s1);
        tmem_wait_ld(s0);
        reg_fence(s1);
        float m = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          m = c < keys ? fmaxf(m, __uint_as_float(s0[c])) : m;
          m = c + 32 < keys ? fmaxf(m, __uint_as_float(s1[c])) : m;
        }
        mx[t] = m * prm.scale_log2 - off;        // -inf for an invalid row or an absent key tile
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T_SEMPTY0 + st));
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx[t] = fmaxf(mx[t], __shfl_xor_sync(0xffffffffu, mx[t], o));
      // the two warps of one query tile (lane quarters 2 qt and 2 qt + 1) meet in
      // shared memory (double buffered by block; a warp writes buffer st again
      // only after every warp has arrived for the next block, i.e. after the
      // reads of this one)
      const int half = q4 & 1;
      float* rb = red + st * 8;
      if (lane == 0) {
        rb[(half * 2 + 0) * 2 + qt] = mx[0];
        rb[(half * 2 + 1) * 2 + qt] = mx[1];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(T_RED0 + st));
      ok = wait_bar(bar(T_RED0 + st), (j >> 1) & 1, abort_flag, gerr, prm.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (lane == 0 && half == 0 && vq >= 0) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int vk = 2 * j + t;
          if (vk < ntv) out_row[vk] = exp2f(fmaxf(rb[t * 2 + qt], rb[(2 + t) * 2 + qt]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem));
}

// Per row of two [.., k] index tables: how many indices the rows share. Both
// rows are ascending (the top-k stage writes them so); one warp per row, each
// lane binary-searches its entries of row a in row b.
__global__ void __launch_bounds__(256) overlap_kernel(Geometry g, const int32_t* __restrict__ a,
                                                      const int32_t* __restrict__ b, int32_t* __restrict__ counts) {
  const int64_t rows = int64_t(g.B) * g.Hh * g.ntv_max;
  const int64_t row = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int h = int((row / g.ntv_max) % g.Hh);
  const int k = g.k[h];
  const int k_max = g.k_max;
  if (int(row % g.ntv_max) >= g.ntv[h]) {       // no such query tile in this head
    if (lane == 0) counts[row] = 0;
    return;
  }
  const int32_t* ra = a + row * k_max;
  const int32_t* rb = b + row * k_max;
  int hits = 0;
  for (int e = lane; e < k; e += 32) {
    const int x = ra[e];
    int lo = 0, hi = k;                           // first position in rb with value >= x
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (rb[mid] < x) lo = mid + 1;
      else hi = mid;
    }
    hits += lo < k && rb[lo] == x;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) hits += __shfl_xor_sync(0xffffffffu, hits, o);
  if (lane == 0) counts[row] = hits;
}

}  // namespace

int teacher_smem_bytes() {
  static_assert(TSmem<64>::oEnd <= TSmem<128>::oEnd, "the d=64 layout fits the d=128 allocation");
  return 1024 + int(TSmem<128>::oEnd);
}

cudaError_t launch_teacher(vsa_plan* p, const void* qp, const void* kp, const float* lse, float* teacher,
                           cudaStream_t s) {
  const Geometry& g = p->geo;
  const int64_t rows = int64_t(g.B) * g.Hh * g.nt_max * VSA_TILE;
  CUtensorMap tq, tk;
  if (!make_map(&tq, qp, rows, g.d) || !make_map(&tk, kp, rows, g.d)) return cudaErrorInvalidValue;
  TeacherParams prm;
  prm.lse = lse;
  prm.counts = p->d_tile_count;
  prm.teacher = teacher;
  prm.state = p->d_state;
  prm.heads = g.Hh;
  prm.nt_max = g.nt_max;
  prm.ntv_max = g.ntv_max;
  prm.n_pre = g.n_pre_tiles;
  prm.pairs_max = (g.ntv_max + 1) / 2;
  prm.scale_log2 = p->desc.softmax_scale * 1.4426950408889634f;
  prm.wait_ns = p->wait_ns;
  for (int h = 0; h < VSA_MAX_HEADS; ++h) prm.ntv[h] = h < g.Hh ? g.ntv[h] : 0;
  const int64_t grid = int64_t(g.B) * g.Hh * prm.pairs_max;
  const int smem = teacher_smem_bytes();
  cudaError_t e;
  if (g.d == 128) {
    e = cudaFuncSetAttribute(teacher_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    teacher_kernel<128><<<grid, kTThreads, smem, s>>>(tq, tk, prm);
  } else {
    e = cudaFuncSetAttribute(teacher_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    teacher_kernel<64><<<grid, kTThreads, smem, s>>>(tq, tk, prm);
  }
  return cudaGetLastError();
}

cudaError_t launch_overlap(vsa_plan* p, const int32_t* a, const int32_t* b, int32_t* counts, cudaStream_t s,
                           const int32_t* k) {
  Geometry g = p->geo;   // by value: this call's k per head
  for (int h = 0; h < g.Hh; ++h) g.k[h] = k[h];
  const int64_t rows = int64_t(g.B) * g.Hh * g.ntv_max;
  overlap_kernel<<<int((rows + 7) / 8), 256, 0, s>>>(g, a, b, counts);
  return cudaGetLastError();
}

}  // namespace vsa
