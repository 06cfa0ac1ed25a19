// a2-a4: tile pooling, projection and tile-pair scores.
//
// Pooling (one warp per tile and tensor, fp32 sums over the tile's valid
// tokens): the mean for the VSA gate score (Ref2VA VSA README: the gating
// projection to_gate_compress picks the tiles), or the TripPool descriptor
// avg, max, min (BSAI VedaSparse README, "Core Technology: TripPool";
// "Implementation": _tripool, eq. 5). Projections are fp32 batched GEMMs
// (q_hat = pooled(Q) W, k_hat = pooled(K) W); the tile-score GEMM
// S = q_hat k_hat^T / sqrt(p) runs on the tensor cores as three-pass TF32
// ("Scorer Modes": per-head projections, eq. 6).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "tc_sm100.h"
#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

struct ScoreLayout {
  int kd;                 // pooled width: d (mean) or 3d (TripPool)
  int p;                  // projected width
  int64_t pooled_elems;   // per tensor: B*heads*ntv_max*kd
  int64_t proj_elems;     // per tensor: B*heads*ntv_max*p
  int64_t off_pq, off_pk, off_hq, off_hk;
  int64_t off_pr, off_hr;  // reference tiles (R2VA budgets): pooled and projected K, [B*heads*n_ref][..]
  int64_t total;
};

ScoreLayout score_layout(const Geometry& g, int mode, int p) {
  ScoreLayout L;
  L.kd = mode == VSA_SCORE_TRIPPOOL ? 3 * g.d : g.d;
  L.p = p;
  const int64_t rows = int64_t(g.B) * g.Hh * g.ntv_max;
  L.pooled_elems = rows * L.kd;
  L.proj_elems = rows * p;
  L.off_pq = 0;
  L.off_pk = L.off_pq + align256(L.pooled_elems * 4);
  L.off_hq = L.off_pk + align256(L.pooled_elems * 4);
  L.off_hk = L.off_hq + align256(L.proj_elems * 4);
  const int64_t ref_rows = int64_t(g.B) * g.Hh * g.n_ref;
  L.off_pr = L.off_hk + align256(L.proj_elems * 4);
  L.off_hr = L.off_pr + align256(ref_rows * L.kd * 4);
  L.total = L.off_hr + align256(ref_rows * p * 4);
  return L;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// One warp per (b, h, video tile, tensor). Lane l owns channels [CH*l, CH*l+CH).
template <int D, bool TRIP>
__global__ void __launch_bounds__(256) pool_kernel(Geometry g, const uint16_t* __restrict__ qp,
                                                   const uint16_t* __restrict__ kp,
                                                   const int32_t* __restrict__ counts, float* __restrict__ pq,
                                                   float* __restrict__ pk) {
  constexpr int CH = D / 32;  // 4 (d=128) or 2 (d=64)
  constexpr int KD = TRIP ? 3 * D : D;
  const int warps_per_block = blockDim.x >> 5;
  const int64_t task = int64_t(blockIdx.x) * warps_per_block + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t n_tasks = int64_t(g.B) * g.Hh * g.ntv_max * 2;
  if (task >= n_tasks) return;
  const int which = int(task & 1);
  const int64_t t2 = task >> 1;
  const int v = int(t2 % g.ntv_max);
  const int bh = int(t2 / g.ntv_max);
  const int h = bh % g.Hh;
  if (v >= g.ntv[h]) return;
  const int n = g.n_pre_tiles + v;
  const int cnt = counts[h * g.nt_max + n];
  const uint16_t* src = (which ? kp : qp) + ((int64_t(bh) * g.nt_max + n) * VSA_TILE) * D + CH * lane;
  float sum[CH], mx[CH], mn[CH];
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    sum[c] = 0.f;
    mx[c] = -INFINITY;
    mn[c] = INFINITY;
  }
  for (int s = 0; s < cnt; ++s) {
    float x[CH];
    if (CH == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(src + int64_t(s) * D);
      x[0] = bf16_lo(u.x);
      x[1] = bf16_hi(u.x);
      x[2] = bf16_lo(u.y);
      x[3] = bf16_hi(u.y);
    } else {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(src + int64_t(s) * D);
      x[0] = bf16_lo(u);
      x[1] = bf16_hi(u);
    }
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      sum[c] += x[c];
      if (TRIP) {
        mx[c] = fmaxf(mx[c], x[c]);
        mn[c] = fminf(mn[c], x[c]);
      }
    }
  }
  float* dst = (which ? pk : pq) + t2 * KD + CH * lane;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    dst[c] = sum[c] / float(cnt);
    if (TRIP) {
      dst[D + c] = mx[c];
      dst[2 * D + c] = mn[c];
    }
  }
}

// Pooled K of the reference tiles (R2VA budgets): one warp per (b, h,
// reference tile); the pooling of pool_kernel, over packed tile ref_tiles[r].
template <int D, bool TRIP>
__global__ void __launch_bounds__(256) pool_ref_kernel(Geometry g, const uint16_t* __restrict__ kp,
                                                       const int32_t* __restrict__ counts,
                                                       const int32_t* __restrict__ ref_tiles, float* __restrict__ pr) {
  constexpr int CH = D / 32;
  constexpr int KD = TRIP ? 3 * D : D;
  const int64_t task = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (task >= int64_t(g.B) * g.Hh * g.n_ref) return;
  const int r = int(task % g.n_ref);
  const int bh = int(task / g.n_ref);
  const int h = bh % g.Hh;
  const int n = ref_tiles[r];
  const int cnt = counts[h * g.nt_max + n];
  const uint16_t* src = kp + ((int64_t(bh) * g.nt_max + n) * VSA_TILE) * D + CH * lane;
  float sum[CH], mx[CH], mn[CH];
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    sum[c] = 0.f;
    mx[c] = -INFINITY;
    mn[c] = INFINITY;
  }
  for (int s = 0; s < cnt; ++s) {
    float x[CH];
    if (CH == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(src + int64_t(s) * D);
      x[0] = bf16_lo(u.x);
      x[1] = bf16_hi(u.x);
      x[2] = bf16_lo(u.y);
      x[3] = bf16_hi(u.y);
    } else {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(src + int64_t(s) * D);
      x[0] = bf16_lo(u);
      x[1] = bf16_hi(u);
    }
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      sum[c] += x[c];
      if (TRIP) {
        mx[c] = fmaxf(mx[c], x[c]);
        mn[c] = fminf(mn[c], x[c]);
      }
    }
  }
  float* dst = pr + task * KD + CH * lane;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    dst[c] = sum[c] / float(cnt);
    if (TRIP) {
      dst[D + c] = mx[c];
      dst[2 * D + c] = mn[c];
    }
  }
}

// The projections: C[z] = alpha * A[z] * B[h] (fp32 SIMT), for one or two problems per launch (the query
// and the key side share the weights' layout): blockIdx.z = problem * Z + z, z = b * heads + h.
// A: [M][K] row-major (lda, stride sA per z). B: [K][N] row-major (ldb, stride sBh per head; 0 when one
// matrix serves every head). M = m_fixed if > 0 else ntv[h]; N = n_fixed. K % 8 == 0, rows 16-byte aligned.
// Output tiles of 32 rows x 128 columns, 64 threads of 8 x 8 each: the problems are a few thousand rows of
// K = 128 or 384, so small tiles keep every SM busy to the end (128-row tiles left one wave of 336 CTAs
// with a nearly empty second). Shared memory is double buffered: the next k slice of B streams in by
// cp.async and the next slice of A is held in registers while this one is used, one barrier per slice.
// Each output is one fp32 FMA chain over k in ascending order.
struct ProjProblem {
  const float* A;
  const float* B;
  float* C;
};
constexpr int kProjRows = 32;
constexpr int kProjThreads = 64;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(tc::smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

__global__ void __launch_bounds__(kProjThreads, 8) sgemm_kernel(Geometry g, ProjProblem p0, ProjProblem p1, int Z,
                                                                int64_t sA, int lda, int64_t sBh, int ldb,
                                                                int64_t sC, int ldc, int K, int N, float alpha,
                                                                int m_fixed) {
  constexpr int BM = kProjRows, NT = kProjThreads, BQ = 8 * 128 / 4 / NT;   // B chunks per thread per slice
  __shared__ __align__(16) float As[2][8][BM];
  __shared__ __align__(16) float Bs[2][8][128];
  const int zz = blockIdx.z;
  const ProjProblem pr = zz < Z ? p0 : p1;
  const int z = zz < Z ? zz : zz - Z;
  const int h = z % g.Hh;
  const int M = m_fixed > 0 ? m_fixed : g.ntv[h];
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * 128;
  if (m0 >= M || n0 >= N) return;
  const float* A = pr.A + z * sA;
  const float* Bm = pr.B + h * sBh;
  float* C = pr.C + z * sC;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;   // 16 column groups x 4 row groups
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  // one k slice: A 32 rows x 8 k (a float4 per thread, stored k-major), B 8 k x 128 n (BQ 16-byte chunks
  // per thread; columns past N are zero-filled)
  const int ar = tid >> 1, akq = (tid & 1) * 4;
  const bool a_in = m0 + ar < M;
  float4 ra;
  auto fetch_a = [&](int k0) {
    ra = a_in ? *reinterpret_cast<const float4*>(A + int64_t(m0 + ar) * lda + k0 + akq)
              : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto fetch_b = [&](int k0, int buf) {
#pragma unroll
    for (int q = 0; q < BQ; ++q) {
      const int e = tid + q * NT, kr = e >> 5, c = (e & 31) * 4;
      const bool in = n0 + c < N;
      cp_async16(&Bs[buf][kr][c], in ? Bm + int64_t(k0 + kr) * ldb + n0 + c : Bm, in);
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  };
  fetch_b(0, 0);
  fetch_a(0);
  for (int k0 = 0, buf = 0; k0 < K; k0 += 8, buf ^= 1) {
    As[buf][akq + 0][ar] = ra.x;
    As[buf][akq + 1][ar] = ra.y;
    As[buf][akq + 2][ar] = ra.z;
    As[buf][akq + 3][ar] = ra.w;
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();   // slice k0 complete in buf; every thread is past its reads of buf ^ 1
    if (k0 + 8 < K) {
      fetch_b(k0 + 8, buf ^ 1);
      fetch_a(k0 + 8);
    }
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      float a[8], b[8];
      *reinterpret_cast<float4*>(a) = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      *reinterpret_cast<float4*>(a + 4) = *reinterpret_cast<const float4*>(&As[buf][kk][BM / 2 + ty * 4]);
      *reinterpret_cast<float4*>(b) = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
      *reinterpret_cast<float4*>(b + 4) = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + (i < 4 ? ty * 4 + i : BM / 2 + ty * 4 + (i - 4));
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (n < N) C[int64_t(m) * ldc + n] = alpha * acc[i][j];
    }
  }
}

// C[z][m][n] = alpha * sum_k A[z][m][k] B[z][n][k] for m < M, n < N (rows and
// columns past them untouched). A, B fp32, K-major rows of K = kdim values.
// Each operand is split in shared memory into hi = tf32(x) (round to nearest)
// and lo = x - hi (exact in fp32), and the tensor core accumulates
// hi*hi + hi*lo + lo*hi in fp32 (the lo*lo term, ~2^-22 relative, is dropped),
// which keeps the scores near fp32 accuracy: the selection is checked against
// an fp64 oracle to 1e-5 of the row's score scale.
struct ScoreTcParams {
  float* C;
  int64_t a_rows_per_z, b_rows_per_z;   // row offsets of batch-head z in the A and B maps
  int64_t c_stride_z;                   // elements between the C matrices of consecutive z
  int32_t ldc;                          // row stride of C (elements)
  int32_t m_fixed, n_fixed;             // > 0: M / N; else the head's video tile count
  int32_t kdim;                         // K, a multiple of 4 (rows 16-byte aligned)
  float alpha;
  uint64_t wait_ns;
  uint32_t* err;
  int32_t heads;
  int32_t ntv[VSA_MAX_HEADS];
};

constexpr int kTcThreads = 128;
constexpr uint32_t kTcTileBytes = 128 * 128;   // 128 rows x 32 fp32 (one 128-byte swizzle row each)

__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// Bounded wait of every thread of the CTA on one phase of an mbarrier.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = tc::globaltimer();
  while (!tc::mbar_try_wait(bar, parity))
    if (tc::globaltimer() - t0 > limit_ns) return false;
  return true;
}

__global__ void __launch_bounds__(kTcThreads) score_tc_kernel(const __grid_constant__ CUtensorMap ta,
                                                              const __grid_constant__ CUtensorMap tb,
                                                              const __grid_constant__ ScoreTcParams prm) {
  const int z = blockIdx.z;
  const int h = z % prm.heads;
  const int M = prm.m_fixed > 0 ? prm.m_fixed : prm.ntv[h];
  const int N = prm.n_fixed > 0 ? prm.n_fixed : prm.ntv[h];
  const int m0 = blockIdx.y * 128, n0 = blockIdx.x * 128;
  if (m0 >= M || n0 >= N) return;   // uniform over the CTA, before any barrier or TMEM use

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // [A hi | A lo | B hi | B lo], each 128 rows x 128 bytes in the 128-byte-swizzled K-major layout
  float* a_hi = reinterpret_cast<float*>(smem);
  float* a_lo = reinterpret_cast<float*>(smem + kTcTileBytes);
  float* b_hi = reinterpret_cast<float*>(smem + 2 * kTcTileBytes);
  float* b_lo = reinterpret_cast<float*>(smem + 3 * kTcTileBytes);
  __shared__ __align__(8) uint64_t bars[3];   // [0] chunk landed, [1] chunk's MMAs done, [2] drain
  __shared__ uint32_t tmem_base;
  const uint32_t sbase = tc::smem_u32(smem);
  const uint32_t bar_full = tc::smem_u32(&bars[0]), bar_mma = tc::smem_u32(&bars[1]);
  const uint32_t bar_drain = tc::smem_u32(&bars[2]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tc::mbar_init(bar_full, 1);
    tc::mbar_init(bar_mma, 1);
    tc::mbar_init(bar_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(tc::smem_u32(&tmem_base)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base;

  // instruction descriptor: kind::tf32 (A, B format 2), fp32 accumulator, both K-major, M = N = 128
  constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(128 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  const int chunks = (prm.kdim + 31) / 32;   // columns past kdim are read as zeros (outside the map)
  const int64_t arow = int64_t(z) * prm.a_rows_per_z + m0;
  const int64_t brow = int64_t(z) * prm.b_rows_per_z + n0;
  bool ok = true;
  int c = 0;
  for (; c < chunks && ok; ++c) {
    if (threadIdx.x == 0) {
      tc::mbar_expect_tx(bar_full, 2 * kTcTileBytes);
      tc::tma_load_2d(sbase, &ta, 32 * c, int(arow), bar_full);
      tc::tma_load_2d(sbase + 2 * kTcTileBytes, &tb, 32 * c, int(brow), bar_full);
    }
    ok = tc_wait(bar_full, c & 1, prm.wait_ns);
    if (__syncthreads_or(!ok)) {
      ok = false;
      tc_wait(bar_full, c & 1, tc::kTimeoutNs);   // let the copy land before shared memory is released
      break;
    }
    // split in place: hi = tf32(x), lo = x - hi; elementwise, so the swizzled layout is kept
    for (int i = threadIdx.x; i < 128 * 32; i += kTcThreads) {
      const float xa = a_hi[i], xb = b_hi[i];
      const float ha = __uint_as_float(tf32_rna(xa)), hb = __uint_as_float(tf32_rna(xb));
      a_hi[i] = ha;
      a_lo[i] = xa - ha;
      b_hi[i] = hb;
      b_lo[i] = xb - hb;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> tensor core
    __syncthreads();
    if (threadIdx.x == 0) {
      tc::tc_fence_after();
      const uint64_t dah = tc::sw128_desc(sbase, 16, 1024), dal = tc::sw128_desc(sbase + kTcTileBytes, 16, 1024);
      const uint64_t dbh = tc::sw128_desc(sbase + 2 * kTcTileBytes, 16, 1024);
      const uint64_t dbl = tc::sw128_desc(sbase + 3 * kTcTileBytes, 16, 1024);
#pragma unroll
      for (int pass = 0; pass < 3; ++pass) {
        const uint64_t da = pass == 2 ? dal : dah;
        const uint64_t db = pass == 1 ? dbl : dbh;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {   // 8 tf32 (32 bytes) of K per instruction
          const uint32_t off = (ks * 32) >> 4;
          asm volatile(
              "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\ntcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
              "l"(da + off), "l"(db + off), "r"(kIdesc), "r"((c | pass | ks) ? 1u : 0u)
              : "memory");
        }
      }
      tc::tc_commit(bar_mma);
    }
    // the chunk's MMAs must finish reading shared memory before the next chunk lands there
    ok = tc_wait(bar_mma, c & 1, prm.wait_ns);
    if (__syncthreads_or(!ok)) ok = false;
  }
  if (!ok) {
    // a wait ran past the limit: latch it, and let every MMA issued here finish before TMEM is freed
    if (threadIdx.x == 0) {
      atomicOr(prm.err, kErrTimeout);
      tc::tc_commit(bar_drain);
    }
    tc_wait(bar_drain, 0, tc::kTimeoutNs);
  } else {
    tc::tc_fence_after();
    // epilogue: warp w owns TMEM lanes (rows) 32w .. 32w+31; 32 columns at a time through a
    // padded shared-memory slab per warp (row stride 144 bytes), then row-contiguous stores
    float* slab = reinterpret_cast<float*>(smem) + warp * (32 * 36);
    const int row0 = m0 + 32 * warp;
    float* Cz = prm.C + int64_t(z) * prm.c_stride_z;
    const bool vec = (prm.ldc & 3) == 0 && (reinterpret_cast<uintptr_t>(prm.C) & 15) == 0 &&
                     (prm.c_stride_z & 3) == 0;
#pragma unroll 1
    for (int s = 0; s < 4; ++s) {
      uint32_t r[32];
      tc::tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + 32 * s, r);
      tc::tmem_wait_ld(r);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float4 v = make_float4(__uint_as_float(r[4 * q]) * prm.alpha, __uint_as_float(r[4 * q + 1]) * prm.alpha,
                               __uint_as_float(r[4 * q + 2]) * prm.alpha, __uint_as_float(r[4 * q + 3]) * prm.alpha);
        *reinterpret_cast<float4*>(slab + lane * 36 + 4 * q) = v;
      }
      __syncwarp();
      // lanes 8j .. 8j+7 write row (4i + j) of the slab: 8 x 16 bytes = the slab's 32 columns
      const int col = n0 + 32 * s + 4 * (lane & 7);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = 4 * i + (lane >> 3);
        const int m = row0 + rr;
        if (m < M) {
          const float4 v = *reinterpret_cast<const float4*>(slab + rr * 36 + 4 * (lane & 7));
          float* dst = Cz + int64_t(m) * prm.ldc + col;
          if (vec && col + 3 < N) {
            *reinterpret_cast<float4*>(dst) = v;
          } else {
            if (col < N) dst[0] = v.x;
            if (col + 1 < N) dst[1] = v.y;
            if (col + 2 < N) dst[2] = v.z;
            if (col + 3 < N) dst[3] = v.w;
          }
        }
      }
      __syncwarp();
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tmem));
}

// fp32 [rows, kdim] viewed as a 2D tensor; boxes of 32 columns (128 bytes) x 128 rows, 128-byte swizzle.
bool make_map_f32(CUtensorMap* m, const void* base, int64_t rows, int kdim) {
  tc::EncodeTiledFn enc = tc::get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cuuint64_t(kdim), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(kdim) * 4};
  cuuint32_t box[2] = {32, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int score_tc_smem_bytes() { return 1024 + 4 * int(kTcTileBytes); }

}  // namespace

int64_t score_workspace_bytes(const Geometry& g, int mode, int p) { return score_layout(g, mode, p).total; }

void score_pooled_ptrs(const vsa_plan* pl, void* workspace, float** pooled_q, float** pooled_k) {
  const ScoreLayout L = score_layout(pl->geo, pl->desc.score_mode, pl->desc.proj_dim);
  char* ws = static_cast<char*>(workspace);
  *pooled_q = reinterpret_cast<float*>(ws + L.off_pq);
  *pooled_k = reinterpret_cast<float*>(ws + L.off_pk);
}

// C[z] = alpha * A[z] B[z]^T on the tensor cores (score_tc_kernel): A rows a_rows_per_z per z,
// B rows b_rows_per_z per z, both [.., kdim] fp32; M, N as in ScoreTcParams.
cudaError_t launch_score_tc(const vsa_plan* pl, const float* A, int64_t a_rows_per_z, const float* B,
                            int64_t b_rows_per_z, int kdim, float* C, int64_t c_stride_z, int ldc, int m_fixed,
                            int n_fixed, int m_max, int n_max, float alpha, cudaStream_t s) {
  const Geometry& g = pl->geo;
  const int Z = g.B * g.Hh;
  CUtensorMap ta, tb;
  if (!make_map_f32(&ta, A, int64_t(Z) * a_rows_per_z, kdim) || !make_map_f32(&tb, B, int64_t(Z) * b_rows_per_z, kdim))
    return cudaErrorInvalidValue;
  ScoreTcParams prm;
  prm.C = C;
  prm.a_rows_per_z = a_rows_per_z;
  prm.b_rows_per_z = b_rows_per_z;
  prm.c_stride_z = c_stride_z;
  prm.ldc = ldc;
  prm.m_fixed = m_fixed;
  prm.n_fixed = n_fixed;
  prm.kdim = kdim;
  prm.alpha = alpha;
  prm.wait_ns = pl->wait_ns;
  prm.err = pl->d_state;
  prm.heads = g.Hh;
  for (int h = 0; h < VSA_MAX_HEADS; ++h) prm.ntv[h] = h < g.Hh ? g.ntv[h] : 0;
  const int smem = score_tc_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((n_max + 127) / 128, (m_max + 127) / 128, Z);
  score_tc_kernel<<<grid, kTcThreads, smem, s>>>(ta, tb, prm);
  return cudaGetLastError();
}

// a3-a4 from the pooled descriptors already in the workspace.
cudaError_t launch_project_score(const vsa_plan* pl, const float* proj_q, const float* proj_k, float* scores,
                                 void* workspace, cudaStream_t s) {
  const Geometry& g = pl->geo;
  const int mode = pl->desc.score_mode;
  const int p = pl->desc.proj_dim;
  const ScoreLayout L = score_layout(g, mode, p);
  char* ws = static_cast<char*>(workspace);
  float* pq = reinterpret_cast<float*>(ws + L.off_pq);
  float* pk = reinterpret_cast<float*>(ws + L.off_pk);
  float* hq = reinterpret_cast<float*>(ws + L.off_hq);
  float* hk = reinterpret_cast<float*>(ws + L.off_hk);
  const bool trip = mode == VSA_SCORE_TRIPPOOL;

  // projection: [ntv, kd] x [kd, p]; the gate is shared by all heads, TripPool weights are per head
  const int Z = g.B * g.Hh;
  const int64_t sW = trip ? int64_t(L.kd) * p : 0;
  dim3 gp((p + 127) / 128, (g.ntv_max + kProjRows - 1) / kProjRows, 2 * Z);
  sgemm_kernel<<<gp, kProjThreads, 0, s>>>(g, ProjProblem{pq, proj_q, hq}, ProjProblem{pk, proj_k, hk}, Z,
                                           int64_t(g.ntv_max) * L.kd, L.kd, sW, p, int64_t(g.ntv_max) * p, p,
                                           L.kd, p, 1.0f, 0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  // scores: q_hat k_hat^T / sqrt(p), on the tensor cores
  return launch_score_tc(pl, hq, g.ntv_max, hk, g.ntv_max, p, scores, int64_t(g.ntv_max) * g.ntv_max, g.ntv_max,
                         0, 0, g.ntv_max, g.ntv_max, 1.0f / sqrtf(float(p)), s);
}

cudaError_t launch_score(const vsa_plan* pl, const void* qp, const void* kp, const float* proj_q,
                         const float* proj_k, float* scores, void* workspace, cudaStream_t s) {
  const Geometry& g = pl->geo;
  const bool trip = pl->desc.score_mode == VSA_SCORE_TRIPPOOL;
  float *pq, *pk;
  score_pooled_ptrs(pl, workspace, &pq, &pk);
  const int64_t tasks = int64_t(g.B) * g.Hh * g.ntv_max * 2;
  const int blocks = int((tasks + 7) / 8);
  auto* q16 = static_cast<const uint16_t*>(qp);
  auto* k16 = static_cast<const uint16_t*>(kp);
  if (g.d == 128) {
    if (trip) pool_kernel<128, true><<<blocks, 256, 0, s>>>(g, q16, k16, pl->d_tile_count, pq, pk);
    else pool_kernel<128, false><<<blocks, 256, 0, s>>>(g, q16, k16, pl->d_tile_count, pq, pk);
  } else {
    if (trip) pool_kernel<64, true><<<blocks, 256, 0, s>>>(g, q16, k16, pl->d_tile_count, pq, pk);
    else pool_kernel<64, false><<<blocks, 256, 0, s>>>(g, q16, k16, pl->d_tile_count, pq, pk);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_project_score(pl, proj_q, proj_k, scores, workspace, s);
}

// R2VA budgets: scores of every video query tile against the reference tiles,
// from the projected pooled Q already in the workspace.
cudaError_t launch_ref_score(const vsa_plan* pl, const void* kp, const float* proj_k, float* scores_ref,
                             void* workspace, cudaStream_t s) {
  const Geometry& g = pl->geo;
  const int mode = pl->desc.score_mode;
  const int p = pl->desc.proj_dim;
  const ScoreLayout L = score_layout(g, mode, p);
  const bool trip = mode == VSA_SCORE_TRIPPOOL;
  char* ws = static_cast<char*>(workspace);
  const float* hq = reinterpret_cast<const float*>(ws + L.off_hq);
  float* pr = reinterpret_cast<float*>(ws + L.off_pr);
  float* hr = reinterpret_cast<float*>(ws + L.off_hr);
  const int64_t tasks = int64_t(g.B) * g.Hh * g.n_ref;
  const int blocks = int((tasks + 7) / 8);
  auto* k16 = static_cast<const uint16_t*>(kp);
  if (g.d == 128) {
    if (trip) pool_ref_kernel<128, true><<<blocks, 256, 0, s>>>(g, k16, pl->d_tile_count, pl->d_ref_tiles, pr);
    else pool_ref_kernel<128, false><<<blocks, 256, 0, s>>>(g, k16, pl->d_tile_count, pl->d_ref_tiles, pr);
  } else {
    if (trip) pool_ref_kernel<64, true><<<blocks, 256, 0, s>>>(g, k16, pl->d_tile_count, pl->d_ref_tiles, pr);
    else pool_ref_kernel<64, false><<<blocks, 256, 0, s>>>(g, k16, pl->d_tile_count, pl->d_ref_tiles, pr);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int Z = g.B * g.Hh;
  const int64_t sW = trip ? int64_t(L.kd) * p : 0;
  dim3 gp((p + 127) / 128, (g.n_ref + kProjRows - 1) / kProjRows, Z);
  const ProjProblem ref{pr, proj_k, hr};
  sgemm_kernel<<<gp, kProjThreads, 0, s>>>(g, ref, ref, Z, int64_t(g.n_ref) * L.kd, L.kd, sW, p,
                                           int64_t(g.n_ref) * p, p, L.kd, p, 1.0f, g.n_ref);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_score_tc(pl, hq, g.ntv_max, hr, g.n_ref, p, scores_ref, int64_t(g.ntv_max) * g.n_ref, g.n_ref, 0,
                         g.n_ref, g.ntv_max, g.n_ref, 1.0f / sqrtf(float(p)), s);
}

}  // namespace vsa

// ---------------------------------------------------------------------------
// vsa_tile_score_static: the same score stage with its scratch (pooled and
// projected tiles) in a fixed device array instead of a caller workspace.
//
// For callers that may not allocate device memory when they run the layer:
// code called under another framework's memory planner or fixed arena, a
// plugin that must not call cudaMalloc (it can synchronise the device or fail
// mid-step), or a latency-critical loop where allocation is not allowed.
// ---------------------------------------------------------------------------
namespace vsa {
namespace {

constexpr size_t kStaticScoreScratchBytes = size_t(32) << 20;   // 32 MiB

// Held by every GPU that loads this library until the process exits. Each
// call overwrites every element it later reads, so nothing needs clearing.
__device__ __align__(256) unsigned char g_static_score_scratch[kStaticScoreScratchBytes];

std::mutex g_static_scratch_mu;
void* g_static_scratch_addr[256] = {};   // device address per device ordinal

// Device address of the scratch array on the current device. The host-side
// symbol is only a stand-in: its device address comes from
// cudaGetSymbolAddress, called with that device current -- by every
// vsa_plan_create (so a plan made after a device reset gets the new module's
// address) and, if no plan has done so yet, by the first call here.
cudaError_t static_scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_addr[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_score_scratch);
    if (e != cudaSuccess) return e;
    g_static_scratch_addr[dev] = ptr;
  }
  *out = g_static_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t refresh_static_scratch_address(int dev) {
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_score_scratch);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  g_static_scratch_addr[dev] = ptr;
  return cudaSuccess;
}

}  // namespace vsa

extern "C" vsa_status vsa_tile_score_static(vsa_plan* p, const void* qp, const void* kp, const float* proj_q,
                                            const float* proj_k, float* scores, void* stream) {
  auto fail = [&](vsa_status st) {
    if (p) p->stats.errors++;
    return st;
  };
  if (!p || !qp || !kp || !proj_q || !proj_k || !scores) return fail(VSA_ERR_INVALID_ARG);
  const auto a16 = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) == 0; };
  if (!a16(qp) || !a16(kp) || !a16(proj_q) || !a16(proj_k) || !a16(scores)) return fail(VSA_ERR_INVALID_ARG);
  if (p->info.workspace_bytes > int64_t(vsa::kStaticScoreScratchBytes)) return fail(VSA_ERR_UNSUPPORTED);
  // R2VA plans continue with vsa_ref_score, which reads the projected pooled Q from the caller's
  // workspace; here that stays in the library's array, so such plans must use vsa_tile_score
  if (p->geo.n_ref > 0) return fail(VSA_ERR_UNSUPPORTED);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return fail(VSA_ERR_CUDA);
  }
  if (dev != p->device || dev < 0 || dev >= 256) return fail(VSA_ERR_INVALID_ARG);
  void* ws = nullptr;
  if (vsa::static_scratch_address(dev, &ws) != cudaSuccess) {
    cudaGetLastError();
    return fail(VSA_ERR_CUDA);
  }
  p->stats.calls_score++;
  if (vsa::launch_score(p, qp, kp, proj_q, proj_k, scores, ws, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(VSA_ERR_CUDA);
  return VSA_OK;
}
