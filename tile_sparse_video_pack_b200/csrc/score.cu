// a2-a4: tile pooling, projection and tile-pair scores.
//
// Pooling (one warp per tile and tensor, fp32 sums over the tile's valid
// tokens): the mean for the VSA gate score (Ref2VA VSA README: the gating
// projection to_gate_compress picks the tiles), or the TripPool descriptor
// avg, max, min (BSAI VedaSparse README, "Core Technology: TripPool";
// "Implementation": _tripool, eq. 5). Projection and scores are fp32 batched
// GEMMs: q_hat = pooled(Q) W, k_hat = pooled(K) W, S = q_hat k_hat^T / sqrt(p)
// ("Scorer Modes": per-head projections, eq. 6).
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

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

// C[z] (+)= alpha * A[z] * op(B[z]); z = b * heads + h; 128 x 128 tiles, 8 x 8 per thread.
// A: [M][K] row-major (lda). B: [K][N] (ldb) or, with BT, [N][K] (ldb).
// M = m_fixed if > 0 else ntv[h]; N = n_fixed if > 0 else ntv[h]. K % 8 == 0, rows 16-byte aligned.
template <bool BT>
__global__ void __launch_bounds__(256) sgemm_kernel(Geometry g, const float* __restrict__ A, int64_t sA, int lda,
                                                    const float* __restrict__ Bm, int64_t sBz, int64_t sBh,
                                                    int ldb, float* __restrict__ C, int64_t sC, int ldc, int K,
                                                    int n_fixed, float alpha, int m_fixed = 0) {
  __shared__ __align__(16) float As[8][128];
  __shared__ __align__(16) float Bs[8][128];
  const int z = blockIdx.z;
  const int h = z % g.Hh;
  const int M = m_fixed > 0 ? m_fixed : g.ntv[h];
  const int N = n_fixed > 0 ? n_fixed : g.ntv[h];
  const int m0 = blockIdx.y * 128, n0 = blockIdx.x * 128;
  if (m0 >= M || n0 >= N) return;
  A += z * sA;
  Bm += z * sBz + h * sBh;
  C += z * sC;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += 8) {
    {  // A tile: 128 rows x 8 k, one float4 per thread, stored k-major
      const int r = tid >> 1, kq = (tid & 1) * 4;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m0 + r < M) a = *reinterpret_cast<const float4*>(A + int64_t(m0 + r) * lda + k0 + kq);
      As[kq + 0][r] = a.x;
      As[kq + 1][r] = a.y;
      As[kq + 2][r] = a.z;
      As[kq + 3][r] = a.w;
    }
    if (BT) {  // B rows are n: 128 n x 8 k
      const int r = tid >> 1, kq = (tid & 1) * 4;
      float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
      if (n0 + r < N) b = *reinterpret_cast<const float4*>(Bm + int64_t(n0 + r) * ldb + k0 + kq);
      Bs[kq + 0][r] = b.x;
      Bs[kq + 1][r] = b.y;
      Bs[kq + 2][r] = b.z;
      Bs[kq + 3][r] = b.w;
    } else {  // B rows are k: 8 k x 128 n
      const int kr = tid >> 5, c = (tid & 31) * 4;
      float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
      if (n0 + c < N) b = *reinterpret_cast<const float4*>(Bm + int64_t(k0 + kr) * ldb + n0 + c);
      *reinterpret_cast<float4*>(&Bs[kr][c]) = b;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      float a[8], b[8];
      *reinterpret_cast<float4*>(a) = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      *reinterpret_cast<float4*>(a + 4) = *reinterpret_cast<const float4*>(&As[kk][64 + ty * 4]);
      *reinterpret_cast<float4*>(b) = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      *reinterpret_cast<float4*>(b + 4) = *reinterpret_cast<const float4*>(&Bs[kk][64 + tx * 4]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (n < N) C[int64_t(m) * ldc + n] = alpha * acc[i][j];
    }
  }
}

}  // namespace

int64_t score_workspace_bytes(const Geometry& g, int mode, int p) { return score_layout(g, mode, p).total; }

void score_pooled_ptrs(const vsa_plan* pl, void* workspace, float** pooled_q, float** pooled_k) {
  const ScoreLayout L = score_layout(pl->geo, pl->desc.score_mode, pl->desc.proj_dim);
  char* ws = static_cast<char*>(workspace);
  *pooled_q = reinterpret_cast<float*>(ws + L.off_pq);
  *pooled_k = reinterpret_cast<float*>(ws + L.off_pk);
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
  dim3 gp((p + 127) / 128, (g.ntv_max + 127) / 128, Z);
  sgemm_kernel<false><<<gp, 256, 0, s>>>(g, pq, int64_t(g.ntv_max) * L.kd, L.kd, proj_q, 0, sW, p, hq,
                                         int64_t(g.ntv_max) * p, p, L.kd, p, 1.0f);
  sgemm_kernel<false><<<gp, 256, 0, s>>>(g, pk, int64_t(g.ntv_max) * L.kd, L.kd, proj_k, 0, sW, p, hk,
                                         int64_t(g.ntv_max) * p, p, L.kd, p, 1.0f);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  // scores: q_hat k_hat^T / sqrt(p)
  dim3 gs((g.ntv_max + 127) / 128, (g.ntv_max + 127) / 128, Z);
  sgemm_kernel<true><<<gs, 256, 0, s>>>(g, hq, int64_t(g.ntv_max) * p, p, hk, int64_t(g.ntv_max) * p, 0, p, scores,
                                        int64_t(g.ntv_max) * g.ntv_max, g.ntv_max, p, 0, 1.0f / sqrtf(float(p)));
  return cudaGetLastError();
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
  dim3 gp((p + 127) / 128, (g.n_ref + 127) / 128, Z);
  sgemm_kernel<false><<<gp, 256, 0, s>>>(g, pr, int64_t(g.n_ref) * L.kd, L.kd, proj_k, 0, sW, p, hr,
                                         int64_t(g.n_ref) * p, p, L.kd, p, 1.0f, g.n_ref);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 gs((g.n_ref + 127) / 128, (g.ntv_max + 127) / 128, Z);
  sgemm_kernel<true><<<gs, 256, 0, s>>>(g, hq, int64_t(g.ntv_max) * p, p, hr, int64_t(g.n_ref) * p, 0, p, scores_ref,
                                        int64_t(g.ntv_max) * g.n_ref, g.n_ref, p, g.n_ref, 1.0f / sqrtf(float(p)));
  return cudaGetLastError();
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
