// a1 / a7: tile pack and unpack -- a 16-byte vectorised permutation of bf16 rows.
//
// Token-major [B, N, heads, d] <-> tile-major [B, heads, nt_max, 64, d].
// Tiling: Ref2VA VSA README ("two-tier attention layout": 4x4x4 video tiles,
// segment-pure prefix tiles) and BSAI VedaSparse README ("Core Technology:
// Head-Aware Tiling", per-head (pt, ph, pw) with product 64).
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <math.h>

#include "vsa_internal.h"

namespace vsa {
namespace {

// Token held by slot s of packed tile n of head h, or -1 for an unused slot.
// Prefix tiles: 64 consecutive tokens of one segment. Video tiles: the tile's
// tokens in (t, h, w) raster order over its actual extent (tiles cut by the
// grid's far edge hold fewer tokens, packed into the first slots).
__device__ __forceinline__ int src_token(const Geometry& g, int h, int n, int s) {
  if (n < g.n_pre_tiles) {
    int i = 0;
#pragma unroll 1
    while (i + 1 < g.n_seg && n >= g.seg_tile0[i + 1]) ++i;
    const int j = (n - g.seg_tile0[i]) * VSA_TILE + s;
    return j < g.seg_len[i] ? g.seg_tok0[i] + j : -1;
  }
  const int v = n - g.n_pre_tiles;
  if (v >= g.ntv[h]) return -1;
  const int nX = g.nX[h], nYX = g.nY[h] * nX;
  const int ti = v / nYX;
  const int r = v - ti * nYX;
  const int yi = r / nX;
  const int xi = r - yi * nX;
  const int t0 = ti * g.pt[h], y0 = yi * g.ph[h], x0 = xi * g.pw[h];
  const int et = min(g.pt[h], g.T - t0), eh = min(g.ph[h], g.H - y0), ew = min(g.pw[h], g.W - x0);
  if (s >= et * eh * ew) return -1;
  const int ehw = eh * ew;
  const int dt = s / ehw;
  const int r2 = s - dt * ehw;
  const int dy = r2 / ew;
  const int dx = r2 - dy * ew;
  return g.n_pre_tok + ((t0 + dt) * g.H + (y0 + dy)) * g.W + (x0 + dx);
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// One thread moves one 16-byte chunk of one packed row of each of up to three
// tensors (Q, K, V share the permutation).
template <int CPR>  // 16-byte chunks per row: d / 8
__global__ void __launch_bounds__(256) pack_kernel(Geometry g, const uint4* __restrict__ q,
                                                   const uint4* __restrict__ k,
                                                   const uint4* __restrict__ v, uint4* __restrict__ qp,
                                                   uint4* __restrict__ kp, uint4* __restrict__ vp) {
  const int64_t total = int64_t(g.B) * g.Hh * g.nt_max * VSA_TILE * CPR;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = i / CPR;
    const int c = int(i - row * CPR);
    const int s = int(row % VSA_TILE);
    const int64_t tile = row / VSA_TILE;
    const int n = int(tile % g.nt_max);
    const int bh = int(tile / g.nt_max);
    const int h = bh % g.Hh, b = bh / g.Hh;
    const int tok = src_token(g, h, n, s);
    const uint4 zero = make_uint4(0, 0, 0, 0);
    const int64_t src = tok >= 0 ? ((int64_t(b) * g.n_tokens + tok) * g.Hh + h) * CPR + c : 0;
    uint4 a = zero, bb = zero, cc = zero;
    if (tok >= 0) {
      if (q) a = ld_stream(q + src);
      if (k) bb = ld_stream(k + src);
      if (v) cc = ld_stream(v + src);
    }
    if (q) qp[i] = a;
    if (k) kp[i] = bb;
    if (v) vp[i] = cc;
  }
}

// Packed row of token `tok` for head h: (tile, slot) -> tile * 64 + slot, the
// inverse of src_token. Prefix tokens: their segment's tiles of 64 consecutive
// tokens. Video tokens (t, y, x): the tile (t / pt, y / ph, x / pw) and the
// token's (t, h, w) raster position inside that tile's actual extent.
__device__ __forceinline__ int packed_row(const Geometry& g, int h, int tok) {
  if (tok < g.n_pre_tok) {
    int i = 0;
#pragma unroll 1
    while (i + 1 < g.n_seg && tok >= g.seg_tok0[i + 1]) ++i;
    const int off = tok - g.seg_tok0[i];
    return (g.seg_tile0[i] + off / VSA_TILE) * VSA_TILE + off % VSA_TILE;
  }
  const int v = tok - g.n_pre_tok;
  const int hw = g.H * g.W;
  const int t = v / hw;
  const int r = v - t * hw;
  const int y = r / g.W;
  const int x = r - y * g.W;
  const int pt = g.pt[h], ph = g.ph[h], pw = g.pw[h];
  const int ti = t / pt, yi = y / ph, xi = x / pw;
  const int eh = min(ph, g.H - yi * ph), ew = min(pw, g.W - xi * pw);
  const int slot = ((t - ti * pt) * eh + (y - yi * ph)) * ew + (x - xi * pw);
  const int n = g.n_pre_tiles + (ti * g.nY[h] + yi) * g.nX[h] + xi;
  return n * VSA_TILE + slot;
}

// Unpack in the output's order: one warp per token, the token's [heads, d]
// row written front to back in 512-byte warp stores, each (head, token) row
// gathered from its packed tile (256-byte reads, the access pattern of the
// pack pass). Lanes first resolve one head's packed row each.
template <int CPR>
__global__ void __launch_bounds__(256) unpack_tok_kernel(Geometry g, const uint4* __restrict__ op,
                                                         uint4* __restrict__ o) {
  __shared__ int64_t src_row[8][VSA_MAX_HEADS];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t n_tok = int64_t(g.B) * g.n_tokens;
  const int per_tok = g.Hh * CPR;   // 16-byte chunks of one token's row
  for (int64_t tk = int64_t(blockIdx.x) * 8 + wib; tk < n_tok; tk += int64_t(gridDim.x) * 8) {
    const int b = int(tk / g.n_tokens), tok = int(tk - int64_t(b) * g.n_tokens);
    for (int h = lane; h < g.Hh; h += 32)
      src_row[wib][h] = (int64_t(b * g.Hh + h) * g.nt_max) * VSA_TILE + packed_row(g, h, tok);
    __syncwarp();
    uint4* dst = o + tk * per_tok;
    constexpr int kBatch = 4;   // loads in flight per lane before the stores
    for (int q0 = 0; q0 < per_tok; q0 += 32 * kBatch) {
      uint4 val[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int q = q0 + 32 * u + lane;
        val[u] = q < per_tok ? ld_stream(op + src_row[wib][q / CPR] * CPR + q % CPR) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int q = q0 + 32 * u + lane;
        if (q < per_tok) dst[q] = val[u];
      }
    }
    __syncwarp();   // src_row is rewritten for the next token
  }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Pack fused with pooling (a1 + a2 in one pass over Q and K): one CTA per
// (b, h, packed tile). Thread t moves chunk t mod CPR of rows t / CPR + RG*i of
// Q, K and V, and for a video tile also sums (TripPool: max, min) its 8
// channels of Q and K over those rows in fp32; the warps' partials are
// combined through shared memory into the tile's descriptor, written in the
// score stage's pooled layout [B*heads*ntv_max][KD]: mean (sum / valid
// tokens), then max and min for TripPool. The pooling itself is that of the
// score stage (Ref2VA VSA README: mean-pooled Q, K for the gate score; BSAI
// VedaSparse README "Core Technology: TripPool", eq. 5).
//
// QUANT: the same pass also writes Q and K of every packed tile as e4m3 (fp8)
// with one fp32 scale per (tile, tensor): with amax the tile's largest
// magnitude, scale = amax / 448 (1 for an all-zero tile) and code = e4m3(x /
// scale) (correctly rounded fp32 division, then rounded to nearest even and
// saturated) -- per-tile 8-bit Q K^T, as the tile-skipping kernels on the Veda
// page run it.
// PACK = false: the pooling alone (no V, no packed copies), for the path whose
// attention reads the token-major tensors directly; CTAs of prefix tiles exit.
template <int CPR, bool TRIP, bool QUANT, bool PACK = true>
__global__ void __launch_bounds__(256) pack_pool_kernel(Geometry g, const uint4* __restrict__ q,
                                                        const uint4* __restrict__ k,
                                                        const uint4* __restrict__ v, uint4* __restrict__ qp,
                                                        uint4* __restrict__ kp, uint4* __restrict__ vp,
                                                        const int32_t* __restrict__ counts,
                                                        float* __restrict__ pq, float* __restrict__ pk,
                                                        uint2* __restrict__ qp8, uint2* __restrict__ kp8,
                                                        float* __restrict__ q_scale, float* __restrict__ k_scale) {
  constexpr int D = CPR * 8;
  constexpr int KD = TRIP ? 3 * D : D;
  constexpr int RG = 256 / CPR;       // row groups: 16 (d = 128) or 32 (d = 64)
  constexpr int RPT = 64 / RG;        // rows per thread: 4 or 2
  constexpr int NS = TRIP ? 3 : 1;    // statistics: sum (, max, min)
  __shared__ float part[NS][2][8][D];
  __shared__ float amax_part[2][8];
  const int64_t tile = blockIdx.x;    // bh * nt_max + n
  const int n = int(tile % g.nt_max);
  const int bh = int(tile / g.nt_max);
  const int h = bh % g.Hh, b = bh / g.Hh;
  const int c = threadIdx.x % CPR;
  const int rg = threadIdx.x / CPR;
  const int vt = n - g.n_pre_tiles;
  const bool pool = vt >= 0 && vt < g.ntv[h];   // uniform over the CTA
  if (!PACK && !pool) return;
  float st[NS][2][8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      st[0][t][e] = 0.f;
      if (TRIP) {
        st[NS - 2][t][e] = -INFINITY;
        st[NS - 1][t][e] = INFINITY;
      }
    }
  }
  const uint4 zero = make_uint4(0, 0, 0, 0);
  uint4 keep_q[QUANT ? RPT : 1], keep_k[QUANT ? RPT : 1];   // this thread's Q, K chunks for the fp8 pass
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int s = rg + RG * i;
    const int tok = src_token(g, h, n, s);
    const int64_t dst = (tile * VSA_TILE + s) * CPR + c;
    uint4 a = zero, bb = zero, cc = zero;
    if (tok >= 0) {
      const int64_t src = ((int64_t(b) * g.n_tokens + tok) * g.Hh + h) * CPR + c;
      a = ld_stream(q + src);
      bb = ld_stream(k + src);
      if (PACK) cc = ld_stream(v + src);
    }
    if (PACK) {
      qp[dst] = a;
      kp[dst] = bb;
      vp[dst] = cc;
    }
    if constexpr (QUANT) {
      keep_q[i] = a;
      keep_k[i] = bb;
    }
    if (pool && tok >= 0) {
      float xq[8], xk[8];
      bf16x8_to_f32(a, xq);
      bf16x8_to_f32(bb, xk);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        st[0][0][e] += xq[e];
        st[0][1][e] += xk[e];
        if (TRIP) {
          st[NS - 2][0][e] = fmaxf(st[NS - 2][0][e], xq[e]);
          st[NS - 2][1][e] = fmaxf(st[NS - 2][1][e], xk[e]);
          st[NS - 1][0][e] = fminf(st[NS - 1][0][e], xq[e]);
          st[NS - 1][1][e] = fminf(st[NS - 1][1][e], xk[e]);
        }
      }
    }
  }
  if constexpr (QUANT) {
    // the tile's largest magnitude of Q and of K, over every thread's rows
    const int lane0 = threadIdx.x & 31, warp0 = threadIdx.x >> 5;
    float am[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      float xq[8], xk[8];
      bf16x8_to_f32(keep_q[i], xq);
      bf16x8_to_f32(keep_k[i], xk);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        am[0] = fmaxf(am[0], fabsf(xq[e]));
        am[1] = fmaxf(am[1], fabsf(xk[e]));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      am[0] = fmaxf(am[0], __shfl_xor_sync(0xffffffffu, am[0], o));
      am[1] = fmaxf(am[1], __shfl_xor_sync(0xffffffffu, am[1], o));
    }
    if (lane0 == 0) {
      amax_part[0][warp0] = am[0];
      amax_part[1][warp0] = am[1];
    }
    __syncthreads();
    float sc[2];   // dequantisation scale amax / 448; codes are x / scale
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      float m = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) m = fmaxf(m, amax_part[t][w]);
      sc[t] = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
    }
    if (threadIdx.x == 0) {
      q_scale[tile] = sc[0];
      k_scale[tile] = sc[1];
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const int s = rg + RG * i;
      const int64_t dst8 = (tile * VSA_TILE + s) * CPR + c;   // 8 bytes per 8 channels
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        float x[8];
        bf16x8_to_f32(t ? keep_k[i] : keep_q[i], x);
        uint32_t w[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
              make_float2(__fdiv_rn(x[4 * e], sc[t]), __fdiv_rn(x[4 * e + 1], sc[t])), __NV_SATFINITE, __NV_E4M3);
          const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
              make_float2(__fdiv_rn(x[4 * e + 2], sc[t]), __fdiv_rn(x[4 * e + 3], sc[t])), __NV_SATFINITE,
              __NV_E4M3);
          w[e] = uint32_t(lo) | (uint32_t(hi) << 16);
        }
        (t ? kp8 : qp8)[dst8] = make_uint2(w[0], w[1]);
      }
    }
  }
  if (!pool) return;
  // lanes l and l ^ CPR (and l ^ 2 CPR for d = 64) hold the same chunk of
  // different rows: fold them so that lanes < CPR hold the warp's partials
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = CPR; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        st[0][t][e] += __shfl_xor_sync(0xffffffffu, st[0][t][e], o);
        if (TRIP) {
          st[NS - 2][t][e] = fmaxf(st[NS - 2][t][e], __shfl_xor_sync(0xffffffffu, st[NS - 2][t][e], o));
          st[NS - 1][t][e] = fminf(st[NS - 1][t][e], __shfl_xor_sync(0xffffffffu, st[NS - 1][t][e], o));
        }
      }
    }
  }
  if (lane < CPR) {
#pragma unroll
    for (int z = 0; z < NS; ++z)
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 8; ++e) part[z][t][warp][8 * lane + e] = st[z][t][e];
  }
  __syncthreads();
  if (threadIdx.x < 2 * D) {
    const int t = threadIdx.x / D, ch = threadIdx.x % D;
    float sum = 0.f, mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      sum += part[0][t][w][ch];
      if (TRIP) {
        mx = fmaxf(mx, part[NS - 2][t][w][ch]);
        mn = fminf(mn, part[NS - 1][t][w][ch]);
      }
    }
    const float cnt = float(counts[h * g.nt_max + n]);
    float* out = (t ? pk : pq) + (int64_t(bh) * g.ntv_max + vt) * KD;
    out[ch] = sum / cnt;
    if (TRIP) {
      out[D + ch] = mx;
      out[2 * D + ch] = mn;
    }
  }
}

int grid_for(const vsa_plan* p, int64_t total) {
  const int64_t want = (total + 255) / 256;
  const int64_t cap = int64_t(p->num_sms) * 8;  // 8 blocks of 256 threads per SM
  return int(want < cap ? want : cap);
}

}  // namespace

cudaError_t launch_pack(const vsa_plan* p, const void* q, const void* k, const void* v, void* qp,
                        void* kp, void* vp, cudaStream_t s) {
  const Geometry& g = p->geo;
  const int cpr = g.d / 8;
  const int64_t total = int64_t(g.B) * g.Hh * g.nt_max * VSA_TILE * cpr;
  const int grid = grid_for(p, total);
  auto* q4 = static_cast<const uint4*>(q);
  auto* k4 = static_cast<const uint4*>(k);
  auto* v4 = static_cast<const uint4*>(v);
  auto* qp4 = q ? static_cast<uint4*>(qp) : nullptr;
  auto* kp4 = k ? static_cast<uint4*>(kp) : nullptr;
  auto* vp4 = v ? static_cast<uint4*>(vp) : nullptr;
  if (cpr == 16)
    pack_kernel<16><<<grid, 256, 0, s>>>(g, q4, k4, v4, qp4, kp4, vp4);
  else
    pack_kernel<8><<<grid, 256, 0, s>>>(g, q4, k4, v4, qp4, kp4, vp4);
  return cudaGetLastError();
}

cudaError_t launch_pool(const vsa_plan* p, const void* q, const void* k, float* pooled_q, float* pooled_k,
                        cudaStream_t s) {
  const Geometry& g = p->geo;
  const int64_t tiles = int64_t(g.B) * g.Hh * g.nt_max;
  const bool trip = p->desc.score_mode == VSA_SCORE_TRIPPOOL;
  auto* q4 = static_cast<const uint4*>(q);
  auto* k4 = static_cast<const uint4*>(k);
  const int32_t* cnt = p->d_tile_count;
  if (g.d == 128) {
    if (trip)
      pack_pool_kernel<16, true, false, false><<<tiles, 256, 0, s>>>(g, q4, k4, nullptr, nullptr, nullptr, nullptr, cnt,
                                                                     pooled_q, pooled_k, nullptr, nullptr, nullptr, nullptr);
    else
      pack_pool_kernel<16, false, false, false><<<tiles, 256, 0, s>>>(g, q4, k4, nullptr, nullptr, nullptr, nullptr, cnt,
                                                                      pooled_q, pooled_k, nullptr, nullptr, nullptr, nullptr);
  } else {
    if (trip)
      pack_pool_kernel<8, true, false, false><<<tiles, 256, 0, s>>>(g, q4, k4, nullptr, nullptr, nullptr, nullptr, cnt,
                                                                    pooled_q, pooled_k, nullptr, nullptr, nullptr, nullptr);
    else
      pack_pool_kernel<8, false, false, false><<<tiles, 256, 0, s>>>(g, q4, k4, nullptr, nullptr, nullptr, nullptr, cnt,
                                                                     pooled_q, pooled_k, nullptr, nullptr, nullptr, nullptr);
  }
  return cudaGetLastError();
}

cudaError_t launch_pack_pool(const vsa_plan* p, const void* q, const void* k, const void* v, void* qp,
                             void* kp, void* vp, float* pooled_q, float* pooled_k, cudaStream_t s,
                             void* qp8, void* kp8, float* q_scale, float* k_scale) {
  const Geometry& g = p->geo;
  const int64_t tiles = int64_t(g.B) * g.Hh * g.nt_max;
  const bool trip = p->desc.score_mode == VSA_SCORE_TRIPPOOL;
  auto* q4 = static_cast<const uint4*>(q);
  auto* k4 = static_cast<const uint4*>(k);
  auto* v4 = static_cast<const uint4*>(v);
  auto* qp4 = static_cast<uint4*>(qp);
  auto* kp4 = static_cast<uint4*>(kp);
  auto* vp4 = static_cast<uint4*>(vp);
  const int32_t* cnt = p->d_tile_count;
  auto* q8 = static_cast<uint2*>(qp8);
  auto* k8 = static_cast<uint2*>(kp8);
  if (qp8) {   // with the fp8 copies of Q and K (head_dim 128 only)
    if (g.d != 128) return cudaErrorInvalidValue;
    if (trip)
      pack_pool_kernel<16, true, true><<<tiles, 256, 0, s>>>(g, q4, k4, v4, qp4, kp4, vp4, cnt, pooled_q, pooled_k,
                                                             q8, k8, q_scale, k_scale);
    else
      pack_pool_kernel<16, false, true><<<tiles, 256, 0, s>>>(g, q4, k4, v4, qp4, kp4, vp4, cnt, pooled_q, pooled_k,
                                                              q8, k8, q_scale, k_scale);
  } else if (g.d == 128) {
    if (trip)
      pack_pool_kernel<16, true, false><<<tiles, 256, 0, s>>>(g, q4, k4, v4, qp4, kp4, vp4, cnt, pooled_q, pooled_k,
                                                              nullptr, nullptr, nullptr, nullptr);
    else
      pack_pool_kernel<16, false, false><<<tiles, 256, 0, s>>>(g, q4, k4, v4, qp4, kp4, vp4, cnt, pooled_q, pooled_k,
                                                               nullptr, nullptr, nullptr, nullptr);
  } else {
    if (trip)
      pack_pool_kernel<8, true, false><<<tiles, 256, 0, s>>>(g, q4, k4, v4, qp4, kp4, vp4, cnt, pooled_q, pooled_k,
                                                             nullptr, nullptr, nullptr, nullptr);
    else
      pack_pool_kernel<8, false, false><<<tiles, 256, 0, s>>>(g, q4, k4, v4, qp4, kp4, vp4, cnt, pooled_q, pooled_k,
                                                              nullptr, nullptr, nullptr, nullptr);
  }
  return cudaGetLastError();
}

cudaError_t launch_unpack(const vsa_plan* p, const void* op, void* o, cudaStream_t s) {
  const Geometry& g = p->geo;
  const int64_t tokens = int64_t(g.B) * g.n_tokens;
  if (tokens == 0) return cudaSuccess;
  const int64_t want = (tokens + 7) / 8;                // eight warps (tokens) per CTA
  const int64_t cap = int64_t(p->num_sms) * 8;         // eight CTAs of 256 threads per SM, grid-stride
  const unsigned grid = unsigned(want < cap ? want : cap);
  if (g.d == 128)
    unpack_tok_kernel<16><<<grid, 256, 0, s>>>(g, static_cast<const uint4*>(op), static_cast<uint4*>(o));
  else
    unpack_tok_kernel<8><<<grid, 256, 0, s>>>(g, static_cast<const uint4*>(op), static_cast<uint4*>(o));
  return cudaGetLastError();
}

}  // namespace vsa
