// a6: block-sparse exact attention over kept tiles, TMA + tcgen05 (TMEM) on sm_100a.
//
// What it computes (BSAI VedaSparse README, "Core Technology: Tile-Skipping"
// and "v3.4 Highlights": conditioning rows and keys stay exact; Ref2VA VSA
// README, "two-tier attention layout"): for every query tile, exact softmax
// attention over the valid keys of the tiles it keeps -- all tiles for a prefix
// query tile, the prefix tiles plus its top-k video tiles for a video query
// tile. Scores and accumulation are fp32, P is rounded to bf16 for the PV
// product, O is rounded to bf16 once.
//
// How: one persistent CTA per SM walks a work list of 128-row blocks. A block
// is two query tiles of one (batch, head) -- neighbours along h on the video
// grid, or two prefix tiles -- so the tensor core runs M = 128 MMAs. They
// share one key list: the union of their kept tiles, each entry tagged with
// which of the two row-halves keeps it; a row-half masks the other's tiles to
// -inf. Key tiles go through smem two at a time (128 keys per step).
//
// Warp roles (416 threads):
//   warp 0  TMA producers: lane 0 the Q pair of every block of rows and the K
//           tile pairs (2 stages), lane 1 the V tile pairs (3 stages)
//   warp 1  MMA issuer for S = Q K^T (Q and K in smem) into one of two TMEM
//           S buffers
//   warps 3, 12  MMA issuers for O_0 += P_0 V_0 and O_1 += P_1 V_1 (P in
//           TMEM over the S columns it came from, V in smem)
//   warp 2  scheduler: fetches the next block from a global counter and builds
//           its merged key list (double buffered, in a per-CTA global slice)
//   warps 4-11 softmax, two warpgroups: warpgroup w owns key tile w of every
//           128-key block for all 128 rows (row = TMEM lane) with its own
//           online softmax (running max, row sum, partial output O_w); the
//           epilogue merges the two partial softmaxes of each row.
//
// Each mbarrier wait and commit costs an issuing thread tens of cycles next
// to a 64-cycle MMA, so S and the two PV halves come from three issuing
// threads, each waiting only on its own barriers. The softmax warpgroups never
// wait for each other inside an item, so one computes exponentials while the
// other loads and reduces its scores.
//
// TMEM holds the two S buffers and the two partial outputs; shared memory the
// Q pair and the K and V stages, in the canonical 128-byte-swizzled UMMA
// layouts that TMA SWIZZLE_128B writes (Q and K K-major, V MN-major). The
// tiles come from the packed tensors as 2-D boxes, or (DIRECT) straight from
// the token-major tensors as 3-D / 5-D boxes with O written token-major: the
// same shared-memory images and the same results, but scattered rows that
// TMA fetches several times more slowly, so that instance is an opt-in.
// Every wait is bounded (about two seconds); on expiry the CTA latches a
// timeout in the plan's error word, drains its copies and MMAs, frees TMEM and
// returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tc_sm100.h"
#include "vsa_internal.h"

namespace vsa {
namespace {

using namespace tc;

constexpr int kThreads = 416;
constexpr int kSBuf = 2;        // TMEM S buffers
constexpr int kPvWarp0 = 3;     // PV MMA issuer for softmax warpgroup 0's keys
constexpr int kPvWarp1 = 12;    // ... and for warpgroup 1's
constexpr int kSmWarps = 8;     // softmax warps (4-11); each arrives once on their barriers
constexpr float kLazy = 8.0f;  // log2 headroom before the running max is raised
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTileBytes = 64 * 64 * 2;  // one 64 x 64 bf16 TMA box
// K / V tile-pair stages in shared memory: a TMA load takes microseconds from
// L2, so several must be in flight per CTA.
#ifndef VSA_K_STAGES
#define VSA_K_STAGES 2
#endif
#ifndef VSA_V_STAGES
#define VSA_V_STAGES 3
#endif

// Packed fp32 pairs (sm_100 FFMA2 / FADD2) and the 3-input max.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// 2^x for two values on the FMA pipe instead of the MUFU unit.
// Cody-Waite style split x = n + f with n = round(x) (adding 1.5 * 2^23 rounds
// to an integer held in the low mantissa bits), f in [-1/2, 1/2], 2^f from a
// degree-4 polynomial fitted here by Remez exchange for minimum relative error
// (max 2.7e-6 in fp32 evaluation; see fit_exp2_poly.py), and 2^n added into
// the exponent field. x is clamped to -125 so the exponent never underflows;
// 2^-125 stands in for 0 next to the row's largest term (>= 2^-8).
#ifndef VSA_EXP_POLY_EVERY
#define VSA_EXP_POLY_EVERY 8   // one pair in eight goes through the polynomial (0: none)
#endif
__device__ __forceinline__ void ex2_fma_pipe(float x0, float x1, float& y0, float& y1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const uint64_t x = f2pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = fadd2(x, f2pack(kRound, kRound));
  const uint64_t n = fadd2(t, f2pack(-kRound, -kRound));
  const uint64_t f = fadd2(x, n ^ 0x8000000080000000ull);   // x - n
  uint64_t p = ffma2(f2pack(0.009570102207362652f, 0.009570102207362652f), f,
                     f2pack(0.05591785907745361f, 0.05591785907745361f));
  p = ffma2(p, f, f2pack(0.240247443318367f, 0.240247443318367f));
  p = ffma2(p, f, f2pack(0.6931217908859253f, 0.6931217908859253f));
  p = ffma2(p, f, f2pack(0.9999992847442627f, 0.9999992847442627f));
  float p0, p1, t0, t1;
  f2unpack(p, p0, p1);
  f2unpack(t, t0, t1);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// ------------------------------------------------------- shared layout ----

struct ItemInfo {
  int32_t bh, qa, qb, n_entries;
  int32_t rows_a, rows_b, end, bad;
};

template <int D, bool F8 = false>
struct Smem {
  static constexpr uint32_t kHalfBytes = 128 * 128;               // 128 rows x 128 B
  // K tile pair (K-major): D bf16 per row in D/64 128-byte halves, or (F8) D = 128 e4m3 bytes in one
  static constexpr uint32_t kKBytes = F8 ? kHalfBytes : (D / 64) * kHalfBytes;
  static constexpr uint32_t kVBytes = (D / 64) * kHalfBytes;       // V tile pair (MN-major, bf16)
  static constexpr int kKStages = VSA_K_STAGES;
  static constexpr int kVStages = VSA_V_STAGES;
  static constexpr uint32_t kQBytes = kKBytes;                     // the Q pair (K-major)
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + kQBytes;
  static constexpr uint32_t oV = oK + kKStages * kKBytes;
  static constexpr uint32_t oBar = oV + kVStages * kVBytes;
  static constexpr uint32_t kNumBars = 40;
  static constexpr uint32_t oInfo = oBar + kNumBars * 8;
  static constexpr uint32_t oMisc = oInfo + 2 * sizeof(ItemInfo);  // tmem base, abort flag
  static constexpr uint32_t oXchg = oMisc + 16;                     // row max / row sum exchange
  static constexpr uint32_t oEnd = oXchg + (2 * 128 + 2 * 128) * 4;
};

// barrier indices
enum {
  B_QFULL = 0, B_QEMPTY, B_KFULL0, B_KEMPTY0 = B_KFULL0 + 4, B_VFULL0 = B_KEMPTY0 + 4, B_VEMPTY0 = B_VFULL0 + 4,
  // P_FULL: [softmax warpgroup][S buffer]; P_DONE: [S buffer], both PV MMAs of the buffer's block
  B_SFULL0 = B_VEMPTY0 + 4, B_PFULL0 = B_SFULL0 + kSBuf, B_PDONE0 = B_PFULL0 + 2 * kSBuf,
  B_LFULL0 = B_PDONE0 + kSBuf, B_LFULL1, B_LEMPTY0, B_LEMPTY1, B_OFULL, B_OFREE, B_LX, B_DRAIN, B_HOLD, B_COUNT
};
static_assert(B_COUNT <= 40, "barrier slots");

struct AttnParams {
  const int32_t* idx;      // [B, heads, ntv_max, k_max]
  const int32_t* idx_ref;  // [B, heads, ntv_max, k_ref_max] kept reference tiles, or null (all prefix dense)
  const int32_t* ref_tiles;   // [n_ref] prefix tile id of each reference tile
  const int32_t* prefix_ref;  // [n_pre] position among the reference tiles, or -1
  const int32_t* counts;   // [heads, nt_max]
  const WorkItem* items;
  int64_t n_items;
  __nv_bfloat16* out;      // packed O
  float* lse;
  uint32_t* state;         // [0] error word, [1] work counter, [2..3] computed pairs
  int32_t heads, nt_max, ntv_max, k_max, n_pre;
  int32_t list_cap, bitmap_words;
  uint32_t* lists;         // [CTAs][2][list_cap] merged key lists (one slice per CTA)
  uint32_t* bitmaps;       // [CTAs][2][bitmap_words] scratch of the list builder
  float scale_log2;
  const float* q_scale;    // fp8 Q K^T: [B, heads, nt_max] per-tile scales of Q and K (else null)
  const float* k_scale;
  int32_t ntv[VSA_MAX_HEADS];
  int32_t k[VSA_MAX_HEADS];
  int32_t n_ref, k_ref_max;
  int32_t k_ref[VSA_MAX_HEADS];
  uint64_t wait_ns;        // bound of every mbarrier wait
  int32_t hold;            // test hook: the softmax waits, at its first block, on a barrier nothing arrives on
};

// Tiles straight from the token-major Q, K, V [1, N, heads, d] (no packed
// copies): a prefix tile is a 3-D box (64 channels, 1 head, 64 tokens) of the
// sequence, a video tile of head h a 5-D box (64 channels, 1 head, pw, ph, pt)
// of the video grid [T][H][W][heads][d], which TMA writes into shared memory
// in the same (t, h, w) row order and swizzle as the packed tile's 2-D box.
// Rows past a prefix segment hold the next tokens (masked keys, unwritten
// query rows); rows past the grid's far edge in t are zero-filled, as the
// packed tile's. O is written token-major.
constexpr int kMaxShapes = 4;   // distinct (pt, ph, pw) among the heads
struct DirectMaps {
  CUtensorMap pre[3];                  // Q, K, V over the whole sequence
  CUtensorMap vid[kMaxShapes][3];      // Q, K, V over the video grid, per tile shape
  int32_t n_pre_tok, n_pre_tiles, n_seg, T, H, W;
  int32_t seg_tok0[VSA_MAX_SEGMENTS + 1], seg_tile0[VSA_MAX_SEGMENTS + 1];
  int32_t shp[kMaxShapes][3];          // pt, ph, pw
  int8_t shape_of[VSA_MAX_HEADS];      // shape index of each head
};

__device__ __forceinline__ int prefix_tile_token0(const DirectMaps& dm, int tile) {
  int s = 0;
#pragma unroll 1
  while (s + 1 < dm.n_seg && tile >= dm.seg_tile0[s + 1]) ++s;
  return dm.seg_tok0[s] + (tile - dm.seg_tile0[s]) * VSA_TILE;
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

template <int D, bool F8 = false, bool DIRECT = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv,
                const __grid_constant__ AttnParams prm, const __grid_constant__ DirectMaps dm) {
  using L = Smem<D, F8>;
  static_assert(!F8 || D == 128, "fp8 Q K^T: one 128-byte swizzle row per token");
  static_assert(!(F8 && DIRECT), "the fp8 instance reads the packed e4m3 copies");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + L::oBar + 8u * uint32_t(i); };
  ItemInfo* info = reinterpret_cast<ItemInfo*>(smem + L::oInfo);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::oMisc);
  volatile uint32_t* abort_flag = misc + 1;
  // this CTA's slice of the key-list table (global memory; written and read
  // inside the CTA, ordered by the list mbarriers)
  uint32_t* lists = prm.lists + size_t(blockIdx.x) * 2 * prm.list_cap;
  uint32_t* bitmaps = prm.bitmaps + size_t(blockIdx.x) * 2 * prm.bitmap_words;
  uint32_t* gerr = prm.state;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar(B_KFULL0 + i), 1);
      mbar_init(bar(B_KEMPTY0 + i), 1);
      mbar_init(bar(B_VFULL0 + i), 1);
      mbar_init(bar(B_VEMPTY0 + i), 2);   // both PV issuers
    }
    for (int i = 0; i < kSBuf; ++i) mbar_init(bar(B_SFULL0 + i), 1);
    for (int i = 0; i < 2 * kSBuf; ++i) mbar_init(bar(B_PFULL0 + i), kSmWarps / 2);   // one softmax warpgroup
    for (int i = 0; i < kSBuf; ++i) mbar_init(bar(B_PDONE0 + i), 2);   // both PV issuers
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_LFULL0 + i), 32);
      mbar_init(bar(B_LEMPTY0 + i), kSmWarps + 5);   // + S issuer, two PV issuers, two producer lanes
    }
    mbar_init(bar(B_OFULL), 2);
    mbar_init(bar(B_OFREE), kSmWarps);
    mbar_init(bar(B_LX), kSmWarps);
    mbar_init(bar(B_DRAIN), 3);   // the three MMA issuers
    mbar_init(bar(B_HOLD), 1);    // test hook: never arrived on
    misc[1] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sbase + L::oMisc),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  // TMEM columns: S buffers [0,128) and [128,256) for alternate key blocks;
  // O_0 [256, 256+D) and O_1 [384, 384+D), the partial outputs of the two
  // softmax warpgroups (keys of tile 0 / tile 1 of every block). P (bf16
  // pairs) is written over the S columns it was computed from: keys 0-63 at
  // [0,32), keys 64-127 at [64,96) of the buffer. S for block g + 2 is issued
  // only after both PV MMAs that read P of block g have completed.
  const uint32_t tS = tmem;
  const uint32_t tO0 = tmem + 256;
  static_assert(D <= 128, "each O fits 128 columns");

  if (warp == 2) {
    // ------------------------------------------------ scheduler / lists ---
    for (uint32_t it = 0;; ++it) {
      const int slot = it & 1;
      bool ok = true;
      if (lane == 0) ok = wait_bar(bar(B_LEMPTY0 + slot), ((it >> 1) & 1) ^ 1, abort_flag, gerr, prm.wait_ns);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      long long item = 0;
      if (lane == 0) item = (long long)atomicAdd(prm.state + 1, 1u);
      item = __shfl_sync(0xffffffffu, item, 0);
      ItemInfo& inf = info[slot];
      if (item >= prm.n_items) {
        if (lane == 0) inf.end = 1;
        __syncwarp();
        mbar_arrive(bar(B_LFULL0 + slot));
        break;
      }
      const WorkItem wi = prm.items[item];
      const int h = wi.bh % prm.heads;
      const int b = wi.bh / prm.heads;
      const int ntv = prm.ntv[h];
      const int nt = prm.n_pre + ntv;
      const int32_t* cnt = prm.counts + size_t(h) * prm.nt_max;
      uint32_t* list = lists + slot * prm.list_cap;
      const uint32_t maskab = wi.qb >= 0 ? 3u : 1u;
      int n_entries = 0;
      bool bad = false;
      if (wi.kind == 0) {
        // prefix query tiles: every tile of the head, kept by both rows-halves
        for (int t = lane; t < nt; t += 32) list[t] = uint32_t(t) | (maskab << 16) | (uint32_t(cnt[t]) << 24);
        n_entries = nt;
      } else {
        int base = 0;
        if (prm.idx_ref) {   // reference segments: the dense prefix tiles first, compacted
          for (int t0 = 0; t0 < prm.n_pre; t0 += 32) {
            const int t = t0 + lane;
            const int keep = (t < prm.n_pre && prm.prefix_ref[t] < 0) ? 1 : 0;
            int total;
            const int pos = base + warp_excl_scan(keep, lane, &total);
            if (keep) list[pos] = uint32_t(t) | (maskab << 16) | (uint32_t(cnt[t]) << 24);
            base += total;
          }
        } else {             // every prefix tile
          for (int t = lane; t < prm.n_pre; t += 32)
            list[t] = uint32_t(t) | (maskab << 16) | (uint32_t(cnt[t]) << 24);
          base = prm.n_pre;
        }
        // The kept tiles of both query tiles, merged: each selection row (ascending
        // positions among nbits candidate tiles) sets bits of its row-half's
        // bitmap; the union is appended in ascending order, each entry tagged with
        // the row-halves that keep it. A row out of range or not ascending marks
        // the item bad (warp-uniform after the vote).
        auto merge = [&](const int32_t* sel, int stride, int kcount, int nbits, bool is_ref) {
          uint32_t* bmA = bitmaps;
          uint32_t* bmB = bitmaps + prm.bitmap_words;
          const int words = (nbits + 31) >> 5;
          for (int w = lane; w < words; w += 32) {
            bmA[w] = 0u;
            bmB[w] = 0u;
          }
          __syncwarp();
          for (int side = 0; side < 2; ++side) {
            const int qt = side == 0 ? wi.qa : wi.qb;
            if (qt < 0) continue;
            const int32_t* row = sel + ((size_t(b) * prm.heads + h) * prm.ntv_max + (qt - prm.n_pre)) * stride;
            uint32_t* bm = side == 0 ? bmA : bmB;
            for (int e = lane; e < kcount; e += 32) {
              const int j = row[e];
              const int jp = e > 0 ? row[e - 1] : -1;
              if (j < 0 || j >= nbits || j <= jp) {
                bad = true;
              } else {
                atomicOr(bm + (j >> 5), 1u << (j & 31));
              }
            }
          }
          bad = __any_sync(0xffffffffu, bad);
          __syncwarp();
          if (!bad) {
            for (int w0 = 0; w0 < words; w0 += 32) {
              const int w = w0 + lane;
              const uint32_t a = w < words ? bmA[w] : 0u;
              const uint32_t bb = w < words ? bmB[w] : 0u;
              uint32_t u = a | bb;
              int total;
              int pos = base + warp_excl_scan(__popc(u), lane, &total);
              while (u) {
                const int bit = __ffs(u) - 1;
                u &= u - 1;
                const int j = (w << 5) + bit;
                const uint32_t m = ((a >> bit) & 1u) | (((bb >> bit) & 1u) << 1);
                const int t = is_ref ? prm.ref_tiles[j] : prm.n_pre + j;
                list[pos++] = uint32_t(t) | (m << 16) | (uint32_t(cnt[t]) << 24);
              }
              base += total;
            }
          }
          __syncwarp();
        };
        if (prm.idx_ref) merge(prm.idx_ref, prm.k_ref_max, prm.k_ref[h], prm.n_ref, true);
        if (!bad) merge(prm.idx, prm.k_max, prm.k[h], ntv, false);
        if (bad && lane == 0) atomicOr(gerr, kErrBadIndex);
        n_entries = base;   // a bad item keeps only entries already validated; its rows are not written
      }
      __syncwarp();
      // valid-pair count for the stats: rows x keys each row-half keeps
      unsigned long long ka = 0, kb = 0;
      for (int e = lane; e < n_entries; e += 32) {
        const uint32_t v = list[e];
        const uint32_t c = v >> 24;
        if (v & (1u << 16)) ka += c;
        if (v & (2u << 16)) kb += c;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ka += __shfl_xor_sync(0xffffffffu, ka, o);
        kb += __shfl_xor_sync(0xffffffffu, kb, o);
      }
      const int rows_a = cnt[wi.qa];
      const int rows_b = wi.qb >= 0 ? cnt[wi.qb] : 0;
      if (lane == 0) {
        inf.bh = wi.bh;
        inf.qa = wi.qa;
        inf.qb = wi.qb;
        inf.n_entries = n_entries;
        inf.rows_a = rows_a;
        inf.rows_b = rows_b;
        inf.end = 0;
        inf.bad = bad ? 1 : 0;
        if (!bad)
          atomicAdd(reinterpret_cast<unsigned long long*>(prm.state + 2),
                    (unsigned long long)rows_a * ka + (unsigned long long)rows_b * kb);
      }
      __syncwarp();
      mbar_arrive(bar(B_LFULL0 + slot));
    }
  } else if (warp == 0) {
    // --------------------------------------------------------- producers ---
    // lane 0: the Q pair of every item and the K tile pairs; lane 1: the V tile
    // pairs. Separate threads (diverged lanes make independent progress), so a
    // K load never queues behind a V load that is waiting for its stage to be
    // released by a PV MMA.
    if (lane < 2) {
      const bool is_k = lane == 0;
      const CUtensorMap* map = is_k ? &tk : &tv;
      const int full0 = is_k ? B_KFULL0 : B_VFULL0;
      const int empty0 = is_k ? B_KEMPTY0 : B_VEMPTY0;
      const int nst = is_k ? L::kKStages : L::kVStages;
      // box c (channels 64c .. 64c + 63) of tile `tile` of tensor m (0 Q, 1 K, 2 V) of (batch, head) bh
      auto load_box = [&](uint32_t dst, int m, const CUtensorMap* map2d, int c, int bh, int tile, uint32_t fb) {
        if constexpr (DIRECT) {
          const int h = bh % prm.heads;
          if (tile < dm.n_pre_tiles) {
            tma_load_3d(dst, &dm.pre[m], 64 * c, h, prefix_tile_token0(dm, tile), fb);
          } else {
            const int sh = dm.shape_of[h];
            const int pt = dm.shp[sh][0], ph = dm.shp[sh][1], pw = dm.shp[sh][2];
            const int nX = dm.W / pw, nYX = (dm.H / ph) * nX;
            const int v = tile - dm.n_pre_tiles;
            const int ti = v / nYX, yi = (v - ti * nYX) / nX, xi = v - ti * nYX - yi * nX;
            tma_load_5d(dst, &dm.vid[sh][m], 64 * c, h, xi * pw, yi * ph, ti * pt, fb);
          }
        } else {
          tma_load_2d(dst, map2d, 64 * c, (bh * prm.nt_max + tile) * 64, fb);
        }
      };
      uint32_t g = 0;          // key blocks issued
      int st = 0;              // stage of block g (g mod nst)
      uint32_t ph = 0;         // phase of that stage ((g / nst) & 1)
      uint32_t issuedQ = 0;    // Q loads issued
      for (uint32_t it = 0;; ++it) {
        const int slot = it & 1;
        if (!wait_bar(bar(B_LFULL0 + slot), (it >> 1) & 1, abort_flag, gerr, prm.wait_ns)) break;
        const ItemInfo inf = info[slot];
        if (inf.end) break;
        const uint32_t* list = lists + slot * prm.list_cap;
        if (is_k) {   // rows 0-63: tile qa, rows 64-127: tile qb (qa again when there is none)
          if (!wait_bar(bar(B_QEMPTY), (it & 1) ^ 1, abort_flag, gerr, prm.wait_ns)) break;
          mbar_expect_tx(bar(B_QFULL), 2 * (F8 ? 1 : D / 64) * kTileBytes);
          const int qb = inf.qb >= 0 ? inf.qb : inf.qa;
          for (int c = 0; c < (F8 ? 1 : D / 64); ++c) {   // 64-row boxes of 128 bytes per row
            load_box(sbase + L::oQ + c * L::kHalfBytes, 0, &tq, c, inf.bh, inf.qa, bar(B_QFULL));
            load_box(sbase + L::oQ + c * L::kHalfBytes + 8192, 0, &tq, c, inf.bh, qb, bar(B_QFULL));
          }
          ++issuedQ;
        }
        const int nblk = (inf.n_entries + 1) >> 1;
        bool ok = true;
        // key-list entries come from global memory: load each block's pair one block ahead
        uint32_t na = nblk > 0 ? list[0] : 0u, nb = 1 < inf.n_entries ? list[1] : na;
        for (int j = 0; j < nblk; ++j) {
          const int ta = int(na & 0xFFFFu);
          const int tb = int(nb & 0xFFFFu);
          if (j + 1 < nblk) {
            na = list[2 * j + 2];
            nb = 2 * j + 3 < inf.n_entries ? list[2 * j + 3] : na;
          }
          if (!(ok = wait_bar(bar(empty0 + st), ph ^ 1, abort_flag, gerr, prm.wait_ns))) break;
          mbar_expect_tx(bar(full0 + st), 2 * (is_k && F8 ? 1 : D / 64) * kTileBytes);
          if (is_k) {   // K-major: tile a rows 0-63, tile b rows 64-127 of each 128-byte half
            const uint32_t sk = sbase + L::oK + st * L::kKBytes;
            for (int c = 0; c < (F8 ? 1 : D / 64); ++c) {
              load_box(sk + c * L::kHalfBytes, 1, map, c, inf.bh, ta, bar(full0 + st));
              load_box(sk + c * L::kHalfBytes + 8192, 1, map, c, inf.bh, tb, bar(full0 + st));
            }
          } else {      // MN-major: tile a then tile b, each as D/64 boxes of 64 keys x 64 columns
            const uint32_t sv = sbase + L::oV + st * L::kVBytes;
            for (int c = 0; c < D / 64; ++c) {
              load_box(sv + c * 8192, 2, map, c, inf.bh, ta, bar(full0 + st));
              load_box(sv + (D / 64) * 8192 + c * 8192, 2, map, c, inf.bh, tb, bar(full0 + st));
            }
          }
          ++g;
          if (++st == nst) {
            st = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        mbar_arrive(bar(B_LEMPTY0 + slot));   // this lane is done with the slot's list
      }
      if (*abort_flag) {
        // let every copy this thread issued land before shared memory is released
        if (is_k && issuedQ) drain_wait(bar(B_QFULL), (issuedQ - 1) & 1);
        for (uint32_t gg = (g >= uint32_t(nst) ? g - nst : 0); gg < g; ++gg)
          drain_wait(bar(full0 + int(gg % nst)), (gg / nst) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- S MMA ---
    if (lane == 0) {
      constexpr uint32_t idS = F8 ? idesc_e4m3(128, 128) : idesc_bf16(128, 128, 0, 0);
      // descriptors of the stage bases; a stage or k-step adds (byte offset >> 4)
      const uint64_t dq = sw128_desc(sbase + L::oQ, 16, 1024);
      const uint64_t dk0 = sw128_desc(sbase + L::oK, 16, 1024);
      int kst = 0;               // K stage of the next S MMA
      uint32_t kph = 0;          // its phase
      int sb = 0;                // S buffer of block g (g mod kSBuf)
      uint32_t su = 0;           // uses of that buffer before block g (g / kSBuf)
      bool ok = true;
      for (uint32_t it = 0; ok; ++it) {
        const int slot = it & 1;
        if (!wait_bar(bar(B_LFULL0 + slot), (it >> 1) & 1, abort_flag, gerr, prm.wait_ns)) break;
        const ItemInfo inf = info[slot];
        if (inf.end) break;
        mbar_arrive(bar(B_LEMPTY0 + slot));     // the item's info is copied
        if (!wait_bar(bar(B_QFULL), it & 1, abort_flag, gerr, prm.wait_ns)) break;
        const int nblk = (inf.n_entries + 1) >> 1;
        if (nblk == 0) tc_commit(bar(B_QEMPTY));   // a rejected item without prefix tiles
        for (int j = 0; j < nblk; ++j) {
          if (!(ok = wait_bar(bar(B_KFULL0 + kst), kph, abort_flag, gerr, prm.wait_ns))) break;
          // the buffer's previous P has been read by both PV MMAs (one barrier counts both)
          if (su > 0 && !(ok = wait_bar(bar(B_PDONE0 + sb), (su - 1) & 1, abort_flag, gerr, prm.wait_ns))) break;
          tc_fence_after();
          const uint64_t dk = dk0 + ((kst * L::kKBytes) >> 4);
          if constexpr (F8) {
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) {   // 32 e4m3 channels (32 bytes) per step
              const uint32_t off = (kk * 32) >> 4;
              tc_mma_f8(tS + sb * 128, dq + off, dk + off, idS, kk > 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {   // 16 channels per step
              const uint32_t off = ((kk >> 2) * L::kHalfBytes + (kk & 3) * 32) >> 4;
              tc_mma(tS + sb * 128, dq + off, dk + off, idS, kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(bar(B_SFULL0 + sb));
          tc_commit(bar(B_KEMPTY0 + kst));
          if (j == nblk - 1) tc_commit(bar(B_QEMPTY));
          if (++kst == L::kKStages) {
            kst = 0;
            kph ^= 1;
          }
          if (++sb == kSBuf) {
            sb = 0;
            ++su;
          }
        }
      }
      // nothing of ours may still run on the tensor core when TMEM is freed
      tc_commit(bar(B_DRAIN));
      drain_wait(bar(B_DRAIN), 0);
    }
    __syncwarp();
  } else if (warp == kPvWarp0 || warp == kPvWarp1) {
    // ------------------------------------------------------------ PV MMA ---
    if (lane == 0) {
      constexpr uint32_t idPV = idesc_bf16(128, D, 0, 1);
      const uint64_t dv0 = sw128_desc(sbase + L::oV, 8192, 1024);
      int vst = 0;               // V stage of the next PV MMA
      uint32_t vph = 0;
      int sb = 0;                // S buffer holding P of block g
      uint32_t su = 0;
      const int w = warp == kPvWarp0 ? 0 : 1;   // O_w += P_w V_w: keys of tile w of every block
      bool ok = true;
      for (uint32_t it = 0; ok; ++it) {
        const int slot = it & 1;
        if (!wait_bar(bar(B_LFULL0 + slot), (it >> 1) & 1, abort_flag, gerr, prm.wait_ns)) break;
        const ItemInfo inf = info[slot];
        if (inf.end) break;
        mbar_arrive(bar(B_LEMPTY0 + slot));     // the item's info is copied
        const int nblk = (inf.n_entries + 1) >> 1;
        // O is free once the previous item's epilogue has read it
        if (!wait_bar(bar(B_OFREE), (it & 1) ^ 1, abort_flag, gerr, prm.wait_ns)) break;
        if (nblk == 0) tc_commit(bar(B_OFULL));    // nothing to accumulate; the epilogue skips it
        for (int j = 0; j < nblk; ++j) {
          if (!(ok = wait_bar(bar(B_VFULL0 + vst), vph, abort_flag, gerr, prm.wait_ns))) break;
          const uint64_t dv = dv0 + ((vst * L::kVBytes) >> 4);
          if (!(ok = wait_bar(bar(B_PFULL0 + w * kSBuf + sb), su & 1, abort_flag, gerr, prm.wait_ns))) break;
          tc_fence_after();
          const uint32_t pcol = tS + sb * 128 + w * 64;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // 16 keys per step: 8 TMEM columns of P
            const uint32_t boff = (w * (D / 64) * 8192 + kk * 2048) >> 4;
            tc_mma_ts(tO0 + w * 128, pcol + kk * 8, dv + boff, idPV, (j == 0 && kk == 0) ? 0u : 1u);
          }
          tc_commit(bar(B_PDONE0 + sb));
          tc_commit(bar(B_VEMPTY0 + vst));
          if (j == nblk - 1) tc_commit(bar(B_OFULL));
          if (++vst == L::kVStages) {
            vst = 0;
            vph ^= 1;
          }
          if (++sb == kSBuf) {
            sb = 0;
            ++su;
          }
        }
      }
      tc_commit(bar(B_DRAIN));
      drain_wait(bar(B_DRAIN), 0);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
    // ----------------------------------------------------------- softmax ---
    // Warpgroup sg owns key tile sg of every 128-key block (S columns
    // [64 sg, 64 sg + 64)) for all 128 rows (row = TMEM lane) and keeps its own
    // online softmax: running max m, row sum l and partial output O_sg. The
    // two warpgroups never wait for each other inside an item, so one can
    // compute exponentials while the other loads and reduces its scores. The
    // running max is raised only when a tile exceeds it by more than kLazy
    // (log2 units), so P < 2^kLazy and O_sg is rarely rescaled. The epilogue
    // merges the two partial softmaxes of each row.
    const int sg = (warp - 4) >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t my_bit = r < 64 ? 1u : 2u;
    const uint32_t tOw = tO0 + sg * 128 + lane_off;          // my warpgroup's O, my row
    float* xm = reinterpret_cast<float*>(smem + L::oXchg);   // [2 groups][128] row max
    float* xl = xm + 2 * 128;                               // [2 groups][128] row sums
    // logit scale in log2 units; fp8 Q K^T also carries the tiles' dequantisation scales
    float csc = prm.scale_log2;
    uint64_t c2 = f2pack(csc, csc);
    uint32_t g = 0;
    bool ok = true;
    for (uint32_t it = 0; ok; ++it) {
      const int slot = it & 1;
      ok = wait_bar(bar(B_LFULL0 + slot), (it >> 1) & 1, abort_flag, gerr, prm.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      const ItemInfo inf = info[slot];
      if (inf.end) break;
      const uint32_t* list = lists + slot * prm.list_cap;
      const int nblk = (inf.n_entries + 1) >> 1;
      float m = -INFINITY, l = 0.f;
      // my tile's entry of each block, from global memory: loaded one block ahead so that
      // its latency is not on the block's path
      uint32_t e_next = sg < inf.n_entries ? list[sg] : 0u;
      for (int j = 0; j < nblk; ++j, ++g) {
        const uint32_t e = e_next;
        if (j + 1 < nblk) e_next = 2 * j + 2 + sg < inf.n_entries ? list[2 * j + 2 + sg] : 0u;
        const int sbuf = int(g % kSBuf);           // S / P buffer
        const uint32_t sph = (g / kSBuf) & 1;      // its phase
        const uint32_t tSb = tS + sbuf * 128 + lane_off + 64 * sg;
        ok = wait_bar(bar(B_SFULL0 + sbuf), sph, abort_flag, gerr, prm.wait_ns);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        if (prm.hold && g == 0) {   // test hook: wait for a release that nothing gives, until the limit
          ok = wait_bar(bar(B_HOLD), 0, abort_flag, gerr, prm.wait_ns);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        }
        tc_fence_after();
        const int cnt = ((e >> 16) & my_bit) ? int(e >> 24) : 0;   // valid keys of my tile for my row
        float alpha = 1.f;
        uint32_t pk[32];
        if (cnt > 0) {
          float sv[64];
          uint32_t sr[2][32];
          tmem_ld32(tSb, sr[0]);
          tmem_ld32(tSb + 32, sr[1]);
          tmem_wait_ld(sr[0]);
          reg_fence(sr[1]);
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] = __uint_as_float(sr[c >> 5][c & 31]);
          if (cnt < 64) {                          // partial tile: missing keys -> -inf
#pragma unroll
            for (int c = 0; c < 64; ++c) sv[c] = c < cnt ? sv[c] : -INFINITY;
          }
          float mq[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float t = fmax3(sv[16 * q], sv[16 * q + 1], sv[16 * q + 2]);
#pragma unroll
            for (int c = 3; c < 15; c += 2) t = fmax3(t, sv[16 * q + c], sv[16 * q + c + 1]);
            mq[q] = fmaxf(t, sv[16 * q + 15]);
          }
          // raw scores; the scale is positive
          if constexpr (F8) {
            // scale of my query tile (row-half) times the key tile's: fixed for this block
            const int qtile = r < 64 ? inf.qa : inf.qb;
            csc = prm.scale_log2 * prm.q_scale[size_t(inf.bh) * prm.nt_max + (qtile >= 0 ? qtile : inf.qa)] *
                  prm.k_scale[size_t(inf.bh) * prm.nt_max + (e & 0xFFFFu)];
            c2 = f2pack(csc, csc);
          }
          const float bmx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * csc;
          if (bmx > m + kLazy) {                   // also taken when m is still -inf
            alpha = m == -INFINITY ? 1.f : ex2(m - bmx);
            m = bmx;
          }
          const uint64_t nm2 = f2pack(-m, -m);
          uint64_t acc[2] = {0ull, 0ull};
          if (cnt == 64) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float x0, x1, p0, p1;
              f2unpack(ffma2(f2pack(sv[2 * i], sv[2 * i + 1]), c2, nm2), x0, x1);
              constexpr int kPoly = VSA_EXP_POLY_EVERY;
              bool on_fma = false;
              if constexpr (kPoly > 0) on_fma = i % kPoly == kPoly - 1;
              if (on_fma) {
                ex2_fma_pipe(x0, x1, p0, p1);
              } else {
                p0 = ex2(x0);
                p1 = ex2(x1);
              }
              acc[i & 1] = fadd2(acc[i & 1], f2pack(p0, p1));
              pk[i] = bf16x2(p0, p1);
            }
          } else {                                 // partial tile: masked keys give exactly 0
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float x0, x1;
              f2unpack(ffma2(f2pack(sv[2 * i], sv[2 * i + 1]), c2, nm2), x0, x1);
              const float p0 = ex2(x0), p1 = ex2(x1);   // ex2(-inf) = 0
              acc[i & 1] = fadd2(acc[i & 1], f2pack(p0, p1));
              pk[i] = bf16x2(p0, p1);
            }
          }
          float r0, r1;
          f2unpack(fadd2(acc[0], acc[1]), r0, r1);
          l = l * alpha + (r0 + r1);
        } else {                                   // my row-half does not keep this tile
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = 0u;
        }
        // P over the first half of my consumed S columns
        tmem_st32u(tSb, pk);
        // earlier blocks of this item sit in O_sg at the old max: rescale it
        // once the previous block's PV MMAs have finished accumulating
        if (__any_sync(0xffffffffu, j > 0 && alpha != 1.f)) {
          const uint32_t gp = g - 1;
          ok = wait_bar(bar(B_PDONE0 + int(gp % kSBuf)), (gp / kSBuf) & 1, abort_flag, gerr, prm.wait_ns);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            tmem_ld32(tOw + 32 * c, orr);
            tmem_wait_ld(orr);
            float o[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(orr[i]) * alpha;
            tmem_st32(tOw + 32 * c, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(bar(B_PFULL0 + sg * kSBuf + sbuf));
      }
      if (!ok) break;
      // epilogue: both partial outputs are final once the item's last PV is
      // done. Row r's two partial softmaxes (m_0, l_0, O_0) and (m_1, l_1, O_1)
      // merge as O = sum_w 2^(m_w - M) O_w / sum_w 2^(m_w - M) l_w, M = max m_w;
      // warpgroup sg writes channels [sg D/2, (sg+1) D/2).
      ok = wait_bar(bar(B_OFULL), it & 1, abort_flag, gerr, prm.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      xm[sg * 128 + r] = m;
      xl[sg * 128 + r] = l;
      warp_arrive(bar(B_LX));
      ok = wait_bar(bar(B_LX), it & 1, abort_flag, gerr, prm.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      const float m0 = xm[r], m1 = xm[128 + r];
      const float mrow = fmaxf(m0, m1);
      const float a0 = m0 == -INFINITY ? 0.f : ex2(m0 - mrow);
      const float a1 = m1 == -INFINITY ? 0.f : ex2(m1 - mrow);
      const float lrow = xl[r] * a0 + xl[128 + r] * a1;
      const int tile = r < 64 ? inf.qa : inf.qb;
      const int slot_r = r & 63;
      const int rows = r < 64 ? inf.rows_a : inf.rows_b;
      const bool write = tile >= 0 && !inf.bad;
      const bool valid = write && slot_r < rows;
      const float inv = (valid && lrow > 0.f) ? 1.f / lrow : 0.f;
      const float w0 = a0 * inv, w1 = a1 * inv;
      const size_t orow = (size_t(inf.bh) * prm.nt_max + (tile >= 0 ? tile : 0)) * 64 + slot_r;
      uint4* dst = reinterpret_cast<uint4*>(prm.out + orow * D + sg * (D / 2));
      bool store = write;
      if constexpr (DIRECT) {   // token-major O: only the tile's real tokens
        store = valid;
        const int h = inf.bh % prm.heads;
        int tok = 0;
        if (valid) {
          if (tile < dm.n_pre_tiles) {
            tok = prefix_tile_token0(dm, tile) + slot_r;
          } else {
            const int sh = dm.shape_of[h];
            const int pt = dm.shp[sh][0], ph = dm.shp[sh][1], pw = dm.shp[sh][2];
            const int nX = dm.W / pw, nYX = (dm.H / ph) * nX;
            const int v = tile - dm.n_pre_tiles;
            const int ti = v / nYX, yi = (v - ti * nYX) / nX, xi = v - ti * nYX - yi * nX;
            const int st = slot_r / (ph * pw), sy = (slot_r / pw) % ph, sx = slot_r % pw;
            tok = dm.n_pre_tok + ((ti * pt + st) * dm.H + yi * ph + sy) * dm.W + xi * pw + sx;
          }
        }
        dst = reinterpret_cast<uint4*>(prm.out + (size_t(tok) * prm.heads + h) * D + sg * (D / 2));
      }
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t o0[32], o1[32];
        tmem_ld32(tO0 + lane_off + sg * (D / 2) + 32 * c, o0);
        tmem_ld32(tO0 + 128 + lane_off + sg * (D / 2) + 32 * c, o1);
        tmem_wait_ld(o0);
        reg_fence(o1);
        if (store) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              v[i] = __uint_as_float(o0[8 * q + i]) * w0 + __uint_as_float(o1[8 * q + i]) * w1;
            uint4 pkq;
            pkq.x = bf16x2(v[0], v[1]);
            pkq.y = bf16x2(v[2], v[3]);
            pkq.z = bf16x2(v[4], v[5]);
            pkq.w = bf16x2(v[6], v[7]);
            dst[c * 4 + q] = pkq;
          }
        }
      }
      if (write && sg == 0 && prm.lse)
        prm.lse[orow] = valid && lrow > 0.f ? (mrow + __log2f(lrow)) * 0.69314718055994531f : 0.f;
      tc_fence_before();
      warp_arrive(bar(B_OFREE));
      warp_arrive(bar(B_LEMPTY0 + slot));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// --------------------------------------------------------------- host ----

}  // namespace

int attn_smem_bytes(int list_cap) {
  (void)list_cap;   // key lists live in global memory
  static_assert(Smem<64>::oEnd <= Smem<128>::oEnd && Smem<128, true>::oEnd <= Smem<128>::oEnd,
                "the d=64 and fp8 layouts fit the d=128 allocation");
  return 1024 + int(Smem<128>::oEnd);
}

namespace {

AttnParams attn_params(const vsa_plan* p, const int32_t* idx, const int32_t* idx_ref, const int32_t* k, void* op,
                       float* lse, const float* q_scale, const float* k_scale) {
  const Geometry& g = p->geo;
  AttnParams prm;
  prm.q_scale = q_scale;
  prm.k_scale = k_scale;
  prm.idx = idx;
  prm.idx_ref = idx_ref;
  prm.ref_tiles = p->d_ref_tiles;
  prm.prefix_ref = p->d_prefix_ref;
  prm.n_ref = g.n_ref;
  prm.k_ref_max = g.k_ref_max;
  prm.counts = p->d_tile_count;
  prm.items = p->d_items;
  prm.n_items = p->n_items;
  prm.out = static_cast<__nv_bfloat16*>(op);
  prm.lse = lse;
  prm.state = p->d_state;
  prm.heads = g.Hh;
  prm.nt_max = g.nt_max;
  prm.ntv_max = g.ntv_max;
  prm.k_max = g.k_max;
  prm.n_pre = g.n_pre_tiles;
  prm.list_cap = p->list_cap;
  prm.bitmap_words = (p->list_cap / 32) + 2;
  prm.lists = p->d_lists;
  prm.bitmaps = p->d_lists + size_t(p->num_sms) * 2 * p->list_cap;
  prm.scale_log2 = p->desc.softmax_scale * 1.4426950408889634f;
  prm.wait_ns = p->wait_ns;
  prm.hold = p->test_hold;
  for (int h = 0; h < VSA_MAX_HEADS; ++h) {
    prm.ntv[h] = h < g.Hh ? g.ntv[h] : 0;
    prm.k[h] = h < g.Hh ? k[h] : 0;
    prm.k_ref[h] = h < g.Hh ? g.k_ref[h] : 0;
  }
  return prm;
}

// The work counter and pair count reset, then the persistent launch.
template <int D, bool F8, bool DIRECT>
cudaError_t attn_launch(vsa_plan* p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const AttnParams& prm, const DirectMaps& dm, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(p->d_state + 1, 0, 12, s);
  if (e != cudaSuccess) return e;
  const int smem = p->attn_smem_bytes;
  const int grid = int(p->n_items < p->num_sms ? p->n_items : p->num_sms);
  e = cudaFuncSetAttribute(attn_kernel<D, F8, DIRECT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_kernel<D, F8, DIRECT><<<grid, kThreads, smem, s>>>(tq, tk, tv, prm, dm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn(vsa_plan* p, const void* qp, const void* kp, const void* vp, const int32_t* idx,
                        const int32_t* idx_ref, const int32_t* k, void* op, float* lse, cudaStream_t s,
                        const float* q_scale, const float* k_scale) {
  const Geometry& g = p->geo;
  const int64_t rows = int64_t(g.B) * g.Hh * g.nt_max * VSA_TILE;
  const bool f8 = q_scale != nullptr;      // qp, kp are e4m3 tiles with per-tile scales
  if (f8 && g.d != 128) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  const bool maps = f8 ? make_map_u8(&tq, qp, rows, g.d) && make_map_u8(&tk, kp, rows, g.d)
                       : make_map(&tq, qp, rows, g.d) && make_map(&tk, kp, rows, g.d);
  if (!maps || !make_map(&tv, vp, rows, g.d)) return cudaErrorInvalidValue;
  const AttnParams prm = attn_params(p, idx, idx_ref, k, op, lse, q_scale, k_scale);
  static const DirectMaps kNoMaps = {};
  if (f8) return attn_launch<128, true, false>(p, tq, tk, tv, prm, kNoMaps, s);
  if (g.d == 128) return attn_launch<128, false, false>(p, tq, tk, tv, prm, kNoMaps, s);
  return attn_launch<64, false, false>(p, tq, tk, tv, prm, kNoMaps, s);
}

bool direct_attn_supported(const vsa_plan* p) {
  const Geometry& g = p->geo;
  if (g.B != 1 || g.n_ref != 0 || (g.d != 64 && g.d != 128) || g.n_seg > VSA_MAX_SEGMENTS) return false;
  int shapes[kMaxShapes][3], n = 0;
  for (int h = 0; h < g.Hh; ++h) {
    if (g.H % g.ph[h] != 0 || g.W % g.pw[h] != 0) return false;   // tiles partial only along t
    int i = 0;
    while (i < n && !(shapes[i][0] == g.pt[h] && shapes[i][1] == g.ph[h] && shapes[i][2] == g.pw[h])) ++i;
    if (i == n) {
      if (n == kMaxShapes) return false;
      shapes[n][0] = g.pt[h];
      shapes[n][1] = g.ph[h];
      shapes[n][2] = g.pw[h];
      ++n;
    }
  }
  return true;
}

cudaError_t launch_attn_direct(vsa_plan* p, const void* q, const void* k, const void* v, const int32_t* idx,
                               const int32_t* kk, void* o, float* lse, cudaStream_t s) {
  const Geometry& g = p->geo;
  if (!direct_attn_supported(p)) return cudaErrorInvalidValue;
  const cuuint64_t e2 = 2;   // bf16 bytes
  const cuuint64_t D = cuuint64_t(g.d), Hh = cuuint64_t(g.Hh);
  DirectMaps dm = {};
  dm.n_pre_tok = g.n_pre_tok;
  dm.n_pre_tiles = g.n_pre_tiles;
  dm.n_seg = g.n_seg;
  dm.T = g.T;
  dm.H = g.H;
  dm.W = g.W;
  for (int i = 0; i <= VSA_MAX_SEGMENTS; ++i) {
    dm.seg_tok0[i] = g.seg_tok0[i];
    dm.seg_tile0[i] = g.seg_tile0[i];
  }
  const void* base[3] = {q, k, v};
  int n = 0;
  for (int h = 0; h < g.Hh; ++h) {
    int i = 0;
    while (i < n && !(dm.shp[i][0] == g.pt[h] && dm.shp[i][1] == g.ph[h] && dm.shp[i][2] == g.pw[h])) ++i;
    if (i == n) {
      dm.shp[n][0] = g.pt[h];
      dm.shp[n][1] = g.ph[h];
      dm.shp[n][2] = g.pw[h];
      // the video grid [T][H][W][heads][d] of each tensor, boxes of one tile of this shape
      const cuuint64_t dims[5] = {D, Hh, cuuint64_t(g.W), cuuint64_t(g.H), cuuint64_t(g.T)};
      const cuuint64_t strides[4] = {D * e2, Hh * D * e2, cuuint64_t(g.W) * Hh * D * e2,
                                     cuuint64_t(g.H) * g.W * Hh * D * e2};
      const cuuint32_t box[5] = {64, 1, cuuint32_t(g.pw[h]), cuuint32_t(g.ph[h]), cuuint32_t(g.pt[h])};
      for (int m = 0; m < 3; ++m) {
        const char* vb = static_cast<const char*>(base[m]) + size_t(g.n_pre_tok) * Hh * D * e2;
        if (!make_map_nd(&dm.vid[n][m], vb, 5, dims, strides, box)) return cudaErrorInvalidValue;
      }
      ++n;
    }
    dm.shape_of[h] = int8_t(i);
  }
  {  // the whole sequence [N][heads][d], boxes of 64 tokens (prefix tiles)
    const cuuint64_t dims[3] = {D, Hh, cuuint64_t(g.n_tokens)};
    const cuuint64_t strides[2] = {D * e2, Hh * D * e2};
    const cuuint32_t box[3] = {64, 1, 64};
    for (int m = 0; m < 3; ++m)
      if (!make_map_nd(&dm.pre[m], base[m], 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const AttnParams prm = attn_params(p, idx, nullptr, kk, o, lse, nullptr, nullptr);
  if (g.d == 128) return attn_launch<128, false, true>(p, dm.pre[0], dm.pre[1], dm.pre[2], prm, dm, s);
  return attn_launch<64, false, true>(p, dm.pre[0], dm.pre[1], dm.pre[2], prm, dm, s);
}

}  // namespace vsa
