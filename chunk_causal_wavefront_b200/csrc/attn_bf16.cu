// Round attention, bf16 tensor-core path for sm_100a (tcgen05 + TMEM + TMA).
//
// "Wave Forcing: Towards Speed-of-Light Streaming Video Generation", Method
// section: full attention inside each chunk, chunk-wise causal attention across
// chunks with M_WF(s, j) = 1[j >= s]; the ordered context of "Como funciona"
// (anchor || history || store || denoising K/V) makes the keys of query slot s
// a prefix of the context, so masked (s, j) chunk pairs are never visited: the
// key loop stops at the slot's own chunk.
//
// One CTA computes O = softmax(Q K^T / sqrt(d)) V for two 128-row query tiles
// (q = 0, 1) of one (slot, head), sharing every K/V page it loads:
//   warp 16 (one lane) TMA producer: Q0, Q1 once, then for every key tile (one
//                      128-token page, found through the page table) K and V
//                      into a two-stage shared-memory ring (128-byte swizzle).
//   warp 17 (one lane) tcgen05 issuer, in the order
//                        S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
//                      S_q = Q_q K^T goes to TMEM columns [128q, 128q+128);
//                      PV_q reads P_q from TMEM (bf16 pairs written over S_q:
//                      keys 0-63 in columns 0-31, keys 64-127 in columns 64-95)
//                      and accumulates O_q in columns 256 + 128q. While the
//                      softmax of tile q works on S_q(j+1), the tensor pipe runs
//                      the other tile's P*V and S (ping-pong).
//   warps 0-15         softmax, four warpgroups: tile q = wg / 2, column half
//                      hf = wg % 2. A query row (TMEM lane) is shared by two
//                      warps, one per 64-column half: each takes the max of its
//                      half, the two exchange it through shared memory (an
//                      mbarrier of 64 arrivals, so every wait stays bounded),
//                      then each computes its half of P, rounds it to bf16 into
//                      TMEM, keeps its half of the row sum and owns its half of
//                      O. O is rescaled only when the running max grows by more
//                      than 2^8 (the exponentials stay <= 256 otherwise). The
//                      epilogue adds the two half sums, divides, stages the bf16
//                      half rows in the tile's (now idle) Q buffer and each warp
//                      writes its 32 x 64 box with a TMA store that clips rows
//                      past C.
// Every wait is bounded: on timeout the CTA records WF_ERR_TIMEOUT, the other
// roles see the abort flag, in-flight copies and MMAs are drained and TMEM is
// freed before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include "f32x2.cuh"
#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {
namespace {

using namespace sm100;

constexpr int kBM = 128;              // query rows per tile
constexpr int kBN = 128;              // keys per tile (one page)
constexpr int kHD = 128;              // head dim
constexpr uint32_t kHalf = 16384;     // one [128 rows][64 cols] bf16 swizzled block
constexpr uint32_t kTile = 2 * kHalf; // [128][128] bf16
constexpr int kPageCache = 1024;      // page ids cached in shared memory
// Warpgroups 0-3 run the softmax (tile, column half); warpgroup 4 holds the
// TMA producer (warp 16) and the MMA issuer (warp 17); warps 18-19 only hand
// their registers over. Launched at 96 registers per thread (640 x 96 =
// 61440), warpgroup 4 drops to 56 and the softmax warpgroups rise to 104:
// 512 x 104 + 128 x 56 = 60416.
constexpr int kThreads = 640;
constexpr int kSoftmaxWarps = 16;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr uint32_t kRegsSoftmax = 104;
constexpr uint32_t kRegsControl = 56;
static_assert(512 * kRegsSoftmax + 128 * kRegsControl <= 640 * 96, "register split");
constexpr long long kWaitLimit = 2000000000LL;  // ~1 s at 2 GHz

// TMEM columns.
constexpr uint32_t kTmemS = 0;        // S_q at 128 q; P_q aliases its first 64 columns
constexpr uint32_t kTmemO = 256;      // O_q at 256 + 128 q

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t kOffQ = 0;                       // Q0, Q1
constexpr uint32_t kOffK = kOffQ + 2 * kTile;       // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;       // 2 stages
constexpr uint32_t kOffBar = kOffV + 2 * kTile;
constexpr int kNumBars = 24;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kOffXchg = kOffMisc + 64;                 // [2 parity][2 q][2 half][128] f32
constexpr uint32_t kOffPages = kOffXchg + 2 * 2 * 2 * 128 * 4;
constexpr uint32_t kSmemBytes = kOffPages + kPageCache * 4 + 1024;   // + alignment slack

enum Bar {
  kQFull = 0, kKFull0 = 1, kKEmpty0 = 3, kVFull0 = 5, kVEmpty0 = 7,
  kSFull0 = 9, kPReady0 = 11, kPVDone0 = 13, kDrain = 15,
  kXchg0 = 16   // 8 barriers: (tile q, TMEM lane quadrant) pairs of softmax warps
};

struct Ctx {
  uint64_t *bars;
  volatile int *abort;
  int32_t *status;
};

// Bounded wait on an mbarrier phase. Returns false (and flags the CTA) on
// timeout or when another role has already aborted.
__device__ __forceinline__ bool wait_bar(const Ctx &c, int b, uint32_t parity) {
  uint64_t *bar = c.bars + b;
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 127u) == 0) {
      if (*c.abort) return false;
      if (clock64() - t0 > kWaitLimit) {
        *c.abort = 1;
        record_status(c.status, WF_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Time-bounded wait used while draining (ignores the abort flag).
__device__ __forceinline__ void drain_wait(const Ctx &c, int b, uint32_t parity) {
  uint64_t *bar = c.bars + b;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimit) {
      record_status(c.status, WF_ERR_TIMEOUT);
      return;
    }
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);   // RNE, lo in the low half
  return *reinterpret_cast<uint32_t *>(&b);
}

// Keep the compiler from using tcgen05.ld results before tcgen05.wait::ld.
#define WF_REG_FENCE8(r, o)                                                                 \
  asm volatile("" : "+r"(r[o + 0]), "+r"(r[o + 1]), "+r"(r[o + 2]), "+r"(r[o + 3]),         \
               "+r"(r[o + 4]), "+r"(r[o + 5]), "+r"(r[o + 6]), "+r"(r[o + 7]))

__device__ __forceinline__ void reg_fence32(uint32_t *r) {
  WF_REG_FENCE8(r, 0);
  WF_REG_FENCE8(r, 8);
  WF_REG_FENCE8(r, 16);
  WF_REG_FENCE8(r, 24);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_bf16_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tq,
                     const __grid_constant__ CUtensorMap tkv,
                     const __grid_constant__ CUtensorMap tout) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
  int32_t *page_cache = reinterpret_cast<int32_t *>(smem + kOffPages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: head-major; inside a head, slots in decreasing context length
  // (slot 0 first: longest first), then pairs of query tiles.
  const int tiles = (p.C + kBM - 1) / kBM;
  const int pairs = (tiles + 1) / 2;
  const int per_head = p.live.n * pairs;
  const int h = blockIdx.x / per_head;
  const int rem = blockIdx.x - h * per_head;
  const int li = p.live.n - 1 - rem / pairs;
  const int pair = rem % pairs;
  const int slot = p.live.slot[li];
  const int npos = p.live.npos[li];
  const int row0 = pair * 2 * kBM;
  const bool has_q1 = 2 * pair + 1 < tiles;

  // Readiness + bounds check of the whole round's context (so that a stale
  // page stops every CTA of the launch), caching the page ids.
  {
    int bad = 0, stale = 0;
    const int total = p.n_pos * p.npc;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
      const int pos = i / p.npc;
      const int pg = __ldcg(p.table + kTabPages + i);
      if (pg < 0 || pg >= p.num_pages) bad = 1;
      else if (__ldcg(p.tags + pg) != __ldcg(p.table + kTabPosTag + pos)) stale = 1;
      if (i < kPageCache) page_cache[i] = pg;
    }
    if (threadIdx.x == 0) {
      *abort_flag = 0;
      for (int b = 0; b < kNumBars; ++b) {
        uint32_t count = 1;
        if (b == kPReady0 || b == kPReady0 + 1) count = 2 * kBM;   // both column halves
        if (b >= kXchg0) count = 64;                               // the two warps of a pair
        mbar_init(bars + b, count);
      }
      fence_barrier_init();
    }
    const int any_bad = __syncthreads_or(bad);
    const int any_stale = __syncthreads_or(stale);
    if (any_bad || any_stale) {
      if (threadIdx.x == 0) record_status(p.status, any_bad ? WF_ERR_BAD_PAGE : WF_ERR_NOT_READY);
      return;
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Ctx ctx{bars, abort_flag, p.status};
  const int n_tiles = npos * p.npc;
  const int last_valid = p.C - (p.npc - 1) * p.P;   // keys in a chunk's last page

  if (warp >= kSoftmaxWarps) {
   setmaxnreg_dec<kRegsControl>();
   if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tkv);
      tma_prefetch_desc(&tout);
      uint8_t *sQ = smem + kOffQ;
      mbar_arrive_expect_tx(bars + kQFull, has_q1 ? 2 * kTile : kTile);
      tma_load_4d(sQ, &tq, bars + kQFull, 0, h, row0, slot);
      tma_load_4d(sQ + kHalf, &tq, bars + kQFull, 64, h, row0, slot);
      if (has_q1) {
        tma_load_4d(sQ + kTile, &tq, bars + kQFull, 0, h, row0 + kBM, slot);
        tma_load_4d(sQ + kTile + kHalf, &tq, bars + kQFull, 64, h, row0 + kBM, slot);
      }
      int nk[2] = {0, 0}, nv[2] = {0, 0};
      for (int j = 0; j < n_tiles; ++j) {
        const int stg = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int phys = j < kPageCache ? page_cache[j] : __ldcg(p.table + kTabPages + j);
        const int rowk = static_cast<int>(p.layer_row0) + ((phys * 2) * p.Hh + h) * p.P;
        const int rowv = rowk + p.Hh * p.P;
        uint8_t *sK = smem + kOffK + stg * kTile;
        uint8_t *sV = smem + kOffV + stg * kTile;
        if (!wait_bar(ctx, kKEmpty0 + stg, ph ^ 1)) break;
        mbar_arrive_expect_tx(bars + kKFull0 + stg, kTile);
        tma_load_2d(sK, &tkv, bars + kKFull0 + stg, 0, rowk);
        tma_load_2d(sK + kHalf, &tkv, bars + kKFull0 + stg, 64, rowk);
        ++nk[stg];
        if (!wait_bar(ctx, kVEmpty0 + stg, ph ^ 1)) break;
        mbar_arrive_expect_tx(bars + kVFull0 + stg, kTile);
        tma_load_2d(sV, &tkv, bars + kVFull0 + stg, 0, rowv);
        tma_load_2d(sV + kHalf, &tkv, bars + kVFull0 + stg, 64, rowv);
        ++nv[stg];
      }
      // Drain: every load this thread issued has landed before the CTA exits.
      for (int s = 0; s < 2; ++s) {
        if (nk[s]) drain_wait(ctx, kKFull0 + s, (nk[s] - 1) & 1);
        if (nv[s]) drain_wait(ctx, kVFull0 + s, (nv[s] - 1) & 1);
      }
      drain_wait(ctx, kQFull, 0);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idS = make_idesc_bf16(kBM, kBN, false);
      constexpr uint32_t idPV = make_idesc_bf16(kBM, kHD, true);
      const uint32_t aQ = smem_u32(smem + kOffQ);
      auto issue_s = [&](int q, int j) {
        const uint32_t aK = smem_u32(smem + kOffK + (j & 1) * kTile);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k) {
          const uint32_t off = (k >> 2) * kHalf + (k & 3) * 32;
          mma_bf16_ss(tmem + kTmemS + q * 128, make_desc_sw128(aQ + q * kTile + off, 16, 1024),
                      make_desc_sw128(aK + off, 16, 1024), idS, k > 0);
        }
        mma_commit(bars + kSFull0 + q);
      };
      auto issue_pv = [&](int q, int j) {
        const uint32_t aV = smem_u32(smem + kOffV + (j & 1) * kTile);
#pragma unroll
        for (int k = 0; k < kBN / 16; ++k) {
          // A = P_q from TMEM: 16 keys = 8 columns of bf16 pairs per step; keys
          // 64-127 sit 64 columns further (each column half writes its own P).
          mma_bf16_ts(tmem + kTmemO + q * 128,
                      tmem + kTmemS + q * 128 + (k < 4 ? k * 8 : 64 + (k - 4) * 8),
                      make_desc_sw128(aV + k * 2048, kHalf, 1024), idPV,
                      (j > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(bars + kPVDone0 + q);
      };
      bool ok = wait_bar(ctx, kQFull, 0) && wait_bar(ctx, kKFull0, 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if (has_q1) issue_s(1, 0);
        mma_commit(bars + kKEmpty0);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int stg = j & 1;
        const bool more = j + 1 < n_tiles;
        if (!wait_bar(ctx, kVFull0 + stg, (j >> 1) & 1)) break;
        if (!wait_bar(ctx, kPReady0, j & 1)) break;
        tc_fence_after();
        issue_pv(0, j);
        if (more) {
          if (!wait_bar(ctx, kKFull0 + ((j + 1) & 1), ((j + 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (has_q1) {
          if (!wait_bar(ctx, kPReady0 + 1, j & 1)) break;
          tc_fence_after();
          issue_pv(1, j);
          if (more) issue_s(1, j + 1);
        }
        mma_commit(bars + kVEmpty0 + stg);
        if (more) mma_commit(bars + kKEmpty0 + ((j + 1) & 1));
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      mma_commit(bars + kDrain);
      drain_wait(ctx, kDrain, 0);
    }
   }
  } else {
   setmaxnreg_inc<kRegsSoftmax>();
   const int wg = warp >> 2;
   const int q = wg >> 1, hf = wg & 1;
   if (q == 0 || has_q1) {
    // ------------------------------------------------------------- softmax --
    const int quad = warp & 3;
    const int r = quad * 32 + lane;                      // query row == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_addr + kTmemS + q * 128 + hf * 64;   // this half's S
    const uint32_t tO = tmem + lane_addr + kTmemO + q * 128 + hf * 64;   // this half's O
    float *xchg = reinterpret_cast<float *>(smem + kOffXchg);
    const int xbar = kXchg0 + q * 4 + quad;
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = __all_sync(0xffffffffu, wait_bar(ctx, kSFull0 + q, j & 1));
      uint32_t s[64];
      float mx = -INFINITY;
      if (ok) {
        tc_fence_after();
        tmem_ld32(tS, s);
        tmem_ld32(tS + 32, s + 32);
        tmem_ld_wait();
        reg_fence32(s);
        reg_fence32(s + 32);
        const int valid = (j % p.npc == p.npc - 1) ? last_valid - hf * 64 : 64;
        if (valid < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= valid) s[c] = __float_as_uint(-INFINITY);
        }
        // Max of this half: eight chains of three-input max, then a tree.
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float a = max3(__uint_as_float(s[i]), __uint_as_float(s[i + 8]), __uint_as_float(s[i + 16]));
          a = max3(a, __uint_as_float(s[i + 24]), __uint_as_float(s[i + 32]));
          a = max3(a, __uint_as_float(s[i + 40]), __uint_as_float(s[i + 48]));
          m8[i] = fmaxf(a, __uint_as_float(s[i + 56]));
        }
        mx = fmaxf(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], max3(m8[5], m8[6], m8[7])));
      }
      // Exchange the half maxima (and whether this warp is still running) with
      // the partner warp; both halves then take the same decisions.
      float *slot_self = xchg + (((j & 1) * 2 + q) * 2 + hf) * 128;
      float *slot_other = xchg + (((j & 1) * 2 + q) * 2 + (hf ^ 1)) * 128;
      slot_self[r] = ok ? mx : __int_as_float(0x7fc00000);   // NaN = partner stopped
      mbar_arrive(bars + xbar);
      ok = __all_sync(0xffffffffu, ok && wait_bar(ctx, xbar, j & 1));
      if (!ok) break;
      const float mo = slot_other[r];
      ok = __all_sync(0xffffffffu, !isnan(mo));
      if (!ok) break;
      const float m_new = fmaxf(m, fmaxf(mx, mo) * p.scale_log2);
      const bool rescale = m_new - m > 8.0f;             // always true on the first tile
      const float alpha = rescale ? ex2(m - m_new) : 1.0f;
      const float m_use = rescale ? m_new : m;
      // P = 2^(s * log2(e) / sqrt(d) - m) on the MUFU unit, the scale-subtract
      // and the row sums in packed f32x2 arithmetic; rounded to bf16 pairs and
      // stored over the first 32 columns of this half's S.
      const uint64_t sc2 = f2(p.scale_log2, p.scale_log2), nm2 = f2(-m_use, -m_use);
      uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t pw[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int k0 = cc * 32 + 2 * c;
          const uint64_t x2 = ffma2(f2(__uint_as_float(s[k0]), __uint_as_float(s[k0 + 1])), sc2, nm2);
          float a, b;
          unf2(x2, a, b);
          const float e0 = ex2(a), e1 = ex2(b);
          acc[c & 3] = fadd2(acc[c & 3], f2(e0, e1));
          pw[c] = pack_bf16(e0, e1);
        }
        tmem_st16(tS + cc * 16, pw);
      }
      float sum0, sum1;
      unf2(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), sum0, sum1);
      l = l * alpha + (sum0 + sum1);
      m = m_use;

      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
        // O_q must hold P*V up to tile j-1 before it is rescaled.
        ok = __all_sync(0xffffffffu, wait_bar(ctx, kPVDone0 + q, (j - 1) & 1));
        if (!ok) break;
        tc_fence_after();
        const uint64_t a2 = f2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
          reg_fence32(o);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const uint64_t v = fmul2(f2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2);
            float lo, hi;
            unf2(v, lo, hi);
            o[i] = __float_as_uint(lo);
            o[i + 1] = __float_as_uint(hi);
          }
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars + kPReady0 + q);
    }
    // Epilogue: add the two half sums (one more exchange), wait for the last
    // P*V, divide and store this half of the rows.
    if (ok && n_tiles > 0) {
      ok = __all_sync(0xffffffffu, wait_bar(ctx, kPVDone0 + q, (n_tiles - 1) & 1));
    }
    {
      const int j = n_tiles;
      float *slot_self = xchg + (((j & 1) * 2 + q) * 2 + hf) * 128;
      float *slot_other = xchg + (((j & 1) * 2 + q) * 2 + (hf ^ 1)) * 128;
      slot_self[r] = ok ? l : __int_as_float(0x7fc00000);
      mbar_arrive(bars + xbar);
      ok = __all_sync(0xffffffffu, ok && wait_bar(ctx, xbar, j & 1));
      const float lo = ok ? slot_other[r] : 0.0f;
      ok = __all_sync(0xffffffffu, ok && !isnan(lo));
      l += lo;
    }
    if (ok && n_tiles > 0) {
      tc_fence_after();
      const float inv = 1.0f / l;
      // Stage this half (64 columns = one 128-byte swizzled block of the output
      // tensor map) in the tile's Q buffer, whose last reader, the final S MMA,
      // has completed: 16-byte chunk c of row r lands at hf * 16 KB + r * 128 +
      // ((c ^ (r & 7)) * 16), so each warp's 32 rows form one contiguous 4 KB
      // box and the warp stores it itself.
      uint8_t *stage = smem + kOffQ + q * kTile + hf * kHalf;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t o[32];
        tmem_ld32(tO + c2 * 32, o);
        tmem_ld_wait();
        reg_fence32(o);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = c2 * 4 + i;                       // 16-byte chunk 0..7 of the half row
          const uint32_t addr = smem_u32(stage + r * 128 + ((c ^ (r & 7)) << 4));
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[4 * i]),
                       "r"(w[4 * i + 1]), "r"(w[4 * i + 2]), "r"(w[4 * i + 3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int wr = quad * 32;                           // this warp's first row in the tile
      if (lane == 0 && row0 + q * kBM + wr < p.C) {       // boxes wholly past C are skipped
        tma_store_4d(&tout, stage + wr * 128, hf * 64, h, row0 + q * kBM + wr, slot);
        tma_store_commit();
        tma_store_wait_all();
      }
      __syncwarp();
    }
   }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_attention_bf16(const AttnParams &p, const void *tmap_q, const void *tmap_kv,
                                  const void *tmap_out, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  if (p.d != kHD || p.P != kBN) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int tiles = (p.C + kBM - 1) / kBM;
  const int64_t blocks = static_cast<int64_t>((tiles + 1) / 2) * p.live.n * p.Hh;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  attn_bf16_kernel<<<static_cast<unsigned>(blocks), kThreads, kSmemBytes, st>>>(
      p, *static_cast<const CUtensorMap *>(tmap_q), *static_cast<const CUtensorMap *>(tmap_kv),
      *static_cast<const CUtensorMap *>(tmap_out));
  return cudaGetLastError();
}

}  // namespace wf
