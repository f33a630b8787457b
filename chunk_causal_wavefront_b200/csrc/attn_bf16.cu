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
//   warp 8 (one lane)  TMA producer: Q0, Q1 once, then for every key tile (one
//                      128-token page, found through the page table) K and V
//                      into a two-stage shared-memory ring (128-byte swizzle).
//   warp 9 (one lane)  tcgen05 issuer, in the order
//                        S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
//                      S_q = Q_q K^T goes to TMEM columns [128q, 128q+128);
//                      PV_q reads P_q from TMEM (the first 64 columns of S_q,
//                      bf16 pairs) and accumulates O_q in columns 256 + 128q.
//                      While softmax q works on S_q(j+1), the tensor pipe runs
//                      the other tile's P*V and S (ping-pong).
//   warps 0-3 / 4-7    softmax of tile 0 / tile 1: thread r owns query row r
//                      (TMEM lane r); row max and sum are thread-local over its
//                      128 columns; P is rounded to bf16 and stored back into
//                      TMEM; O is rescaled in TMEM only when the running max
//                      grows by more than 2^8 (the exponentials stay <= 256
//                      otherwise), which is the only time softmax waits for the
//                      previous P*V. The epilogue divides by the row sum, stages
//                      the bf16 rows in the tile's (now idle) Q buffer and each
//                      warp writes its 32 rows with a TMA store that clips rows
//                      past C.
// Every wait is bounded: on timeout the CTA records WF_ERR_TIMEOUT, the other
// roles see the abort flag, in-flight copies and MMAs are drained and TMEM is
// freed before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include "f32x2.cuh"
#include "pipeline.cuh"
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
// Warpgroups 0 and 1 run the softmax of tiles 0 and 1; warpgroup 2 holds the
// TMA producer (warp 8) and the MMA issuer (warp 9); warps 10-11 only hand
// their registers over. Launched at 168 registers per thread (384 x 168 =
// 64512), warpgroup 2 moves to 96 and the softmax warpgroups to 200:
// 256 x 200 + 128 x 96 = 63488.
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kRegsSoftmax = 200;
constexpr uint32_t kRegsControl = 96;
static_assert(256 * kRegsSoftmax + 128 * kRegsControl <= 384 * 168, "register split");

// TMEM columns.
constexpr uint32_t kTmemS = 0;        // S_q at 128 q; P_q aliases its first 64 columns
constexpr uint32_t kTmemO = 256;      // O_q at 256 + 128 q

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t kOffQ = 0;                       // Q0, Q1
constexpr uint32_t kOffK = kOffQ + 2 * kTile;       // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;       // 2 stages
constexpr uint32_t kOffBar = kOffV + 2 * kTile;
constexpr int kNumBars = 16;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kOffPages = kOffMisc + 64;
constexpr uint32_t kSmemBytes = kOffPages + kPageCache * 4 + 1024;   // + alignment slack

enum Bar {
  kQFull = 0, kKFull0 = 1, kKEmpty0 = 3, kVFull0 = 5, kVEmpty0 = 7,
  kSFull0 = 9, kPReady0 = 11, kPVDone0 = 13, kDrain = 15
};

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

// S_q = Q_q K(stage)^T: 8 k-steps of 16 along d; Q and K are [128][128] bf16
// tiles stored as two 64-column 128-byte-swizzled halves.
__device__ __forceinline__ void issue_s(uint32_t tmem_s, uint32_t q_lo, uint32_t k_lo,
                                        uint32_t hi) {
  constexpr uint32_t idS = make_idesc_bf16(kBM, kBN, false);
#pragma unroll
  for (int k = 0; k < kHD / 16; ++k) {
    const uint32_t off = ((k >> 2) * kHalf + (k & 3) * 32) >> 4;
    mma_bf16_ss2(tmem_s, q_lo + off, k_lo + off, hi, idS, k > 0);
  }
}

// O_q (+)= P_q V(stage): 8 k-steps of 16 keys; P_q is read from TMEM (8
// columns of bf16 pairs per step), V is MN-major in shared memory.
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_lo,
                                         uint32_t hi, bool accumulate_first) {
  constexpr uint32_t idPV = make_idesc_bf16(kBM, kHD, true);
#pragma unroll
  for (int k = 0; k < kBN / 16; ++k) {
    mma_bf16_ts2(tmem_o, tmem_p + k * 8, v_lo + ((k * 2048) >> 4), hi, idPV,
                 (accumulate_first || k > 0) ? 1u : 0u);
  }
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
        // p_ready: one elected arrival per softmax warp of the tile
        const bool softmax_arrives = b == kPReady0 || b == kPReady0 + 1;
        mbar_init(bars + b, softmax_arrives ? kBM / 32 : 1);
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

  if (warp >= 8) {
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
      int nk0 = 0, nk1 = 0, nv0 = 0, nv1 = 0;   // loads issued per stage
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
        if (stg) ++nk1; else ++nk0;
        if (!wait_bar(ctx, kVEmpty0 + stg, ph ^ 1)) break;
        mbar_arrive_expect_tx(bars + kVFull0 + stg, kTile);
        tma_load_2d(sV, &tkv, bars + kVFull0 + stg, 0, rowv);
        tma_load_2d(sV + kHalf, &tkv, bars + kVFull0 + stg, 64, rowv);
        if (stg) ++nv1; else ++nv0;
      }
      // Drain: every load this thread issued has landed before the CTA exits.
      if (nk0) drain_wait(ctx, kKFull0, (nk0 - 1) & 1);
      if (nk1) drain_wait(ctx, kKFull0 + 1, (nk1 - 1) & 1);
      if (nv0) drain_wait(ctx, kVFull0, (nv0 - 1) & 1);
      if (nv1) drain_wait(ctx, kVFull0 + 1, (nv1 - 1) & 1);
      drain_wait(ctx, kQFull, 0);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      // Descriptor words: the high word (stride 1 KB, version, swizzle) is the
      // same for Q, K and V; a k-step or a stage only moves the low word.
      const uint32_t hi = desc_hi_sw128(1024);
      const uint32_t q_lo = desc_lo_sw128(smem_u32(smem + kOffQ), 16);
      const uint32_t k_lo = desc_lo_sw128(smem_u32(smem + kOffK), 16);
      const uint32_t v_lo = desc_lo_sw128(smem_u32(smem + kOffV), kHalf);
      constexpr uint32_t kTileStep = kTile >> 4;
      bool ok = wait_bar(ctx, kQFull, 0) && wait_bar(ctx, kKFull0, 0);
      if (ok) {
        tc_fence_after();
        issue_s(tmem + kTmemS, q_lo, k_lo, hi);
        mma_commit(bars + kSFull0);
        if (has_q1) {
          issue_s(tmem + kTmemS + 128, q_lo + kTileStep, k_lo, hi);
          mma_commit(bars + kSFull0 + 1);
        }
        mma_commit(bars + kKEmpty0);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int stg = j & 1, nstg = (j + 1) & 1;
        const bool more = j + 1 < n_tiles;
        if (!wait_bar(ctx, kVFull0 + stg, (j >> 1) & 1)) break;
        if (!wait_bar(ctx, kPReady0, j & 1)) break;
        tc_fence_after();
        issue_pv(tmem + kTmemO, tmem + kTmemS, v_lo + stg * kTileStep, hi, j > 0);
        mma_commit(bars + kPVDone0);
        if (more) {
          if (!wait_bar(ctx, kKFull0 + nstg, ((j + 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_s(tmem + kTmemS, q_lo, k_lo + nstg * kTileStep, hi);
          mma_commit(bars + kSFull0);
        }
        if (has_q1) {
          if (!wait_bar(ctx, kPReady0 + 1, j & 1)) break;
          tc_fence_after();
          issue_pv(tmem + kTmemO + 128, tmem + kTmemS + 128, v_lo + stg * kTileStep, hi, j > 0);
          mma_commit(bars + kPVDone0 + 1);
          if (more) {
            issue_s(tmem + kTmemS + 128, q_lo + kTileStep, k_lo + nstg * kTileStep, hi);
            mma_commit(bars + kSFull0 + 1);
          }
        }
        mma_commit(bars + kVEmpty0 + stg);
        if (more) mma_commit(bars + kKEmpty0 + nstg);
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      mma_commit(bars + kDrain);
      drain_wait(ctx, kDrain, 0);
    }
   }
  } else {
   setmaxnreg_inc<kRegsSoftmax>();
   if (warp < 4 || has_q1) {
    // ------------------------------------------------------------- softmax --
    const int q = warp >> 2;
    const int r = (warp & 3) * 32 + lane;               // query row == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + kTmemS + q * 128;
    const uint32_t tO = tmem + lane_addr + kTmemO + q * 128;
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = __all_sync(0xffffffffu, wait_bar(ctx, kSFull0 + q, j & 1));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, s + c * 32);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence32(s + c * 32);

      const int valid = (j % p.npc == p.npc - 1) ? last_valid : kBN;
      if (valid < kBN) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) s[c] = __float_as_uint(-INFINITY);
      }
      // Row max: eight independent chains of three-input max, then a tree.
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float a = max3(__uint_as_float(s[i]), __uint_as_float(s[i + 8]), __uint_as_float(s[i + 16]));
#pragma unroll
        for (int b = 24; b < 120; b += 16)
          a = max3(a, __uint_as_float(s[b + i]), __uint_as_float(s[b + 8 + i]));
        m8[i] = fmaxf(a, __uint_as_float(s[120 + i]));
      }
      const float mx = fmaxf(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], max3(m8[5], m8[6], m8[7])));
      const float m_new = fmaxf(m, mx * p.scale_log2);
      const bool rescale = m_new - m > 8.0f;             // always true on the first tile
      const float alpha = rescale ? ex2(m - m_new) : 1.0f;
      const float m_use = rescale ? m_new : m;
      // P = 2^(s * log2(e) / sqrt(d) - m) on the MUFU unit, the scale-subtract
      // and the row sums in packed f32x2 arithmetic; rounded to bf16 pairs and
      // streamed back into the first 64 columns of S_q, 16 columns (32 keys) at
      // a time.
      const uint64_t sc2 = f2(p.scale_log2, p.scale_log2), nm2 = f2(-m_use, -m_use);
      uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
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
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
          reg_fence32(o);
          const uint64_t a2 = f2(alpha, alpha);
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
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + kPReady0 + q);
    }
    if (ok && n_tiles > 0) {
      ok = __all_sync(0xffffffffu, wait_bar(ctx, kPVDone0 + q, (n_tiles - 1) & 1));
    }
    if (ok && n_tiles > 0) {
      tc_fence_after();
      const float inv = 1.0f / l;
      // Stage the bf16 rows in this tile's Q buffer (its last reader, the final
      // S MMA, has completed) in the 128-byte swizzled layout of the output
      // tensor map, whose box is 32 rows: 16-byte chunk c of row r in 64-column
      // half kt lands at kt * 16 KB + r * 128 + ((c ^ (r & 7)) * 16), so each
      // warp's 32 rows form one contiguous 4 KB box per half and the warp
      // stores them itself (no cross-warp barrier).
      uint8_t *stage = smem + kOffQ + q * kTile;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t o[32];
        tmem_ld32(tO + c4 * 32, o);
        tmem_ld_wait();
        reg_fence32(o);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int cc = c4 * 4 + i;                      // 16-byte chunk 0..15 of the row
          const int kt = cc >> 3, c = cc & 7;
          const uint32_t addr = smem_u32(stage + kt * kHalf + r * 128 + ((c ^ (r & 7)) << 4));
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[4 * i]),
                       "r"(w[4 * i + 1]), "r"(w[4 * i + 2]), "r"(w[4 * i + 3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int wr = (warp & 3) * 32;                     // this warp's first row in the tile
      if (lane == 0 && row0 + q * kBM + wr < p.C) {       // boxes wholly past C are skipped
        tma_store_4d(&tout, stage + wr * 128, 0, h, row0 + q * kBM + wr, slot);
        tma_store_4d(&tout, stage + kHalf + wr * 128, 64, h, row0 + q * kBM + wr, slot);
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
