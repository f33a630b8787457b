// Round attention on the 5th-generation tensor cores for sm_100a (tcgen05 +
// TMEM + TMA), for bf16 pools and for FP8 (E4M3) pools.
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
//   warp 8 (one lane)  TMA producer of Q0, Q1 (once) and, for every key tile
//                      (one 128-token page, found through the page table), K
//                      into a shared-memory ring (128-byte swizzle; two stages
//                      for bf16, three for E4M3).
//   warp 10 (one lane) TMA producer of V into a ring of the same depth, apart
//                      from K so that no K load queues behind a V load.
//   warp 9 (one lane)  tcgen05 issuer, in the order
//                        S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
//                      S_q = Q_q K^T goes to TMEM columns [128q, 128q+128);
//                      PV_q reads P_q from TMEM (the first columns of S_q) and
//                      accumulates O_q in columns 256 + 128q. While softmax q
//                      works on S_q(j+1), the tensor pipe runs the other
//                      tile's P*V and S (ping-pong).
//   warps 0-3 / 4-7    softmax of tile 0 / tile 1: thread r owns query row r
//                      (TMEM lane r); row max and sum are thread-local over its
//                      128 columns; P is rounded to the operand format and
//                      stored back into TMEM; O is rescaled in TMEM only when
//                      the running max grows by more than a threshold (lazy
//                      rescaling: the exponentials stay below 2^threshold
//                      otherwise), the only time softmax waits for the previous
//                      P*V. A share of the exponentials runs as a polynomial on
//                      the FMA pipe (the MUFU unit does 16 per clock per SM).
//                      Only the row max and the exponentials sit between
//                      S ready and P ready: the row sum and the correction
//                      factor are updated after P is handed over, and the
//                      last-page test is taken before the wait for S. The
//                      epilogue divides by the row sum, stages bf16
//                      rows in shared memory and each warp writes its 32 rows
//                      with a TMA store that clips rows past C.
// Operand formats:
//   bf16: kind::f16 MMAs (K = 16 per instruction); P as bf16 pairs (64 TMEM
//         columns); lazy threshold 2^8.
//   E4M3: kind::f8f6f4 MMAs (K = 32 per instruction) on the pool's FP8 codes.
//         Every Q tile and K/V page block carries a power-of-two scale (the
//         FP8 K/V payload plus scales of Appendix Table 8). The S of key tile j
//         is scaled by 2^(eq + ek_j) inside the softmax's scale-subtract; the
//         V scale of tile j is folded into P: P'_j = P * 2^(ev_j - ev_max + 4),
//         rounded to E4M3 (4 per TMEM column, 32 columns), so O accumulates in
//         units of 2^(ev_max - 4) and the row sum adds P'_j * 2^(ev_max + 4 - ev_j).
//         The lazy threshold is 2^4, so P' <= 2^8 stays inside E4M3's range
//         (448) while small probabilities keep 4 more binades above its
//         subnormal range. P_q lives in shared memory (the tile's 32 KB output
//         staging block, idle until the epilogue), read by an SS P*V MMA, so
//         the issuer computes S_q(j+1) as soon as the softmax has read S_q(j)
//         into registers (an "S read" barrier) instead of after P_q(j)*V: the
//         MMA latency leaves the softmax's chain. The softmax still waits
//         for P_q(j-1)*V before it overwrites P_q; that wait keeps the two
//         tiles' softmax warps of a sub-partition out of phase, so their
//         exponentials do not contend for MUFU and issue slots (computing the
//         whole row before the wait, or issuing the MMAs in the order their
//         inputs become ready, measured slower). (Turn-taking between the two
//         tiles' softmax warps on the MUFU unit is kept as an option, off.)
// Every wait is bounded: on timeout the CTA records WF_ERR_TIMEOUT, the other
// roles see the abort flag, in-flight copies and MMAs are drained (with a
// separate, longer bound), pending TMEM stores are waited for, and TMEM is
// freed before the CTA exits. No output of a CTA that gave up is written.
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
constexpr int kPageCache = 1024;      // page ids (and FP8 scale exponents) cached in smem
// Warpgroups 0 and 1 run the softmax of tiles 0 and 1; warpgroup 2 holds the
// TMA producers (warp 8: Q and K, warp 10: V) and the MMA issuer (warp 9);
// warp 11 only hands its registers over. Launched at 168 registers per thread (384 x 168 =
// 64512), warpgroup 2 gives registers to the softmax warpgroups: 96 / 200 for
// bf16, 80 / 208 for E4M3 (whose softmax also carries the block scales; timed
// 1.8 % faster than 96 / 200, which is the faster split for bf16).
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;    // Q and K loads
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;  // V loads
template <bool kF8> constexpr uint32_t kRegsSoftmax = kF8 ? 208 : 200;
template <bool kF8> constexpr uint32_t kRegsControl = kF8 ? 80 : 96;
static_assert(256 * kRegsSoftmax<false> + 128 * kRegsControl<false> <= 384 * 168, "register split");
static_assert(256 * kRegsSoftmax<true> + 128 * kRegsControl<true> <= 384 * 168, "register split");

// TMEM columns.
constexpr uint32_t kTmemS = 0;        // S_q at 128 q; P_q aliases its first columns
constexpr uint32_t kTmemO = 256;      // O_q at 256 + 128 q

template <bool kF8>
struct Fmt {
  // One [128 rows][128 elements] operand tile in shared memory: bf16 as two
  // 64-column 128-byte-swizzled halves, E4M3 as one 128-byte-swizzled block.
  static constexpr uint32_t kTile = kF8 ? 16384 : 32768;
  static constexpr uint32_t kHalf = 16384;          // bf16 half / fp8 whole tile
  // Stages of the K ring and of the V ring: three for E4M3 (16 KB tiles leave
  // room), two for bf16 (whose rings already fill 128 KB of shared memory).
  static constexpr int kStages = kF8 ? 3 : 2;
  static constexpr uint32_t kOffQ = 0;                          // Q0, Q1
  static constexpr uint32_t kOffK = kOffQ + 2 * kTile;          // K ring
  static constexpr uint32_t kOffV = kOffK + kStages * kTile;    // V ring
  // bf16 output staging: the tile's own Q buffer (bf16) or a separate 32 KB
  // buffer per tile (E4M3, whose Q tile is only 16 KB).
  static constexpr uint32_t kOffStage = kOffV + kStages * kTile;
  static constexpr uint32_t kOffBar = kF8 ? kOffStage + 2 * 32768 : kOffStage;
  static constexpr float kLazy = kF8 ? 4.0f : 8.0f;             // rescale threshold (log2)
  static constexpr int kPShift = 4;                             // E4M3 headroom of P'
  static constexpr int kNumBars = 30;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // TMEM base, abort, 12 ints
  static constexpr uint32_t kOffPages = kOffMisc + 64;
  static constexpr uint32_t kOffExps = kOffPages + kPageCache * 4;   // int16 ek, ev (FP8)
  static constexpr uint32_t kSmemBytes = kOffExps + (kF8 ? kPageCache * 4 : 0) + 1024;
};

constexpr int kNumBars = Fmt<false>::kNumBars;
enum Bar {
  kQFull = 0, kKFull0 = 1, kKEmpty0 = 4, kVFull0 = 7, kVEmpty0 = 10,   // up to 3 stages each
  kSFull0 = 13, kPReady0 = 15, kPVDone0 = 17, kDrain = 19,
  kTurn0 = 20, kTurn1 = 24,  // E4M3: exponential-phase turns, one per sub-partition and tile
  kSRead0 = 28               // E4M3: the softmax has read S_q into registers (one per tile)
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

#ifndef WF_F8_POLY_PAIRS
#define WF_F8_POLY_PAIRS 6
#endif
#ifndef WF_F8_TURNS
#define WF_F8_TURNS 0
#endif
#ifndef WF_BF16_POLY_PAIRS
#define WF_BF16_POLY_PAIRS 4
#endif
constexpr int kBf16PolyPairs = WF_BF16_POLY_PAIRS;
// E4M3: of every 16 pairs of exponentials, this many run as a polynomial on
// the FMA pipe instead of the MUFU unit (which does 16 exponentials per clock
// per SM, in the f32 form as in the packed f16x2/bf16x2 forms: measured).
constexpr int kF8PolyPairs = WF_F8_POLY_PAIRS;
constexpr bool kF8Turns = WF_F8_TURNS != 0;

// 2^x for a pair of values on the FMA pipe: x = n + f with n = round(x) (adding
// and subtracting 1.5 * 2^23 rounds to an integer) and f in [-1/2, 1/2]; 2^f
// from a degree-2 polynomial whose coefficients minimise the largest relative
// error on [-1/2, 1/2] (1.73e-3, far below E4M3's half unit of 2^-4); n is
// added to the exponent field. x is clamped below at -126 first, so -inf
// (masked keys) and very small probabilities come out below 2^-125 (n >= -126
// keeps the exponent field from borrowing into the sign bit even when
// 2^f < 1), which rounds to zero in E4M3 at any block scale the kernel uses.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  float a, b;
  unf2(x2, a, b);
  const uint64_t xc = f2(fmaxf(a, -126.0f), fmaxf(b, -126.0f));
  const uint64_t t = fadd2(xc, f2(12582912.0f, 12582912.0f));    // 1.5 * 2^23 + n
  float t0, t1;
  unf2(t, t0, t1);
  const uint64_t nf = fadd2(t, f2(-12582912.0f, -12582912.0f));  // n
  const uint64_t fr = ffma2(nf, f2(-1.0f, -1.0f), xc);            // f = x - n, exact
  uint64_t p = ffma2(fr, f2(0.23842734f, 0.23842734f), f2(0.70344603f, 0.70344603f));
  p = ffma2(p, fr, f2(1.0004431f, 1.0004431f));
  float p0, p1;
  unf2(p, p0, p1);
  // the low bits of t's pattern hold n (two's complement); shifted into the
  // exponent field they scale p by 2^n
  p0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
  return f2(p0, p1);
}

// The same with a degree-3 polynomial (largest relative error 7.5e-5 on
// [-1/2, 1/2], far below bf16's half unit of 2^-9), for bf16 P; clamped
// inputs give less than 2^-125, nothing next to a row sum of at least 1.
__device__ __forceinline__ uint64_t exp2_poly3(uint64_t x2) {
  float a, b;
  unf2(x2, a, b);
  const uint64_t xc = f2(fmaxf(a, -126.0f), fmaxf(b, -126.0f));
  const uint64_t t = fadd2(xc, f2(12582912.0f, 12582912.0f));
  float t0, t1;
  unf2(t, t0, t1);
  const uint64_t nf = fadd2(t, f2(-12582912.0f, -12582912.0f));
  const uint64_t fr = ffma2(nf, f2(-1.0f, -1.0f), xc);
  uint64_t p = ffma2(fr, f2(0.0551715f, 0.0551715f), f2(0.24261096f, 0.24261096f));
  p = ffma2(p, fr, f2(0.69326097f, 0.69326097f));
  p = ffma2(p, fr, f2(0.99992806f, 0.99992806f));
  float p0, p1;
  unf2(p, p0, p1);
  p0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
  return f2(p0, p1);
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

// 2^k for -126 <= k <= 127, exactly.
__device__ __forceinline__ float exp2i(int k) {
  k = k < -126 ? -126 : (k > 127 ? 127 : k);
  return __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

// Exponent e of a power-of-two scale 2^e stored as fp32.
__device__ __forceinline__ int scale_exp(float s) {
  return static_cast<int>((__float_as_uint(s) >> 23) & 0xFFu) - 127;
}

// S_q = Q_q K(stage)^T along d = 128.
//   bf16: 8 k-steps of 16, each 32 bytes into a 64-column half.
//   E4M3: 4 k-steps of 32, each 32 bytes along the 128-byte row.
template <bool kF8>
__device__ __forceinline__ void issue_s(uint32_t tmem_s, uint32_t q_lo, uint32_t k_lo,
                                        uint32_t hi) {
  if constexpr (kF8) {
    constexpr uint32_t idS = make_idesc_e4m3(kBM, kBN, false);
#pragma unroll
    for (int k = 0; k < kHD / 32; ++k) {
      const uint32_t off = (k * 32) >> 4;
      mma_f8_ss2(tmem_s, q_lo + off, k_lo + off, hi, idS, k > 0);
    }
  } else {
    constexpr uint32_t idS = make_idesc_bf16(kBM, kBN, false);
#pragma unroll
    for (int k = 0; k < kHD / 16; ++k) {
      const uint32_t off = ((k >> 2) * Fmt<false>::kHalf + (k & 3) * 32) >> 4;
      mma_bf16_ss2(tmem_s, q_lo + off, k_lo + off, hi, idS, k > 0);
    }
  }
}

// O_q (+)= P_q V(stage) over the 128 keys of the tile; P_q is read from TMEM
// (8 columns per k-step: 16 bf16 or 32 E4M3 keys), V is MN-major in shared
// memory (one k-step = 16 or 32 key rows of 128 bytes).
template <bool kF8>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_lo,
                                         uint32_t hi, bool accumulate_first) {
  if constexpr (kF8) {
    constexpr uint32_t idPV = make_idesc_e4m3(kBM, kHD, true);
#pragma unroll
    for (int k = 0; k < kBN / 32; ++k)
      mma_f8_ts2(tmem_o, tmem_p + k * 8, v_lo + ((k * 4096) >> 4), hi, idPV,
                 (accumulate_first || k > 0) ? 1u : 0u);
  } else {
    constexpr uint32_t idPV = make_idesc_bf16(kBM, kHD, true);
#pragma unroll
    for (int k = 0; k < kBN / 16; ++k)
      mma_bf16_ts2(tmem_o, tmem_p + k * 8, v_lo + ((k * 2048) >> 4), hi, idPV,
                   (accumulate_first || k > 0) ? 1u : 0u);
  }
}

// O_q (+)= P_q V(stage) with P_q in shared memory (E4M3: one 128-byte-swizzled
// [128 rows][128 keys] block, K-major like Q), V MN-major as above.
__device__ __forceinline__ void issue_pv_f8_smem(uint32_t tmem_o, uint32_t p_lo, uint32_t v_lo,
                                                 uint32_t hi, bool accumulate_first) {
  constexpr uint32_t idPV = make_idesc_e4m3(kBM, kHD, true);
#pragma unroll
  for (int k = 0; k < kBN / 32; ++k)
    mma_f8_ss2(tmem_o, p_lo + ((k * 32) >> 4), v_lo + ((k * 4096) >> 4), hi, idPV,
               (accumulate_first || k > 0) ? 1u : 0u);
}

template <bool kF8>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tq,
                   const __grid_constant__ CUtensorMap tkv,
                   const __grid_constant__ CUtensorMap tout) {
  using F = Fmt<kF8>;
  constexpr uint32_t kTile = F::kTile;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + F::kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + F::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + F::kOffMisc + 4);
  int *ev_red = reinterpret_cast<int *>(smem + F::kOffMisc + 8);   // 12 warps
  int32_t *page_cache = reinterpret_cast<int32_t *>(smem + F::kOffPages);
  int16_t *ek_cache = reinterpret_cast<int16_t *>(smem + F::kOffExps);
  int16_t *ev_cache = ek_cache + kPageCache;
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
  const int n_tiles = npos * p.npc;

  // Readiness + bounds check of the whole round's context (so that a stale
  // page stops every CTA of the launch), caching the page ids and, for FP8,
  // the K/V scale exponents of this head over the slot's own key tiles.
  int ev_max = -127;
  {
    int bad = 0, stale = 0, evm = -127;
    const int total = p.n_pos * p.npc;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
      const int pos = i / p.npc;
      const int pg = __ldcg(p.table + kTabPages + i);
      if (pg < 0 || pg >= p.num_pages) {
        bad = 1;
      } else {
        if (__ldcg(p.tags + pg) != __ldcg(p.table + kTabPosTag + pos)) stale = 1;
        if (kF8 && i < n_tiles) {
          const int ek = scale_exp(__ldcg(p.kv_scale + (static_cast<size_t>(pg) * 2) * p.Hh + h));
          const int ev = scale_exp(__ldcg(p.kv_scale + (static_cast<size_t>(pg) * 2 + 1) * p.Hh + h));
          evm = max(evm, ev);
          if (i < kPageCache) {
            ek_cache[i] = static_cast<int16_t>(ek);
            ev_cache[i] = static_cast<int16_t>(ev);
          }
        }
      }
      if (i < kPageCache) page_cache[i] = pg;
    }
    if (kF8) {
      evm = __reduce_max_sync(0xffffffffu, evm);
      if (lane == 0) ev_red[warp] = evm;
    }
    if (threadIdx.x == 0) {
      *abort_flag = 0;
      for (int b = 0; b < kNumBars; ++b) {
        // p_ready, s_read: one elected arrival per softmax warp of the tile
        const bool softmax_arrives = b == kPReady0 || b == kPReady0 + 1 || b == kSRead0 ||
                                     b == kSRead0 + 1;
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
    if (kF8) {
#pragma unroll
      for (int w = 0; w < kThreads / 32; ++w) ev_max = max(ev_max, ev_red[w]);
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
  const Ctx ctx{bars, abort_flag, p.status, p.wait_limit};
  const int last_valid = p.C - (p.npc - 1) * p.P;   // keys in a chunk's last page

  if (warp >= 8) {
   setmaxnreg_dec<kRegsControl<kF8>>();
   if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tkv);
      tma_prefetch_desc(&tout);
      uint8_t *sQ = smem + F::kOffQ;
      mbar_arrive_expect_tx(bars + kQFull, has_q1 ? 2 * kTile : kTile);
      if constexpr (kF8) {
        tma_load_4d(sQ, &tq, bars + kQFull, 0, h, row0, slot);
        if (has_q1) tma_load_4d(sQ + kTile, &tq, bars + kQFull, 0, h, row0 + kBM, slot);
      } else {
        tma_load_4d(sQ, &tq, bars + kQFull, 0, h, row0, slot);
        tma_load_4d(sQ + F::kHalf, &tq, bars + kQFull, 64, h, row0, slot);
        if (has_q1) {
          tma_load_4d(sQ + kTile, &tq, bars + kQFull, 0, h, row0 + kBM, slot);
          tma_load_4d(sQ + kTile + F::kHalf, &tq, bars + kQFull, 64, h, row0 + kBM, slot);
        }
      }
      // K of key tile j goes to stage j % kStages as that stage's fill
      // j / kStages, behind the S MMAs of tile j - kStages (K empty).
      int jk_last = -1;                          // last K tile loaded
      for (int j = 0; j < n_tiles; ++j) {
        const int stg = j % F::kStages;
        const uint32_t ph = (j / F::kStages) & 1;
        const int phys = j < kPageCache ? page_cache[j] : __ldcg(p.table + kTabPages + j);
        const int rowk = static_cast<int>(p.layer_row0) + ((phys * 2) * p.Hh + h) * p.P;
        uint8_t *sK = smem + F::kOffK + stg * kTile;
        if (!wait_bar(ctx, kKEmpty0 + stg, ph ^ 1)) break;
        if (j != p.skip_key_tile) {   // test hook: a skipped load leaves its wait to run out
          mbar_arrive_expect_tx(bars + kKFull0 + stg, kTile);
          tma_load_2d(sK, &tkv, bars + kKFull0 + stg, 0, rowk);
          if (!kF8) tma_load_2d(sK + F::kHalf, &tkv, bars + kKFull0 + stg, 64, rowk);
          jk_last = j;
        }
      }
      // Drain: every load this thread issued has landed before the CTA exits.
      // Loads into one stage complete its phases in order, so waiting for the
      // phase of the last one issued into each stage covers them all.
#pragma unroll
      for (int st = 0; st < F::kStages; ++st) {
        int jl = jk_last - ((jk_last - st) % F::kStages + F::kStages) % F::kStages;
        if (jl == p.skip_key_tile) jl -= F::kStages;   // the hook's tile was never loaded
        if (jl >= 0) drain_wait(ctx, kKFull0 + st, (jl / F::kStages) & 1);
      }
      drain_wait(ctx, kQFull, 0);
    }
  } else if (warp == kVProducerWarp) {
    // ---------------------------------------------------------- V producer --
    // V of key tile j goes to stage j % kStages behind the P*V MMAs of tile
    // j - kStages (V empty); a separate thread, so that K loads never queue
    // behind a V load waiting for its stage.
    if (lane == 0) {
      int jv_last = -1;
      for (int j = 0; j < n_tiles; ++j) {
        const int stg = j % F::kStages;
        const uint32_t ph = (j / F::kStages) & 1;
        const int phys = j < kPageCache ? page_cache[j] : __ldcg(p.table + kTabPages + j);
        const int rowv = static_cast<int>(p.layer_row0) + ((phys * 2 + 1) * p.Hh + h) * p.P;
        uint8_t *sV = smem + F::kOffV + stg * kTile;
        if (!wait_bar(ctx, kVEmpty0 + stg, ph ^ 1)) break;
        mbar_arrive_expect_tx(bars + kVFull0 + stg, kTile);
        tma_load_2d(sV, &tkv, bars + kVFull0 + stg, 0, rowv);
        if (!kF8) tma_load_2d(sV + F::kHalf, &tkv, bars + kVFull0 + stg, 64, rowv);
        jv_last = j;
      }
#pragma unroll
      for (int st = 0; st < F::kStages; ++st) {
        const int jl = jv_last - ((jv_last - st) % F::kStages + F::kStages) % F::kStages;
        if (jl >= 0) drain_wait(ctx, kVFull0 + st, (jl / F::kStages) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      // Descriptor words: the high word (stride 1 KB, version, swizzle) is the
      // same for Q, K and V; a k-step or a stage only moves the low word.
      const uint32_t hi = desc_hi_sw128(1024);
      const uint32_t q_lo = desc_lo_sw128(smem_u32(smem + F::kOffQ), 16);
      const uint32_t k_lo = desc_lo_sw128(smem_u32(smem + F::kOffK), 16);
      const uint32_t v_lo = desc_lo_sw128(smem_u32(smem + F::kOffV), F::kHalf);
      constexpr uint32_t kTileStep = kTile >> 4;
      bool ok = wait_bar(ctx, kQFull, 0) && wait_bar(ctx, kKFull0, 0);
      if (ok) {
        tc_fence_after();
        issue_s<kF8>(tmem + kTmemS, q_lo, k_lo, hi);
        mma_commit(bars + kSFull0);
        if (has_q1) {
          issue_s<kF8>(tmem + kTmemS + 128, q_lo + kTileStep, k_lo, hi);
          mma_commit(bars + kSFull0 + 1);
        }
        mma_commit(bars + kKEmpty0);
      }
      // E4M3: P_q lives in shared memory (in the tile's output staging buffer),
      // so S_q(j+1) may overwrite S_q(j) in TMEM as soon as the softmax has read
      // it; the next S is computed while the softmax works on this one, and
      // only P_q V(j) waits for P_q(j).
      const uint32_t p_lo = desc_lo_sw128(smem_u32(smem + F::kOffStage), 16);
      constexpr uint32_t kPStep = 32768 >> 4;                 // tile 1's P (staging) buffer
      for (int j = 0; kF8 && ok && j < n_tiles; ++j) {
        const int stg = j % F::kStages, nstg = (j + 1) % F::kStages;
        if (j + 1 < n_tiles) {
          if (!wait_bar(ctx, kKFull0 + nstg, ((j + 1) / F::kStages) & 1)) break;
          if (!wait_bar(ctx, kSRead0, j & 1)) break;
          tc_fence_after();
          issue_s<kF8>(tmem + kTmemS, q_lo, k_lo + nstg * kTileStep, hi);
          mma_commit(bars + kSFull0);
          if (has_q1) {
            if (!wait_bar(ctx, kSRead0 + 1, j & 1)) break;
            tc_fence_after();
            issue_s<kF8>(tmem + kTmemS + 128, q_lo + kTileStep, k_lo + nstg * kTileStep, hi);
            mma_commit(bars + kSFull0 + 1);
          }
          mma_commit(bars + kKEmpty0 + nstg);
        }
        if (!wait_bar(ctx, kVFull0 + stg, (j / F::kStages) & 1)) break;
        if (!wait_bar(ctx, kPReady0, j & 1)) break;
        tc_fence_after();
        issue_pv_f8_smem(tmem + kTmemO, p_lo, v_lo + stg * kTileStep, hi, j > 0);
        mma_commit(bars + kPVDone0);
        if (has_q1) {
          if (!wait_bar(ctx, kPReady0 + 1, j & 1)) break;
          tc_fence_after();
          issue_pv_f8_smem(tmem + kTmemO + 128, p_lo + kPStep, v_lo + stg * kTileStep, hi, j > 0);
          mma_commit(bars + kPVDone0 + 1);
        }
        mma_commit(bars + kVEmpty0 + stg);
      }
      for (int j = 0; !kF8 && ok && j < n_tiles; ++j) {
        const int stg = j % F::kStages, nstg = (j + 1) % F::kStages;
        const bool more = j + 1 < n_tiles;
        if (!wait_bar(ctx, kVFull0 + stg, (j / F::kStages) & 1)) break;
        if (!wait_bar(ctx, kPReady0, j & 1)) break;
        tc_fence_after();
        issue_pv<kF8>(tmem + kTmemO, tmem + kTmemS, v_lo + stg * kTileStep, hi, j > 0);
        mma_commit(bars + kPVDone0);
        if (more) {
          if (!wait_bar(ctx, kKFull0 + nstg, ((j + 1) / F::kStages) & 1)) break;
          tc_fence_after();
          issue_s<kF8>(tmem + kTmemS, q_lo, k_lo + nstg * kTileStep, hi);
          mma_commit(bars + kSFull0);
        }
        if (has_q1) {
          if (!wait_bar(ctx, kPReady0 + 1, j & 1)) break;
          tc_fence_after();
          issue_pv<kF8>(tmem + kTmemO + 128, tmem + kTmemS + 128, v_lo + stg * kTileStep, hi,
                        j > 0);
          mma_commit(bars + kPVDone0 + 1);
          if (more) {
            issue_s<kF8>(tmem + kTmemS + 128, q_lo + kTileStep, k_lo + nstg * kTileStep, hi);
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
   setmaxnreg_inc<kRegsSoftmax<kF8>>();
   if (warp < 4 || has_q1) {
    // ------------------------------------------------------------- softmax --
    const int q = warp >> 2;
    const int r = (warp & 3) * 32 + lane;               // query row == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + kTmemS + q * 128;
    const uint32_t tO = tmem + lane_addr + kTmemO + q * 128;
    // FP8: the S of tile j in log2 units is acc * scale_log2 * 2^eq * 2^ek_j.
    float qs_log2 = p.scale_log2;
    if (kF8) {
      const int qt = 2 * pair + q;
      qs_log2 *= exp2i(scale_exp(__ldg(p.q_scale + (static_cast<size_t>(slot) * p.npc + qt) * p.Hh + h)));
    }
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    int jp = 0;                      // page of tile j inside its chunk (no division in the loop)
    for (int j = 0; j < n_tiles; ++j) {
      float c_j = p.scale_log2;      // log2(e)/sqrt(d) times the FP8 block scales
      float dv = 0.0f;               // FP8: log2 of P's V-scale factor, ev_j - ev_max + 4
      if (kF8) {
        int ek, ev;
        if (j < kPageCache) {
          ek = ek_cache[j];
          ev = ev_cache[j];
        } else {
          const int pg = __ldcg(p.table + kTabPages + j);
          ek = scale_exp(__ldcg(p.kv_scale + (static_cast<size_t>(pg) * 2) * p.Hh + h));
          ev = scale_exp(__ldcg(p.kv_scale + (static_cast<size_t>(pg) * 2 + 1) * p.Hh + h));
        }
        // kept normal so that masked keys (-inf) stay -inf when both blocks are ~0
        c_j = fmaxf(qs_log2 * exp2i(ek), 1.17549435e-38f);
        dv = static_cast<float>(ev - ev_max + F::kPShift);
      }
      // Keys past the chunk's length on its last page are masked. Worked out
      // before the wait: after it, the integer division would queue on the
      // MUFU unit behind the other tile's exponentials.
      const int valid = jp == p.npc - 1 ? last_valid : kBN;
      if (++jp == p.npc) jp = 0;
      ok = __all_sync(0xffffffffu, wait_bar(ctx, kSFull0 + q, j & 1));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, s + c * 32);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence32(s + c * 32);
      if constexpr (kF8) {
        // S_q is in registers: the issuer may compute the next S_q over it.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + kSRead0 + q);
      }

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
      const float m_new = fmaxf(m, mx * c_j);
      const bool rescale = m_new - m > F::kLazy;         // always true on the first tile
      const float m_use = rescale ? m_new : m;
      // P = 2^(s * c_j - m [+ dv]) on the MUFU unit, the scale-subtract and
      // the row sums in packed f32x2 arithmetic; rounded to the operand format
      // and streamed back into the first columns of S_q, 32 keys at a time.
      // E4M3: the two tiles' softmax warps of a sub-partition take turns on the
      // exponentials (tile 0 first), so that each runs them with the MUFU unit
      // to itself; the turn is handed on after three quarters of the row. With
      // the FP8 MMAs' shorter P*V + S the two phases would otherwise overlap
      // (bf16 tiles stay apart by themselves, and a turn only delays them).
      if (kF8 && kF8Turns && has_q1 && (q == 1 || j > 0)) {
        ok = __all_sync(0xffffffffu, wait_bar(ctx, (q == 0 ? kTurn0 : kTurn1) + (warp & 3),
                                              q == 0 ? ((j - 1) & 1) : (j & 1)));
        if (!ok) break;
      }
      if (kF8 && j > 0) {
        // P_q(j-1) in shared memory is read by P*V(j-1) until that completes.
        ok = __all_sync(0xffffffffu, wait_bar(ctx, kPVDone0 + q, (j - 1) & 1));
        if (!ok) break;
      }
      // E4M3: row r of P_q in its 128-byte-swizzled staging block (K-major,
      // the layout of a Q tile): 16-byte chunk c at r * 128 + (c ^ (r & 7)) * 16.
      const uint32_t p_row = smem_u32(smem + F::kOffStage + q * 32768 + r * 128);
      const uint64_t sc2 = f2(c_j, c_j), nm2 = f2(dv - m_use, dv - m_use);
      uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        if constexpr (kF8) {
          uint32_t pw[8], half = 0;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int k0 = cc * 32 + 2 * c;
            const uint64_t x2 = ffma2(f2(__uint_as_float(s[k0]), __uint_as_float(s[k0 + 1])), sc2, nm2);
            float e0, e1;
            if (c % 8 >= 8 - kF8PolyPairs / 2 - (c < 8 ? kF8PolyPairs % 2 : 0)) {
              unf2(exp2_poly2(x2), e0, e1);
            } else {
              float a, b;
              unf2(x2, a, b);
              e0 = ex2(a);
              e1 = ex2(b);
            }
            acc[c & 3] = fadd2(acc[c & 3], f2(e0, e1));
            const uint32_t pr = pack_e4m3x2(e0, e1);
            if (c & 1) pw[c >> 1] = join16(half, pr);
            else half = pr;
          }
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const uint32_t addr = p_row + ((((2 * cc + h2) ^ (r & 7)) & 7) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pw[4 * h2]),
                         "r"(pw[4 * h2 + 1]), "r"(pw[4 * h2 + 2]), "r"(pw[4 * h2 + 3])
                         : "memory");
          }
          if (kF8Turns && cc == 2 && has_q1 && lane == 0)
            mbar_arrive(bars + (q == 0 ? kTurn1 : kTurn0) + (warp & 3));
        } else {
          uint32_t pw[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int k0 = cc * 32 + 2 * c;
            const uint64_t x2 = ffma2(f2(__uint_as_float(s[k0]), __uint_as_float(s[k0 + 1])), sc2, nm2);
            float e0, e1;
            if (c % 8 >= 8 - kBf16PolyPairs / 2 - (c < 8 ? kBf16PolyPairs % 2 : 0)) {
              unf2(exp2_poly3(x2), e0, e1);
            } else {
              float a, b;
              unf2(x2, a, b);
              e0 = ex2(a);
              e1 = ex2(b);
            }
            acc[c & 3] = fadd2(acc[c & 3], f2(e0, e1));
            pw[c] = pack_bf16(e0, e1);
          }
          tmem_st16(tS + cc * 16, pw);
        }
      }

      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
        // O_q must hold P*V up to tile j-1 before it is rescaled.
        ok = __all_sync(0xffffffffu, wait_bar(ctx, kPVDone0 + q, (j - 1) & 1));
        if (!ok) break;
        tc_fence_after();
        const float alpha = rescale ? ex2(m - m_use) : 1.0f;
        const uint64_t a2 = f2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
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
      if (kF8) fence_proxy_async_smem();   // P_q's shared-memory stores, read by the MMA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + kPReady0 + q);
      // The row sum and the correction factor come after P is handed over, off
      // the path from S to P.
      float sum0, sum1;
      unf2(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), sum0, sum1);
      float tile_sum = sum0 + sum1;
      if (kF8) tile_sum *= exp2i(-static_cast<int>(dv));   // back to units of P
      if (rescale) l *= ex2(m - m_use);   // the MUFU only when the max moved
      l += tile_sum;
      m = m_use;
    }
    if (ok && n_tiles > 0) {
      ok = __all_sync(0xffffffffu, wait_bar(ctx, kPVDone0 + q, (n_tiles - 1) & 1));
    }
    if (ok && n_tiles > 0) {
      tc_fence_after();
      // FP8: O accumulated in units of 2^(ev_max - 4).
      const float inv = (kF8 ? exp2i(ev_max - F::kPShift) : 1.0f) / l;
      // Stage the bf16 rows in the 128-byte swizzled layout of the output
      // tensor map, whose box is 32 rows: 16-byte chunk c of row r in 64-column
      // half kt lands at kt * 16 KB + r * 128 + ((c ^ (r & 7)) * 16), so each
      // warp's 32 rows form one contiguous 4 KB box per half and the warp
      // stores them itself (no cross-warp barrier). bf16 stages in the tile's
      // Q buffer (its last reader, the final S MMA, has completed); E4M3 in a
      // buffer of its own.
      uint8_t *stage = kF8 ? smem + F::kOffStage + q * 32768 : smem + F::kOffQ + q * kTile;
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
          const uint32_t addr = smem_u32(stage + kt * 16384 + r * 128 + ((c ^ (r & 7)) << 4));
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
        tma_store_4d(&tout, stage + 16384 + wr * 128, 64, h, row0 + q * kBM + wr, slot);
        tma_store_commit();
        tma_store_wait_all();
      }
      __syncwarp();
    }
    // A softmax that gave up mid-tile may still have TMEM stores in flight.
    tmem_st_wait();
   }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <bool kF8>
cudaError_t launch_tc(const AttnParams &p, const void *tmap_q, const void *tmap_kv,
                      const void *tmap_out, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  if (p.d != kHD || p.P != kBN) return cudaErrorInvalidValue;
  if (kF8 && (!p.kv_scale || !p.q_scale)) return cudaErrorInvalidValue;
  constexpr uint32_t bytes = Fmt<kF8>::kSmemBytes;
  static_assert(bytes <= 227 * 1024, "shared memory");
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<kF8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  const int tiles = (p.C + kBM - 1) / kBM;
  const int64_t blocks = static_cast<int64_t>((tiles + 1) / 2) * p.live.n * p.Hh;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  attn_tc_kernel<kF8><<<static_cast<unsigned>(blocks), kThreads, bytes, st>>>(
      p, *static_cast<const CUtensorMap *>(tmap_q), *static_cast<const CUtensorMap *>(tmap_kv),
      *static_cast<const CUtensorMap *>(tmap_out));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_bf16(const AttnParams &p, const void *tmap_q, const void *tmap_kv,
                                  const void *tmap_out, cudaStream_t st) {
  return launch_tc<false>(p, tmap_q, tmap_kv, tmap_out, st);
}

cudaError_t launch_attention_fp8(const AttnParams &p, const void *tmap_q, const void *tmap_kv,
                                 const void *tmap_out, cudaStream_t st) {
  return launch_tc<true>(p, tmap_q, tmap_kv, tmap_out, st);
}

}  // namespace wf
