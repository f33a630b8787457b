// Fused QKV projection + 3D rotary + early publication, tcgen05 GEMM on CTA
// pairs (cta_group::2) for sm_100a.
//
// "Wave Forcing: Towards Speed-of-Light Streaming Video Generation", Method
// section: each rank's local QKV projection runs without waiting for remote
// K/V, and K/V are published right after the QKV projection and RoPE, with
// direct writes into ordered attention slots. Here the projection's epilogue
// is the publication: q_rot is written, K and V go straight into the slot's
// pages, the rows past C in the chunk's last page are zeroed and the ready tag
// is stamped, so q, k and v never make a round trip through HBM.
//
// Y[token][f] = sum_i x[token][i] * w[f][i] for the live slots' tokens, with
// f over the 3 * hidden stacked q, k, v output features.
//   Tile: 256 tokens (two 128-token pages of the slot's chunk) x 256 output
//   features (two heads of q, k or v), computed by a cluster of two CTAs with
//   M = 256, N = 256, K = 16 MMAs issued by the leader (rank 0). CTA r holds
//   page 2 mt + r of x (128 rows) and features [128 r, 128 r + 128) of w in its
//   own shared memory, so each SM reads 32 KB of operands per 64-element
//   k-block for 128 FLOP per byte, and receives its page's 128 x 256
//   accumulator in its own TMEM.
//   The kernel is persistent: pair p walks the tiles p, p + pairs, ... (feature
//   tiles fastest, so the x pages and all of w stay in L2). Accumulators are
//   double-buffered in TMEM (columns [256 b, 256 b + 256)), so the epilogue of
//   one tile overlaps the main loop of the next.
//   warp 8 (one lane)  TMA producer of its CTA: a 6-stage ring of 32 KB stages
//                      (128-byte swizzle); the loads of both CTAs count on the
//                      leader's full barrier, and the leader's commits free the
//                      stage in both CTAs.
//   warp 9 (one lane)  leader only: tcgen05 issuer.
//   warps 0-7          epilogue: warpgroup e drains head e of the tile (128
//                      accumulator columns) for the CTA's 128 token rows; thread
//                      r owns token r (TMEM lane r) and drains 32 columns at a
//                      time, the next piece's TMEM load and (cos, sin) loads in
//                      flight, rotates q and k pairs in fp32 with the pool's
//                      tables, rounds once to bf16 and stages the rows
//                      (128-byte swizzle). Each warp writes its 32 rows with TMA
//                      stores: q_rot through the activation map, K and V into
//                      the page rows; the accumulator is released to the next
//                      tile as soon as its last TMEM load has completed.
// Every wait is bounded (timeout recorded in the pool's status word).
#include <cuda.h>
#include <cuda_bf16.h>

#include "pipeline.cuh"
#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {
namespace {

using namespace sm100;

constexpr int kPage = 128;                    // tokens per page (M per CTA)
constexpr int kGN = 256;                      // output features per tile (N)
constexpr int kHalfN = kGN / 2;               // features of w held by each CTA
constexpr int kGK = 64;                       // hidden elements per k-block (128 bytes)
constexpr int kStages = 6;
constexpr uint32_t kABytes = kPage * kGK * 2;     // 16 KB
constexpr uint32_t kBBytes = kHalfN * kGK * 2;    // 16 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
// Epilogue staging: per head slot, one 64-dimension half of 128 rows x 128 B
// at a time (each warp's 32 rows are its own; the second half waits until the
// first half's TMA store has read them).
constexpr uint32_t kHalfStage = kPage * 128;      // 16 KB
constexpr uint32_t kOffStage = kStages * kStageBytes;
constexpr uint32_t kOffBar = kOffStage + 2 * kHalfStage;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
enum {
  kFull0 = 0,                     // [kStages] leader: both CTAs' operand bytes landed
  kEmpty0 = kStages,              // [kStages] both: stage consumed by the MMAs
  kAccFull0 = 2 * kStages,        // [2] both: accumulator b complete
  kAccEmpty0 = 2 * kStages + 2,   // [2] leader: accumulator b drained by both CTAs
  kDrain = 2 * kStages + 4,
  kNumBars = 2 * kStages + 5
};
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;   // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&b);
}

struct Tile {
  int li, mt, nt;
};

// Tile t: feature tile fastest, then token tile (page pair), then live slot.
__device__ __forceinline__ Tile decode(int t, int n_tiles, int m_tiles) {
  Tile k;
  k.nt = t % n_tiles;
  const int rest = t / n_tiles;
  k.mt = rest % m_tiles;
  k.li = rest / m_tiles;
  return k;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    project_kernel(const __grid_constant__ ProjectParams p, const __grid_constant__ CUtensorMap tx,
                   const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tq,
                   const __grid_constant__ CUtensorMap tkv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  const int n_tiles = 3 * p.hidden / kGN;
  const int m_tiles = (p.npc + 1) / 2;
  const int total = p.live.n * m_tiles * n_tiles;
  const int n_kb = p.hidden / kGK;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int b = 0; b < kNumBars; ++b)
      mbar_init(bars + b, (b == kAccEmpty0 || b == kAccEmpty0 + 1) ? 2 * kEpiWarps : 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {                   // same warp in both CTAs, same slot offset
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();                           // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Ctx ctx{bars, abort_flag, p.status};

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      tma_prefetch_desc(&tx);
      tma_prefetch_desc(&tw);
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tkv);
      int g = 0;                            // k-blocks issued by this CTA
      bool ok = true;
      for (int t = pair; ok && t < total; t += npairs) {
        const Tile tl = decode(t, n_tiles, m_tiles);
        const int slot = p.live.slot[tl.li];
        for (int kb = 0; kb < n_kb; ++kb, ++g) {
          const int s = g % kStages;
          if (!wait_bar(ctx, kEmpty0 + s, ((g / kStages) & 1) ^ 1)) {
            ok = false;
            break;
          }
          // The leader expects the bytes of both CTAs on its full barrier.
          if (rank == 0) mbar_arrive_expect_tx(bars + kFull0 + s, 2 * kStageBytes);
          uint8_t *sa = smem + s * kStageBytes;
          const uint32_t lb = leader_bar(bars + kFull0 + s);
          tma_load_3d_pair(sa, &tx, lb, kb * kGK, (2 * tl.mt + static_cast<int>(rank)) * kPage,
                           slot);
          tma_load_2d_pair(sa + kABytes, &tw, lb, kb * kGK,
                           tl.nt * kGN + static_cast<int>(rank) * kHalfN);
        }
      }
      // Tail: every stage this CTA filled has been consumed by the MMAs (their
      // commits free the stage in both CTAs), so no load of this CTA is in
      // flight when it exits.
      for (int s = 0; s < kStages && g > 0; ++s) {
        const int fills = g / kStages + (s < g % kStages ? 1 : 0);
        if (fills > 0) drain_wait(ctx, kEmpty0 + s, (fills - 1) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(2 * kPage, kGN, false);
      const uint32_t hi = desc_hi_sw128(1024);
      const uint32_t lo0 = desc_lo_sw128(smem_u32(smem), 16);
      int g = 0, i = 0;
      bool ok = true;
      for (int t = pair; ok && t < total; t += npairs, ++i) {
        const int b = i & 1;
        if (!wait_bar_cluster(ctx, kAccEmpty0 + b, ((i >> 1) & 1) ^ 1)) break;
        tc_fence_after();
        for (int kb = 0; kb < n_kb; ++kb, ++g) {
          const int s = g % kStages;
          if (!wait_bar_cluster(ctx, kFull0 + s, (g / kStages) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_lo = lo0 + ((s * kStageBytes) >> 4);
          const uint32_t b_lo = a_lo + (kABytes >> 4);
#pragma unroll
          for (int k = 0; k < kGK / 16; ++k)
            mma_bf16_ss2_pair(tmem + 256 * b, a_lo + k * 2, b_lo + k * 2, hi, idesc,
                              (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit_pair(bars + kEmpty0 + s);
        }
        if (ok) mma_commit_pair(bars + kAccFull0 + b);
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      mma_commit_pair(bars + kDrain);
      drain_wait(ctx, kDrain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int e = warp >> 2;                             // head slot of the tile
    const int wr = (warp & 3) * 32;                      // first row of this warp
    const int r = wr + lane;                             // token row in the page == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(wr) << 16;
    uint8_t *stage = smem + kOffStage + e * kHalfStage;  // [128 rows][128 B]
    const int h0 = p.split0 >> 1, h1 = p.split1 >> 1, h2 = p.split2 >> 1;
    int i = 0;
    for (int t = pair; t < total; t += npairs, ++i) {
      const int b = i & 1;
      const bool ok = __all_sync(0xffffffffu, wait_bar_cluster(ctx, kAccFull0 + b, (i >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      const Tile tl = decode(t, n_tiles, m_tiles);
      const int slot = p.live.slot[tl.li];
      const int page = 2 * tl.mt + static_cast<int>(rank);
      const int n = page * kPage + r;                    // token inside the chunk
      const bool valid = n < p.C;
      const int f0 = tl.nt * kGN + e * kHalfN;           // first feature of this head
      const int sec = f0 / p.hidden;                     // 0 q, 1 k, 2 v
      const int head = (f0 - sec * p.hidden) / p.d;
      const bool live_page = page < p.npc;
      const bool rot = sec < 2 && p.rope && valid;
      int tpos = 0, ypos = 0, xpos = 0;
      if (p.rope && valid) {
        const int hw = p.gh * p.gw;
        tpos = p.F * p.live.chunk[tl.li] + n / hw;
        ypos = (n / p.gw) % p.gh;
        xpos = n % p.gw;
      }
      int phys = -1;
      if (live_page) {
        const int pos = __ldg(p.table + kTabSlotPos + slot);
        phys = pos < 0 ? -1 : __ldg(p.table + kTabPages + pos * p.npc + page);
        if (phys >= p.num_pages) phys = -1;
      }
      const bool kv_ok = sec > 0 && phys >= 0;
      if (lane == 0 && live_page && sec > 0 && phys < 0) record_status(p.status, WF_ERR_BAD_PAGE);
      // This warp's previous TMA stores must have read the staging rows.
      if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      __syncwarp();
      // (cos, sin) of the 16 pairs of dimensions 32 c .. 32 c + 31 of the head;
      // the band of a pair is picked by selects, all 16 loads issue at once.
      auto load_cs = [&](int c, float2 (&cs)[16]) {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int pr = c * 16 + q;
          const float2 *src = pr < h0        ? p.rope_t + tpos * h0 + pr
                              : pr < h0 + h1 ? p.rope_h + ypos * h1 + (pr - h0)
                                             : p.rope_w + xpos * h2 + (pr - h0 - h1);
          cs[q] = __ldg(src);
        }
      };
      auto store_half = [&](int kt) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const uint8_t *src = stage + wr * 128;
          if (sec == 0) {
            if (page * kPage + wr < p.C)                 // boxes wholly past C are skipped
              tma_store_4d(&tq, src, kt * 64, head, page * kPage + wr, slot);
          } else if (kv_ok) {
            const int64_t row = p.layer_row0 +
                ((static_cast<int64_t>(phys) * 2 + (sec - 1)) * p.Hh + head) * p.P + wr;
            tma_store_2d(&tkv, src, kt * 64, static_cast<int>(row));
          }
          tma_store_commit();
        }
      };
      // Dimensions 32 c .. 32 c + 31 per step, the next step's TMEM load and
      // (cos, sin) in flight; the first 64-dimension half is stored after step
      // 1, while steps 2 and 3 are computed.
      const uint32_t tcol = tmem + lane_addr + 256 * b + e * kHalfN;
      uint32_t cur[32], nxt[32];
      float2 cs[16], csn[16];
      tmem_ld32(tcol, cur);
      if (rot) load_cs(0, cs);
      tmem_ld_wait();
      reg_fence32(cur);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < 3) {
          tmem_ld32(tcol + (c + 1) * 32, nxt);
          if (rot) load_cs(c + 1, csn);
        }
        if (rot) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float a = __uint_as_float(cur[2 * q]), bb = __uint_as_float(cur[2 * q + 1]);
            // Each product and sum rounded once, as in the publish kernels.
            cur[2 * q] = __float_as_uint(__fsub_rn(__fmul_rn(a, cs[q].x), __fmul_rn(bb, cs[q].y)));
            cur[2 * q + 1] = __float_as_uint(__fadd_rn(__fmul_rn(a, cs[q].y), __fmul_rn(bb, cs[q].x)));
          }
        }
        if (live_page && c == 2) {
          // The first half's TMA store has read this warp's staging rows.
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          __syncwarp();
        }
        if (live_page) {
          uint32_t w[16];
#pragma unroll
          for (int q = 0; q < 16; ++q)
            w[q] = valid ? pack_bf16(__uint_as_float(cur[2 * q]), __uint_as_float(cur[2 * q + 1])) : 0u;
          uint8_t *row = stage + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (c & 1) * 4 + q;           // 16-byte chunk of the 128-byte row
            const uint32_t addr = smem_u32(row + ((chunk ^ (r & 7)) << 4));
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[4 * q]),
                         "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                         : "memory");
          }
        }
        if (c < 3) {
          tmem_ld_wait();
          reg_fence32(nxt);
#pragma unroll
          for (int q = 0; q < 32; ++q) cur[q] = nxt[q];
          if (rot) {
#pragma unroll
            for (int q = 0; q < 16; ++q) cs[q] = csn[q];
          }
        } else {
          // Last TMEM load of this accumulator done: release it to the leader.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(bars + kAccEmpty0 + b, 0);
        }
        if (live_page && (c == 1 || c == 3)) store_half(c >> 1);
      }
      if (lane == 0 && sec == 1 && head == 0 && wr == 0 && kv_ok) {
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // page rows written
        p.tags[phys] = p.live.tag[tl.li];
      }
      __syncwarp();
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();                           // no MMA or load of the pair is in flight
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_project_bf16(const ProjectParams &p, const void *tmap_x, const void *tmap_w,
                                const void *tmap_q, const void *tmap_kv, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  if (p.d != 128 || p.P != kPage || p.hidden % kGN != 0) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t tiles = static_cast<int64_t>(p.live.n) * ((p.npc + 1) / 2) * (3 * p.hidden / kGN);
  if (tiles > 0x7fffffff) return cudaErrorInvalidValue;
  const int64_t pairs = tiles < sms / 2 ? tiles : sms / 2;
  project_kernel<<<static_cast<unsigned>(2 * pairs), kThreads, kSmemBytes, st>>>(
      p, *static_cast<const CUtensorMap *>(tmap_x), *static_cast<const CUtensorMap *>(tmap_w),
      *static_cast<const CUtensorMap *>(tmap_q), *static_cast<const CUtensorMap *>(tmap_kv));
  return cudaGetLastError();
}

}  // namespace wf
