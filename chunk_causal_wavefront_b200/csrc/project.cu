// Fused QKV projection + 3D rotary + early publication, tcgen05 GEMM for sm_100a.
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
//   CTA tile: 256 tokens (exactly two 128-token pages of the slot's chunk) x
//   256 output features (two heads of q, k or v); hidden is walked in
//   64-element (128-byte) blocks through a 3-stage TMA ring (128-byte swizzle,
//   A = x tile, B = w tile, both K-major). Each 256 x 256 tile reads 128 FLOP
//   per byte of operands (a 128-token tile would read 85), which matters
//   because the operands come from L2.
//   warp 8 (one lane)  TMA producer;
//   warp 9 (one lane)  tcgen05 issuer: two M = 128, N = 256, K = 16 MMAs per
//                      k-step (one per page of the tile), fp32 accumulation
//                      in TMEM columns [0, 256) and [256, 512);
//   warps 0-7          epilogue, one warpgroup per page: thread r owns token r
//                      of its page (TMEM lane r) and drains its row 32 columns
//                      at a time (the next piece's TMEM load and (cos, sin)
//                      loads in flight), rotates q and k pairs in fp32 with the
//                      pool's tables, rounds once to bf16 and stages the rows in
//                      the drained operand ring (128-byte swizzle). Each warp
//                      then writes its 32 rows with TMA stores: q_rot through
//                      the activation map, K and V into the page rows; the
//                      first 64-dimension half is stored while the second is
//                      computed.
// Order of CTAs: feature tiles fastest, so consecutive CTAs share the x tile
// and sweep w (14 MB for the 1.3B shape), which both stay in L2.
#include <cuda.h>
#include <cuda_bf16.h>

#include "pipeline.cuh"
#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {
namespace {

using namespace sm100;

constexpr int kPage = 128;                    // tokens per page (and per MMA, M)
constexpr int kGM = 2 * kPage;                // tokens per tile
constexpr int kGN = 256;                      // output features per tile
constexpr int kGK = 64;                       // hidden elements per k-block
constexpr int kStages = 3;
constexpr uint32_t kABytes = kGM * kGK * 2;   // 32 KB
constexpr uint32_t kBBytes = kGN * kGK * 2;   // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
// Epilogue staging in the drained operand ring: per page of the tile, two
// heads x two 64-dimension halves of 128 rows x 128 bytes.
constexpr uint32_t kHalfStage = kPage * 128;                    // 16 KB
constexpr uint32_t kHeadStage = 2 * kHalfStage;                 // 32 KB
static_assert(2 * 2 * kHeadStage <= kStages * kStageBytes, "epilogue staging fits the ring");
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kOffBar = kStages * kStageBytes;
enum { kFull0 = 0, kEmpty0 = kStages, kAccFull = 2 * kStages, kDrain = 2 * kStages + 1,
       kNumBars = 2 * kStages + 2 };
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;   // + alignment slack

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&b);
}

// Rotate the 16 pairs of a 32-column piece whose first column is dimension
// dim0 of its head, for a token at rotary position (t, y, x).
__device__ __forceinline__ void rope32(float *v, int dim0, int t, int y, int x,
                                       const ProjectParams &p) {
  const int h0 = p.split0 >> 1, h1 = p.split1 >> 1, h2 = p.split2 >> 1;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int pr = (dim0 >> 1) + i;
    float2 cs;
    if (pr < h0) cs = __ldg(p.rope_t + t * h0 + pr);
    else if (pr < h0 + h1) cs = __ldg(p.rope_h + y * h1 + (pr - h0));
    else cs = __ldg(p.rope_w + x * h2 + (pr - h0 - h1));
    const float a = v[2 * i], b = v[2 * i + 1];
    v[2 * i] = a * cs.x - b * cs.y;
    v[2 * i + 1] = a * cs.y + b * cs.x;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
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

  const int n_tiles = 3 * p.hidden / kGN;
  const int m_tiles = (p.npc + 1) / 2;
  const int nt = blockIdx.x % n_tiles;
  const int rest = blockIdx.x / n_tiles;
  const int mt = rest % m_tiles;                // token tile == pages 2 mt, 2 mt + 1
  const int li = rest / m_tiles;
  const int slot = p.live.slot[li];
  const int n_kb = p.hidden / kGK;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int b = 0; b < kNumBars; ++b) mbar_init(bars + b, 1);
    fence_barrier_init();
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

  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tx);
      tma_prefetch_desc(&tw);
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tkv);
      int issued = 0;
      for (int kb = 0; kb < n_kb; ++kb) {
        const int s = kb % kStages;
        if (!wait_bar(ctx, kEmpty0 + s, ((kb / kStages) & 1) ^ 1)) break;
        uint8_t *sa = smem + s * kStageBytes;
        mbar_arrive_expect_tx(bars + kFull0 + s, kStageBytes);
        tma_load_3d(sa, &tx, bars + kFull0 + s, kb * kGK, mt * kGM, slot);
        tma_load_2d(sa + kABytes, &tw, bars + kFull0 + s, kb * kGK, nt * kGN);
        issued = kb + 1;
      }
      // Drain: the last load of every stage has landed before the CTA exits.
      for (int kb = issued - kStages < 0 ? 0 : issued - kStages; kb < issued; ++kb)
        drain_wait(ctx, kFull0 + kb % kStages, (kb / kStages) & 1);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(kPage, kGN, false);
      const uint32_t hi = desc_hi_sw128(1024);
      const uint32_t lo0 = desc_lo_sw128(smem_u32(smem), 16);
      bool ok = true;
      for (int kb = 0; kb < n_kb; ++kb) {
        const int s = kb % kStages;
        if (!wait_bar(ctx, kFull0 + s, (kb / kStages) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_lo = lo0 + ((s * kStageBytes) >> 4);
        const uint32_t b_lo = a_lo + (kABytes >> 4);
#pragma unroll
        for (int k = 0; k < kGK / 16; ++k) {
#pragma unroll
          for (int h = 0; h < 2; ++h)   // rows 128 h .. 128 h + 127 of the A tile
            mma_bf16_ss2(tmem + h * kGN, a_lo + ((h * kPage * 128) >> 4) + k * 2, b_lo + k * 2,
                         hi, idesc, (kb > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(bars + kEmpty0 + s);
      }
      if (ok) mma_commit(bars + kAccFull);
      mma_commit(bars + kDrain);
      drain_wait(ctx, kDrain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    // Warpgroup h drains page h of the tile; warp w holds rows 32 (w % 4) ..
    // +31 (TMEM lanes), thread = one token row. The 256 features of the tile
    // are two heads (head0, head0 + 1) of one section (q, k or v) with the
    // same rotary angles per dimension, so each 32-dimension chunk of both
    // heads is rotated with one set of (cos, sin) loads. Rounded bf16 rows are
    // staged in the drained operand ring (128-byte swizzled, one 16 KB half
    // per 64 dimensions) and every warp writes its 32 rows with TMA stores:
    // q_rot through the activation map (rows past C clipped), K/V straight
    // into the page rows (rows past C are zeros).
    const int h = warp >> 2;                             // page of the tile
    const int page = 2 * mt + h;                         // page of the chunk
    const int wr = (warp & 3) * 32;                      // first row of this warp
    const int r = wr + lane;                             // token row in the page == TMEM lane
    const int n = page * kPage + r;                      // token inside the chunk
    const bool valid = n < p.C;
    const uint32_t lane_addr = static_cast<uint32_t>(wr) << 16;
    const bool ok = __all_sync(0xffffffffu, wait_bar(ctx, kAccFull, 0));
    if (ok && page < p.npc) {
      tc_fence_after();
      int tpos = 0, ypos = 0, xpos = 0;
      if (p.rope && valid) {
        const int hw = p.gh * p.gw;
        tpos = p.F * p.live.chunk[li] + n / hw;
        ypos = (n / p.gw) % p.gh;
        xpos = n % p.gw;
      }
      const int pos = __ldg(p.table + kTabSlotPos + slot);
      int phys = pos < 0 ? -1 : __ldg(p.table + kTabPages + pos * p.npc + page);
      if (phys >= p.num_pages) phys = -1;
      const int f0 = nt * kGN;                           // first output feature of the tile
      const int sec = f0 / p.hidden;                     // 0 q, 1 k, 2 v
      const int head0 = (f0 - sec * p.hidden) / p.d;     // heads head0, head0 + 1
      const bool rot = sec < 2 && p.rope && valid;
      uint8_t *stage = smem + h * 2 * kHeadStage;        // [head slot][64-dim half][128 rows][128 B]
      const int h0 = p.split0 >> 1, h1 = p.split1 >> 1, h2 = p.split2 >> 1;
      const bool kv_ok = sec > 0 && phys >= 0;
      if (lane == 0 && sec > 0 && phys < 0) record_status(p.status, WF_ERR_BAD_PAGE);
      // (cos, sin) of the 16 pairs of dimensions 32 c .. 32 c + 31; the band of
      // a pair is picked by selects, and all 16 loads issue before any use.
      auto load_cs = [&](int c, float2 (&cs)[16]) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int pr = c * 16 + i;
          const float2 *src = pr < h0        ? p.rope_t + tpos * h0 + pr
                              : pr < h0 + h1 ? p.rope_h + ypos * h1 + (pr - h0)
                                             : p.rope_w + xpos * h2 + (pr - h0 - h1);
          cs[i] = __ldg(src);
        }
      };
      // Step s drains dimensions 32 c .. 32 c + 31 (c = s / 2) of head slot
      // hs = s % 2 while the TMEM load of step s + 1 and, on even steps, the
      // (cos, sin) of the next chunk are in flight. The 64-dimension half kt
      // of both heads is complete after steps 3 and 7; its TMA stores are
      // issued at once, so the first half's stores overlap the second half.
      uint32_t cur[32], nxt[32];
      float2 cs[16], csn[16];
      tmem_ld32(tmem + lane_addr + h * kGN, cur);
      if (rot) load_cs(0, cs);
      tmem_ld_wait();
      reg_fence32(cur);
#pragma unroll
      for (int st = 0; st < 8; ++st) {
        const int c = st >> 1, hs = st & 1, kt = c >> 1;
        if (st < 7) {
          const int cn = (st + 1) >> 1, hn = (st + 1) & 1;
          tmem_ld32(tmem + lane_addr + h * kGN + hn * 128 + cn * 32, nxt);
        }
        if (rot && hs == 0 && c < 3) load_cs(c + 1, csn);
        if (rot) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = __uint_as_float(cur[2 * i]), b = __uint_as_float(cur[2 * i + 1]);
            cur[2 * i] = __float_as_uint(a * cs[i].x - b * cs[i].y);
            cur[2 * i + 1] = __float_as_uint(a * cs[i].y + b * cs[i].x);
          }
        }
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = valid ? pack_bf16(__uint_as_float(cur[2 * i]), __uint_as_float(cur[2 * i + 1])) : 0u;
        uint8_t *half = stage + hs * kHeadStage + kt * kHalfStage + r * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int chunk = (c & 1) * 4 + i;             // 16-byte chunk of the 128-byte row
          const uint32_t addr = smem_u32(half + ((chunk ^ (r & 7)) << 4));
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[4 * i]),
                       "r"(w[4 * i + 1]), "r"(w[4 * i + 2]), "r"(w[4 * i + 3])
                       : "memory");
        }
        if (st == 3 || st == 7) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint8_t *src = stage + hh * kHeadStage + kt * kHalfStage + wr * 128;
              if (sec == 0) {
                if (page * kPage + wr < p.C)            // boxes wholly past C are skipped
                  tma_store_4d(&tq, src, kt * 64, head0 + hh, page * kPage + wr, slot);
              } else if (kv_ok) {
                const int64_t row = p.layer_row0 +
                    ((static_cast<int64_t>(phys) * 2 + (sec - 1)) * p.Hh + head0 + hh) * p.P + wr;
                tma_store_2d(&tkv, src, kt * 64, static_cast<int>(row));
              }
            }
            tma_store_commit();
          }
        }
        if (st < 7) {
          tmem_ld_wait();
          reg_fence32(nxt);
#pragma unroll
          for (int i = 0; i < 32; ++i) cur[i] = nxt[i];
        }
        if (rot && hs == 1 && c < 3) {
#pragma unroll
          for (int i = 0; i < 16; ++i) cs[i] = csn[i];
        }
      }
      if (lane == 0) {
        tma_store_wait_all();                            // the staging smem stays live until read
        if (sec == 1 && head0 == 0 && wr == 0 && kv_ok) p.tags[phys] = p.live.tag[li];
      }
      __syncwarp();
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

cudaError_t launch_project_bf16(const ProjectParams &p, const void *tmap_x, const void *tmap_w,
                                const void *tmap_q, const void *tmap_kv, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  if (p.d != 128 || p.P != kPage || p.hidden % kGN != 0) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t blocks = static_cast<int64_t>(p.live.n) * ((p.npc + 1) / 2) * (3 * p.hidden / kGN);
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  project_kernel<<<static_cast<unsigned>(blocks), kThreads, kSmemBytes, st>>>(
      p, *static_cast<const CUtensorMap *>(tmap_x), *static_cast<const CUtensorMap *>(tmap_w),
      *static_cast<const CUtensorMap *>(tmap_q), *static_cast<const CUtensorMap *>(tmap_kv));
  return cudaGetLastError();
}

}  // namespace wf
