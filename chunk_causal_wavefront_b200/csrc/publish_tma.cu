// Early K/V publication into a bf16 pool with 128-token pages and d = 128:
// rotary embedding + scatter of (page, head) tiles, half a page at a time,
// through TMA.
//
// "Wave Forcing: Towards Speed-of-Light Streaming Video Generation", Method
// section: K/V are published right after the QKV projection and RoPE, and
// paged delivery writes them directly into ordered attention slots, followed
// by a ready signal (here a per-page tag).
//
// Work unit: one half of a (live slot, page j, head) block, i.e. 64 token rows
// x 128 dims of q, k and v (48 KB of bf16 in, 48 KB out). The kernel is
// persistent, one CTA per SM walking the units blockIdx.x, blockIdx.x +
// gridDim.x, ... through a four-stage shared-memory ring (half-page units in
// four stages timed 3 % faster than whole pages in two, quarter pages slower):
//   * a TMA warp loads a unit's q, k and v tiles (box 128 dims x 1 head x 64
//     rows, rows past C zero-filled), and once the unit is rotated stores the
//     q_rot tile (rows past C clipped by the tensor map) and the K and V tiles
//     into the unit's half of the page (a 2D map over the layer's pool rows);
//     it refills the stage with the unit four steps ahead as soon as the
//     stores have read it;
//   * 512 threads rotate q and k in place in shared memory, 16 threads per row
//     (16 bytes = 4 rotary pairs each), in fp32 with one rounding to bf16;
//     rows past C stay +0 (rotating them could turn +0 into -0); V is stored
//     as loaded.
// HBM-bound: every element is read once and written once.
#include <cuda.h>
#include <cuda_bf16.h>

#include "pipeline.cuh"
#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {
namespace {

using namespace sm100;

constexpr int kRows = 64;                              // token rows per unit (half a page)
constexpr int kPage = 128;                             // token rows per page
constexpr int kSplit = kPage / kRows;                  // units per (page, head)
constexpr int kComputeThreads = 512;
constexpr int kComputeWarps = kComputeThreads / 32;    // 16
constexpr int kThreads = kComputeThreads + 32;         // + the TMA warp
constexpr int kTPR = 16;                               // threads per row
constexpr int kRowsPerPass = kComputeThreads / kTPR;   // 32
constexpr int kPasses = kRows / kRowsPerPass;          // 2
constexpr uint32_t kTileBytes = kRows * 128 * 2;       // one bf16 tile, 16 KB
constexpr uint32_t kStageBytes = 3 * kTileBytes;       // q, k, v
constexpr int kStages = 4;
constexpr uint32_t kOffBars = kStages * kStageBytes;   // full[kStages], rotated[kStages]
constexpr uint32_t kOffMisc = kOffBars + 2 * kStages * 8;  // abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
enum { kFull0 = 0, kRotated0 = kStages };

struct Unit {
  int li, j, h, row0, part;
};

__device__ __forceinline__ Unit decode(int b, const PublishParams &p) {
  Unit k;
  const int per_slot = p.npc * kSplit * p.Hh;
  k.li = b / per_slot;
  const int rem = b - k.li * per_slot;
  const int jp = rem / p.Hh;
  k.h = rem - jp * p.Hh;
  k.j = jp / kSplit;
  k.part = jp - k.j * kSplit;
  k.row0 = k.j * kPage + k.part * kRows;
  return k;
}

// Physical page holding page j of live slot li's chunk (-1 if the table is bad).
__device__ __forceinline__ int block_page(const PublishParams &p, int slot, int j) {
  const int tpos = __ldg(p.table + kTabSlotPos + slot);
  const int phys = tpos < 0 ? -1 : __ldg(p.table + kTabPages + tpos * p.npc + j);
  return (phys < 0 || phys >= p.num_pages) ? -1 : phys;
}

// The three TMA tile loads of unit b into stage buffer `buf`.
__device__ __forceinline__ void load_unit(int b, uint8_t *buf, uint64_t *bar,
                                           const PublishParams &p, const CUtensorMap *tq,
                                           const CUtensorMap *tk, const CUtensorMap *tv) {
  const Unit k = decode(b, p);
  const int slot = p.live.slot[k.li];
  mbar_arrive_expect_tx(bar, kStageBytes);
  tma_load_4d(buf, tq, bar, 0, k.h, k.row0, slot);
  tma_load_4d(buf + kTileBytes, tk, bar, 0, k.h, k.row0, slot);
  tma_load_4d(buf + 2 * kTileBytes, tv, bar, 0, k.h, k.row0, slot);
}

// OR of a predicate over the 512 compute threads (named barrier 1), the same
// result in every one of them.
__device__ __forceinline__ bool compute_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kComputeThreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void rotate_vec(uint4 &u, const float2 (&cs)[4]) {
  uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = __uint_as_float(w[i] << 16), b = __uint_as_float(w[i] & 0xFFFF0000u);
    // Each product and sum rounded once (no contraction into FMAs), then one
    // rounding to bf16: the published values are a function of the inputs alone.
    __nv_bfloat162 r = __floats2bfloat162_rn(__fsub_rn(__fmul_rn(a, cs[i].x), __fmul_rn(b, cs[i].y)),
                                             __fadd_rn(__fmul_rn(a, cs[i].y), __fmul_rn(b, cs[i].x)));
    w[i] = *reinterpret_cast<uint32_t *>(&r);
  }
  u = make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(kThreads, 1)
    publish_tma_kernel(const __grid_constant__ PublishParams p,
                       const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv,
                       const __grid_constant__ CUtensorMap tqr,
                       const __grid_constant__ CUtensorMap tpg) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc);
  const int nblk = p.live.n * p.npc * kSplit * p.Hh;
  const int G = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Ctx ctx{bars, abort_flag, p.status};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + kFull0 + s, 1);
      mbar_init(bars + kRotated0 + s, kComputeWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------ TMA warp --
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      tma_prefetch_desc(&tqr);
      tma_prefetch_desc(&tpg);
      int issued[kStages] = {};
      for (int s = 0; s < kStages; ++s) {
        const int b = blockIdx.x + s * G;
        if (b < nblk) {
          load_unit(b, smem + s * kStageBytes, bars + kFull0 + s, p, &tq, &tk, &tv);
          ++issued[s];
        }
      }
      for (int i = 0;; ++i) {
        const int b = blockIdx.x + i * G;
        if (b >= nblk) break;
        const int s = i % kStages;
        if (!wait_bar(ctx, kRotated0 + s, (i / kStages) & 1)) break;
        const Unit blk = decode(b, p);
        const int slot = p.live.slot[blk.li];
        const int phys = block_page(p, slot, blk.j);
        const uint8_t *buf = smem + s * kStageBytes;
        tma_store_4d(&tqr, buf, 0, blk.h, blk.row0, slot);
        if (phys >= 0) {
          const int rowk = (phys * 2 * p.Hh + blk.h) * kPage + blk.part * kRows;
          tma_store_2d(&tpg, buf + kTileBytes, 0, rowk);
          tma_store_2d(&tpg, buf + 2 * kTileBytes, 0, rowk + p.Hh * kPage);
          if (blk.h == 0 && blk.part == 0) p.tags[phys] = p.live.tag[blk.li];
        } else {
          record_status(p.status, WF_ERR_BAD_PAGE);
        }
        tma_store_commit();
        // Refill the stage with the unit kStages ahead once the stores have read it.
        if (b + kStages * G < nblk) {
          tma_store_wait_read_all();
          load_unit(b + kStages * G, smem + s * kStageBytes, bars + kFull0 + s, p, &tq, &tk, &tv);
          ++issued[s];
        }
      }
      // Every store has written global memory and every load has landed
      // before the CTA exits (only an aborted loop leaves loads behind).
      tma_store_wait_all();
      for (int s = 0; s < kStages; ++s)
        if (issued[s]) drain_wait(ctx, kFull0 + s, (issued[s] - 1) & 1);
    }
    return;
  }

  // -------------------------------------------------------- compute warps --
  const int cv = threadIdx.x & (kTPR - 1);        // 16-byte vector of the head row
  const int r0 = threadIdx.x / kTPR;              // first row of this thread
  // Rotary (cos, sin) entries of this thread's 4 pairs (pairs 4 cv .. 4 cv + 3):
  // pair pr lies in band t, h or w (band index b); its entry for a row is
  // rope_t[o + q_b], o the pair's offset from the t table (the three tables
  // share the pool buffer) and q_b the row's position in band b times that
  // band's pair count. ctab[i] packs 4 o + b.
  const int h0 = p.split0 >> 1, h1 = p.split1 >> 1, h2 = p.split2 >> 1;
  int ctab[4] = {0, 0, 0, 0};
  if (p.rope) {
    const int oh = static_cast<int>(p.rope_h - p.rope_t), ow = static_cast<int>(p.rope_w - p.rope_t);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int pr = cv * 4 + i;
      if (pr < h0) ctab[i] = 4 * pr;
      else if (pr < h0 + h1) ctab[i] = 4 * (oh + pr - h0) + 1;
      else ctab[i] = 4 * (ow + pr - h0 - h1) + 2;
    }
  }
  for (int i = 0;; ++i) {
    const int b = blockIdx.x + i * G;
    if (b >= nblk) break;
    const int s = i % kStages;
    const Unit blk = decode(b, p);
    // The (cos, sin) entries of this thread's rows and pairs are loaded while
    // the unit's tiles are still in flight. Rotary positions are absolute:
    // frame F * chunk + n / (gh gw), row y, column x.
    float2 cs[kPasses][4];
    if (p.rope) {
      const int hw = p.gh * p.gw, t0 = p.F * p.live.chunk[blk.li];
#pragma unroll
      for (int ps = 0; ps < kPasses; ++ps) {
        int n = blk.row0 + r0 + ps * kRowsPerPass;
        if (n >= p.C) n = 0;
        const int f = n / hw, yx = n - f * hw, y = yx / p.gw;
        const int pt = (t0 + f) * h0, py = y * h1, px = (yx - y * p.gw) * h2;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int band = ctab[c] & 3;
          cs[ps][c] = __ldg(p.rope_t + (ctab[c] >> 2) + (band == 0 ? pt : band == 1 ? py : px));
        }
      }
    }
    // The n-th use of a stage waits for its n-th fill: parity (i / kStages) & 1.
    const bool ok = __all_sync(0xffffffffu, wait_bar(ctx, kFull0 + s, (i / kStages) & 1));
    if (compute_any(!ok)) break;

    if (p.rope) {
      uint8_t *buf = smem + s * kStageBytes;
#pragma unroll
      for (int ps = 0; ps < kPasses; ++ps) {
        const int r = r0 + ps * kRowsPerPass;
        if (blk.row0 + r >= p.C) continue;       // zero rows past C stay +0
        const uint32_t off = r * 256 + cv * 16;
        uint4 *qa = reinterpret_cast<uint4 *>(buf + off);
        uint4 *ka = reinterpret_cast<uint4 *>(buf + kTileBytes + off);
        uint4 qv = *qa, kv = *ka;
        rotate_vec(qv, cs[ps]);
        rotate_vec(kv, cs[ps]);
        *qa = qv;
        *ka = kv;
      }
    }
    // The rotated tiles are read by the TMA stores (async proxy).
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + kRotated0 + s);
  }
}

}  // namespace

cudaError_t launch_publish_bf16_tma(const PublishParams &p, const void *tmap_q, const void *tmap_k,
                                    const void *tmap_v, const void *tmap_qrot,
                                    const void *tmap_pages, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  if (p.d != 128 || p.P != kPage) return cudaErrorInvalidValue;
  const int64_t nblk = static_cast<int64_t>(p.live.n) * p.npc * kSplit * p.Hh;
  if (nblk > 0x7fffffff) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(publish_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(nblk < sms ? nblk : sms);
  publish_tma_kernel<<<grid, kThreads, kSmemBytes, st>>>(
      p, *static_cast<const CUtensorMap *>(tmap_q), *static_cast<const CUtensorMap *>(tmap_k),
      *static_cast<const CUtensorMap *>(tmap_v), *static_cast<const CUtensorMap *>(tmap_qrot),
      *static_cast<const CUtensorMap *>(tmap_pages));
  return cudaGetLastError();
}

}  // namespace wf
