// Early publication into an FP8 (E4M3) pool: rotary embedding, block scaling
// and quantisation of q, k and v, scatter into the paged pool.
//
// "Wave Forcing: Towards Speed-of-Light Streaming Video Generation": K/V are
// published right after the QKV projection and RoPE into ordered attention
// slots (Method section), and travel as FP8 payload plus scale factors
// (Appendix Table 8). Storage format of this library's FP8 pool:
//   * E4M3 codes (round to nearest even, saturating);
//   * one power-of-two scale 2^e per block, e the smallest integer with
//     amax * 2^-e <= 448 (clamped below at -100); a block is one page (128
//     tokens) of one head for K and for V, and one 128-row query tile of one
//     head for q_rot;
//   * q and k are rotated in fp32 with every product and sum rounded once
//     (no fused multiply-add), so the codes do not depend on compiler
//     contraction choices.
//
// Work unit: one block of one tensor, i.e. (live slot, page j, head, q|k|v):
// 128 token rows x 128 dims of bf16 in (32 KB), 16 KB of codes and one scale
// out. q, k and v of a (slot, page, head) are independent units, since each
// has its own scale. The kernel is persistent, one CTA per SM walking the
// units blockIdx.x, blockIdx.x + gridDim.x, ... through a six-stage
// shared-memory ring:
//   * a TMA warp loads each unit's tile (box 128 dims x 1 head x 128 rows,
//     rows past C zero-filled); once the unit is quantised it stores the codes
//     from the same stage: q_rot through a tensor map over the codes (rows
//     past C clipped), a K or V page block (16 KB, contiguous in the pool) as
//     one bulk copy; it writes the block's scale, stamps the page's ready tag
//     (at the K block of head 0) and refills the stage with the unit six steps
//     ahead once the stores have read it;
//   * 512 threads, 16 per row (8 dims = 16 bytes each), 32 rows per pass, 4
//     passes: the (cos, sin) entries of the thread's rows are loaded before
//     the wait for the tile; pass 1 rotates q and k in registers and takes the
//     block maximum (warp max, then one named barrier over the 16 warps);
//     pass 2 scales by 2^-e, converts to E4M3 and writes the codes in place
//     over the stage (row r at byte 128 r: every thread has read the tile by
//     the barrier). Rows past C are +0 in the tile and stay +0 (rotating them
//     could turn +0 into -0), so the K and V page blocks get zero codes there.
// HBM-bound: 2 bytes read and 1 written per (token, head, dim) of q, k and v.
#include <cuda.h>
#include <cuda_bf16.h>

#include "f32x2.cuh"
#include "pipeline.cuh"
#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {
namespace {

using namespace sm100;

constexpr int kRows = 128;                              // rows per block (page / query tile)
constexpr int kComputeThreads = 512;
constexpr int kComputeWarps = kComputeThreads / 32;     // 16
constexpr int kThreads = kComputeThreads + 32;          // + the TMA warp
constexpr int kTPR = 16;                                // threads per row
constexpr int kRowsPerPass = kComputeThreads / kTPR;    // 32
constexpr int kPasses = kRows / kRowsPerPass;           // 4
constexpr uint32_t kTileBytes = kRows * 128 * 2;        // one bf16 tile, 32 KB
constexpr uint32_t kCodeBytes = kRows * 128;            // its codes, 16 KB
constexpr int kStages = 6;
constexpr uint32_t kOffBars = kStages * kTileBytes;     // full[kStages], quantised[kStages]
constexpr uint32_t kOffExp = kOffBars + 2 * kStages * 8;          // int [kStages]
constexpr uint32_t kOffRed = kOffExp + kStages * 4;               // uint32 [2][kComputeWarps]
constexpr uint32_t kOffMisc = kOffRed + 2 * kComputeWarps * 4;    // abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
enum { kFull0 = 0, kQuant0 = kStages };

// Smallest e with amax * 2^-e <= 448 = 1.75 * 2^8, clamped below at -100:
// for amax = f * 2^E (f in [1, 2)), e = E - 8 if f <= 1.75, else E - 7.
// Zero and subnormal amax give -100.
__device__ __forceinline__ int scale_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ef = static_cast<int>((b >> 23) & 0xFFu);
  if (ef == 0) return -100;
  const int E = ef - 127;
  const int e = (b & 0x7FFFFFu) <= 0x600000u ? E - 8 : E - 7;
  return e < -100 ? -100 : e;
}

// 2^k for -126 <= k <= 127, exactly.
__device__ __forceinline__ float exp2i(int k) { return __uint_as_float(static_cast<uint32_t>(k + 127) << 23); }

__device__ __forceinline__ void widen(const uint4 &u, float *f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Running max of |x| over the 8 bf16 values of a 16-byte vector, kept as a
// bf16 pair (exact: max and abs do not round).
__device__ __forceinline__ uint32_t absmax_bf16x8(uint32_t m, const uint4 &u) {
  const uint32_t w[4] = {u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu, u.z & 0x7FFF7FFFu, u.w & 0x7FFF7FFFu};
#pragma unroll
  for (int i = 0; i < 4; ++i) asm("max.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(w[i]));
  return m;
}

// (a c - b s, a s + b c) for 4 pairs, each product and sum rounded once.
__device__ __forceinline__ void rotate8(float *v, const float2 (&cs)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = v[2 * i], b = v[2 * i + 1];
    v[2 * i] = __fsub_rn(__fmul_rn(a, cs[i].x), __fmul_rn(b, cs[i].y));
    v[2 * i + 1] = __fadd_rn(__fmul_rn(a, cs[i].y), __fmul_rn(b, cs[i].x));
  }
}

// 8 values times the power of two `mul` (exact unless it underflows), as E4M3.
__device__ __forceinline__ uint2 quant8(const float *v, float mul) {
  const uint64_t m2 = f2(mul, mul);
  float y[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) unf2(fmul2(f2(v[2 * i], v[2 * i + 1]), m2), y[2 * i], y[2 * i + 1]);
  uint2 w;
  w.x = pack_e4m3x4(y[0], y[1], y[2], y[3]);
  w.y = pack_e4m3x4(y[4], y[5], y[6], y[7]);
  return w;
}

struct Unit {
  int li, j, h, t;   // live slot index, page of the chunk, head, tensor (0 q, 1 k, 2 v)
};

__device__ __forceinline__ Unit decode(int b, const PublishParams &p) {
  Unit u;
  u.t = b % 3;
  const int blk = b / 3;
  const int per_slot = p.npc * p.Hh;
  u.li = blk / per_slot;
  const int rem = blk - u.li * per_slot;
  u.j = rem / p.Hh;
  u.h = rem - u.j * p.Hh;
  return u;
}

// Physical page holding page j of a slot's chunk (-1 if the table is bad).
__device__ __forceinline__ int block_page(const PublishParams &p, int slot, int j) {
  const int tpos = __ldg(p.table + kTabSlotPos + slot);
  const int phys = tpos < 0 ? -1 : __ldg(p.table + kTabPages + tpos * p.npc + j);
  return (phys < 0 || phys >= p.num_pages) ? -1 : phys;
}

// The TMA load of unit b's tile into stage buffer `buf`.
__device__ __forceinline__ void load_unit(int b, uint8_t *buf, uint64_t *bar,
                                          const PublishParams &p, const CUtensorMap *tq,
                                          const CUtensorMap *tk, const CUtensorMap *tv) {
  const Unit u = decode(b, p);
  const int slot = p.live.slot[u.li];
  mbar_arrive_expect_tx(bar, kTileBytes);
  tma_load_4d(buf, u.t == 0 ? tq : (u.t == 1 ? tk : tv), bar, 0, u.h, u.j * kRows, slot);
}

// Max over the 512 compute threads (named barrier 1) of non-negative floats
// compared as bit patterns (the same order for every non-negative value, NaN
// above +inf), the same result in every one of them. `red` holds one value
// per warp. A thread passes kAbortBits (above every non-negative pattern)
// when its wait ran out, so that all threads leave at the same unit.
constexpr uint32_t kAbortBits = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t compute_max(uint32_t bits, uint32_t *red) {
  const uint32_t w = __reduce_max_sync(0xffffffffu, bits);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = w;
  asm volatile("bar.sync 1, %0;" ::"n"(kComputeThreads) : "memory");
  uint32_t m = red[0];
#pragma unroll
  for (int i = 1; i < kComputeWarps; ++i) m = max(m, red[i]);
  return m;
}

__global__ void __launch_bounds__(kThreads, 1)
    publish_fp8_kernel(const __grid_constant__ PublishParams p,
                       const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv,
                       const __grid_constant__ CUtensorMap tqr) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
  volatile int *exps = reinterpret_cast<volatile int *>(smem + kOffExp);
  uint32_t *red = reinterpret_cast<uint32_t *>(smem + kOffRed);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc);
  const int nunits = p.live.n * p.npc * p.Hh * 3;
  const int G = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Ctx ctx{bars, abort_flag, p.status};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + kFull0 + s, 1);
      mbar_init(bars + kQuant0 + s, kComputeWarps);
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
      int issued[kStages] = {};
      for (int s = 0; s < kStages; ++s) {
        const int b = blockIdx.x + s * G;
        if (b < nunits) {
          load_unit(b, smem + s * kTileBytes, bars + kFull0 + s, p, &tq, &tk, &tv);
          ++issued[s];
        }
      }
      for (int i = 0;; ++i) {
        const int b = blockIdx.x + i * G;
        if (b >= nunits) break;
        const int s = i % kStages;
        if (!wait_bar(ctx, kQuant0 + s, (i / kStages) & 1)) break;
        const Unit u = decode(b, p);
        const int slot = p.live.slot[u.li];
        const float scale = exp2i(exps[s]);
        const uint8_t *buf = smem + s * kTileBytes;
        if (u.t == 0) {
          tma_store_4d(&tqr, buf, 0, u.h, u.j * kRows, slot);
          p.q_scale[(static_cast<size_t>(slot) * p.npc + u.j) * p.Hh + u.h] = scale;
        } else {
          const int phys = block_page(p, slot, u.j);
          if (phys >= 0) {
            const size_t blk = (static_cast<size_t>(phys) * 2 + (u.t - 1)) * p.Hh + u.h;
            bulk_store(reinterpret_cast<uint8_t *>(p.pages) + blk * kCodeBytes, buf, kCodeBytes);
            p.kv_scale[blk] = scale;
            if (u.t == 1 && u.h == 0) p.tags[phys] = p.live.tag[u.li];
          } else {
            record_status(p.status, WF_ERR_BAD_PAGE);
          }
        }
        tma_store_commit();
        // Refill the previous unit's stage once its stores have read it (the
        // store just issued may still be reading this one).
        if (i > 0) {
          const int bp = b - G + kStages * G;
          if (bp < nunits) {
            const int sp = (i - 1) % kStages;
            tma_store_wait_read_but_last();
            load_unit(bp, smem + sp * kTileBytes, bars + kFull0 + sp, p, &tq, &tk, &tv);
            ++issued[sp];
          }
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
    if (b >= nunits) break;
    const int s = i % kStages;
    const Unit u = decode(b, p);
    const bool rot = p.rope && u.t < 2;
    // The (cos, sin) entries of this thread's rows are loaded while the tile
    // is still in flight. Rotary positions are absolute: frame F * chunk +
    // n / (gh gw), row y, column x.
    float2 cs[kPasses][4];
    if (rot) {
      const int hw = p.gh * p.gw, t0 = p.F * p.live.chunk[u.li];
#pragma unroll
      for (int ps = 0; ps < kPasses; ++ps) {
        int n = u.j * kRows + r0 + ps * kRowsPerPass;
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
    uint8_t *buf = smem + s * kTileBytes;
    float x[kPasses][8];
    float amax = 0.0f;
    if (!ok) {
      // nothing to read: the tile never arrived
    } else if (u.t < 2) {
#pragma unroll
      for (int ps = 0; ps < kPasses; ++ps) {
        const int r = r0 + ps * kRowsPerPass;
        widen(*reinterpret_cast<const uint4 *>(buf + r * 256 + cv * 16), x[ps]);
        if (rot && u.j * kRows + r < p.C) rotate8(x[ps], cs[ps]);   // rows past C stay +0
#pragma unroll
        for (int c = 0; c < 8; c += 2) amax = max3(amax, fabsf(x[ps][c]), fabsf(x[ps][c + 1]));
      }
    } else {
      uint32_t av = 0;
#pragma unroll
      for (int ps = 0; ps < kPasses; ++ps) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(buf + (r0 + ps * kRowsPerPass) * 256 + cv * 16);
        av = absmax_bf16x8(av, raw);
        widen(raw, x[ps]);
      }
      amax = fmaxf(__uint_as_float(av << 16), __uint_as_float(av & 0xFFFF0000u));
    }
    const uint32_t m = compute_max(ok ? __float_as_uint(amax) : kAbortBits,
                                   red + (i & 1) * kComputeWarps);
    if (m == kAbortBits) break;
    const int e = scale_exponent(__uint_as_float(m));
    const float mul = exp2i(-e);
#pragma unroll
    for (int ps = 0; ps < kPasses; ++ps) {
      const int r = r0 + ps * kRowsPerPass;
      const uint2 w = quant8(x[ps], mul);
      asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(smem_u32(buf + r * 128 + cv * 8)),
                   "r"(w.x), "r"(w.y)
                   : "memory");
    }
    if (threadIdx.x == 0) exps[s] = e;
    // The codes are read by the TMA / bulk stores (async proxy).
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + kQuant0 + s);
  }
}

}  // namespace

cudaError_t launch_publish_fp8(const PublishParams &p, const void *tmap_q, const void *tmap_k,
                               const void *tmap_v, const void *tmap_qrot, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  if (p.d != 128 || p.P != kRows) return cudaErrorInvalidValue;
  const int64_t nunits = static_cast<int64_t>(p.live.n) * p.npc * p.Hh * 3;
  if (nunits > 0x7fffffff) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(publish_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(nunits < sms ? nunits : sms);
  publish_fp8_kernel<<<grid, kThreads, kSmemBytes, st>>>(
      p, *static_cast<const CUtensorMap *>(tmap_q), *static_cast<const CUtensorMap *>(tmap_k),
      *static_cast<const CUtensorMap *>(tmap_v), *static_cast<const CUtensorMap *>(tmap_qrot));
  return cudaGetLastError();
}

}  // namespace wf
