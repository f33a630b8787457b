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
// Work unit: one (live slot, page j, head) block, i.e. 128 token rows x 128
// dims of q, k and v (96 KB of bf16 in, 48 KB of codes out). The kernel is a
// persistent streaming loop, one CTA per SM, each walking the blocks
// blockIdx.x, blockIdx.x + gridDim.x, ...:
//   * thread 0 loads the next-but-one block's q, k and v tiles with TMA into a
//     two-stage shared-memory ring (box 128 dims x 1 head x 128 rows, rows past
//     C zero-filled), so HBM reads of block i+1 overlap the work on block i;
//   * 512 threads, 16 per row (8 dims = 16 bytes each), 32 rows per pass, 4
//     passes: pass 1 rotates q and k (kept in registers) and takes the three
//     block maxima (warp max, then shared memory across the 16 warps); pass 2
//     scales by 2^-e, converts to E4M3 and writes 8 bytes per row and thread
//     (q_rot rows < C, and the whole 128-row K and V page blocks, whose rows
//     past C are zero codes).
// HBM-bound: 6 bytes read and 3 written per (token, head, dim).
#include <cuda.h>
#include <cuda_bf16.h>

#include "f32x2.cuh"
#include "pipeline.cuh"
#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {
namespace {

using namespace sm100;

constexpr int kRows = 128;                     // rows per block (page / query tile)
constexpr int kThreads = 512;
constexpr int kTPR = 16;                       // threads per row
constexpr int kRowsPerPass = kThreads / kTPR;  // 32
constexpr int kPasses = kRows / kRowsPerPass;  // 4
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kTensorBytes = kRows * 128 * 2;      // one bf16 tile, 32 KB
constexpr uint32_t kStageBytes = 3 * kTensorBytes;      // q, k, v
constexpr uint32_t kOffBars = 2 * kStageBytes;          // two stages
constexpr uint32_t kOffRed = kOffBars + 64;             // [3][kWarps] block maxima
constexpr uint32_t kOffPos = kOffRed + 3 * kWarps * 4;  // [kRows][4] rotary table offsets
constexpr uint32_t kSmemBytes = kOffPos + 4 * kRows * 4 + 1024;

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

struct Block {
  int li, j, h;
};

__device__ __forceinline__ Block decode(int b, const PublishParams &p) {
  Block k;
  const int per_slot = p.npc * p.Hh;
  k.li = b / per_slot;
  const int rem = b - k.li * per_slot;
  k.j = rem / p.Hh;
  k.h = rem - k.j * p.Hh;
  return k;
}

// Thread 0: the three TMA tile loads of block b into stage buffer `buf`.
__device__ __forceinline__ void load_block(int b, uint8_t *buf, uint64_t *bar,
                                           const PublishParams &p, const CUtensorMap *tq,
                                           const CUtensorMap *tk, const CUtensorMap *tv) {
  const Block k = decode(b, p);
  const int slot = p.live.slot[k.li];
  mbar_arrive_expect_tx(bar, kStageBytes);
  tma_load_4d(buf, tq, bar, 0, k.h, k.j * kRows, slot);
  tma_load_4d(buf + kTensorBytes, tk, bar, 0, k.h, k.j * kRows, slot);
  tma_load_4d(buf + 2 * kTensorBytes, tv, bar, 0, k.h, k.j * kRows, slot);
}

// Block-wide maxima of three non-negative values (every thread gets them).
__device__ __forceinline__ void block_max3(float (&a)[3], float *red) {
  const int warp = threadIdx.x >> 5;
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    const uint32_t w = __reduce_max_sync(0xffffffffu, __float_as_uint(a[t]));
    if ((threadIdx.x & 31) == 0) red[t * kWarps + warp] = __uint_as_float(w);
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    float m = red[t * kWarps];
#pragma unroll
    for (int i = 1; i < kWarps; ++i) m = fmaxf(m, red[t * kWarps + i]);
    a[t] = m;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    publish_fp8_kernel(const __grid_constant__ PublishParams p,
                       const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kOffBars);   // [2]
  float *red = reinterpret_cast<float *>(smem + kOffRed);
  int32_t *pos = reinterpret_cast<int32_t *>(smem + kOffPos);      // [row][t, h, w, -]
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBars + 16);
  const int nblk = p.live.n * p.npc * p.Hh;
  const int G = gridDim.x;
  const int cv = threadIdx.x & (kTPR - 1);        // 16-byte vector of the head row
  const int r0 = threadIdx.x / kTPR;              // first row of this thread
  const Ctx ctx{full, abort_flag, p.status};
  // Rotary (cos, sin) entries of this thread's 4 pairs (pairs 4 cv .. 4 cv + 3):
  // pair pr lies in band t, h or w (band index b); its entry for row r is
  // rope_t[o + pos[4 r + b]], o the pair's offset from the t table (the three
  // tables share the pool buffer) and pos the row's position in each band
  // times that band's pair count. ctab[i] packs 4 o + b.
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

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(full + 1, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  __syncthreads();
  int issued0 = 0, issued1 = 0;                   // loads issued per stage (thread 0)
  if (threadIdx.x == 0) {
    if (static_cast<int>(blockIdx.x) < nblk) {
      load_block(blockIdx.x, smem, full, p, &tq, &tk, &tv);
      ++issued0;
    }
    if (static_cast<int>(blockIdx.x) + G < nblk) {
      load_block(blockIdx.x + G, smem + kStageBytes, full + 1, p, &tq, &tk, &tv);
      ++issued1;
    }
  }

  for (int i = 0;; ++i) {
    const int b = blockIdx.x + i * G;
    if (b >= nblk) break;
    const int stage = i & 1;
    const Block blk = decode(b, p);
    const int li = blk.li, j = blk.j, h = blk.h;
    const int slot = p.live.slot[li];
    const int tpos = __ldg(p.table + kTabSlotPos + slot);
    int phys = tpos < 0 ? -1 : __ldg(p.table + kTabPages + tpos * p.npc + j);
    if (phys >= p.num_pages) phys = -1;
    if (phys < 0 && threadIdx.x == 0) record_status(p.status, WF_ERR_BAD_PAGE);

    // Rotary positions of the block's rows (absolute: frame F * chunk + n / (gh gw)).
    if (p.rope && threadIdx.x < kRows) {
      int n = j * kRows + threadIdx.x;
      if (n >= p.C) n = 0;
      const int hw = p.gh * p.gw, f = n / hw, yx = n - f * hw, y = yx / p.gw;
      pos[4 * threadIdx.x] = (p.F * p.live.chunk[li] + f) * h0;
      pos[4 * threadIdx.x + 1] = y * h1;
      pos[4 * threadIdx.x + 2] = (yx - y * p.gw) * h2;
    }
    // The n-th use of a stage waits for its n-th fill: parity (i / 2) & 1.
    const bool ok = __all_sync(0xffffffffu, wait_bar(ctx, stage, (i >> 1) & 1));
    if (__syncthreads_or(!ok)) break;             // also publishes pos[] to all threads

    const uint8_t *buf = smem + stage * kStageBytes;
    float xq[kPasses][8], xk[kPasses][8];
    uint4 rv[kPasses];
    float aq = 0.0f, ak = 0.0f;
    uint32_t av = 0;
#pragma unroll
    for (int ps = 0; ps < kPasses; ++ps) {
      const int r = r0 + ps * kRowsPerPass;
      const uint32_t off = r * 256 + cv * 16;
      widen(*reinterpret_cast<const uint4 *>(buf + off), xq[ps]);
      widen(*reinterpret_cast<const uint4 *>(buf + kTensorBytes + off), xk[ps]);
      rv[ps] = *reinterpret_cast<const uint4 *>(buf + 2 * kTensorBytes + off);
      // rows past C stay +0 (zero codes): rotating them could turn +0 into -0
      if (p.rope && j * kRows + r < p.C) {
        float2 cs[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) cs[c] = __ldg(p.rope_t + (ctab[c] >> 2) + pos[4 * r + (ctab[c] & 3)]);
        rotate8(xq[ps], cs);
        rotate8(xk[ps], cs);
      }
#pragma unroll
      for (int c = 0; c < 8; c += 2) {
        aq = max3(aq, fabsf(xq[ps][c]), fabsf(xq[ps][c + 1]));
        ak = max3(ak, fabsf(xk[ps][c]), fabsf(xk[ps][c + 1]));
      }
      av = absmax_bf16x8(av, rv[ps]);
    }
    float amax[3] = {aq, ak, fmaxf(__uint_as_float(av << 16), __uint_as_float(av & 0xFFFF0000u))};
    block_max3(amax, red);
    // Every thread has read this stage (and red[]): thread 0 refills the stage
    // with the next-but-one block while the codes below are written.
    __syncthreads();
    if (threadIdx.x == 0 && b + 2 * G < nblk) {
      load_block(b + 2 * G, smem + stage * kStageBytes, full + stage, p, &tq, &tk, &tv);
      if (stage) ++issued1; else ++issued0;
    }

    const int eq = scale_exponent(amax[0]), ek = scale_exponent(amax[1]), ev = scale_exponent(amax[2]);
    const float mq = exp2i(-eq), mk = exp2i(-ek), mv = exp2i(-ev);
    const size_t slot_off = static_cast<size_t>(slot) * p.C * p.Hh * p.d;
    uint8_t *qdst = static_cast<uint8_t *>(p.q_rot) + slot_off + static_cast<size_t>(h) * p.d + cv * 8;
    const size_t kblk = (static_cast<size_t>(phys < 0 ? 0 : phys) * 2) * p.Hh + h;
    uint8_t *kdst = reinterpret_cast<uint8_t *>(p.pages) + kblk * p.P * p.d + cv * 8;
    uint8_t *vdst = kdst + static_cast<size_t>(p.Hh) * p.P * p.d;
    if (threadIdx.x == 0) {
      p.q_scale[(static_cast<size_t>(slot) * p.npc + j) * p.Hh + h] = exp2i(eq);
      if (phys >= 0) {
        p.kv_scale[kblk] = exp2i(ek);
        p.kv_scale[kblk + p.Hh] = exp2i(ev);
      }
    }
#pragma unroll
    for (int ps = 0; ps < kPasses; ++ps) {
      const int r = r0 + ps * kRowsPerPass;
      const int n = j * kRows + r;
      if (n < p.C)
        *reinterpret_cast<uint2 *>(qdst + static_cast<size_t>(n) * p.Hh * p.d) = quant8(xq[ps], mq);
      if (phys >= 0) {
        float xv[8];
        widen(rv[ps], xv);
        *reinterpret_cast<uint2 *>(kdst + r * p.d) = quant8(xk[ps], mk);
        *reinterpret_cast<uint2 *>(vdst + r * p.d) = quant8(xv, mv);
      }
    }
    if (phys >= 0 && h == 0 && threadIdx.x == 0) p.tags[phys] = p.live.tag[li];
  }
  // Drain: every load thread 0 issued has landed before the CTA exits. Only
  // an aborted loop leaves loads behind; waiting on the parity of a stage's
  // last fill returns at once when that fill was already consumed.
  if (threadIdx.x == 0) {
    if (issued0) drain_wait(ctx, 0, (issued0 - 1) & 1);
    if (issued1) drain_wait(ctx, 1, (issued1 - 1) & 1);
  }
}

}  // namespace

cudaError_t launch_publish_fp8(const PublishParams &p, const void *tmap_q, const void *tmap_k,
                               const void *tmap_v, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  if (p.d != 128 || p.P != kRows) return cudaErrorInvalidValue;
  const int64_t nblk = static_cast<int64_t>(p.live.n) * p.npc * p.Hh;
  if (nblk > 0x7fffffff) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(publish_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(nblk < sms ? nblk : sms);
  publish_fp8_kernel<<<grid, kThreads, kSmemBytes, st>>>(
      p, *static_cast<const CUtensorMap *>(tmap_q), *static_cast<const CUtensorMap *>(tmap_k),
      *static_cast<const CUtensorMap *>(tmap_v));
  return cudaGetLastError();
}

}  // namespace wf
