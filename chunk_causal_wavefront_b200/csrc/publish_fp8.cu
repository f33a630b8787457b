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
// One CTA handles one (live slot, page j, head) block for q, k and v: 256
// threads, 16 per token row (8 bf16 values = 16 bytes each), 8 passes of 16
// rows. Per tensor: streaming 16-byte loads of all 8 passes, rotation, block
// amax (warp max + shared-memory max over the 8 warps), scaling by 2^-e,
// conversion to E4M3 and 8-byte stores; rows past C are zero codes in the K/V
// page. HBM-bound: 6 bytes read and 3 written per (token, head, dim).
#include <cuda_bf16.h>

#include "sm100.cuh"
#include "wf_internal.h"

namespace wf {
namespace {

using sm100::pack_e4m3x4;

constexpr int kRows = 128;                     // rows per block (page / query tile)
constexpr int kThreads = 256;
constexpr int kTPR = 16;                       // threads per row
constexpr int kRowsPerPass = kThreads / kTPR;  // 16
constexpr int kPasses = kRows / kRowsPerPass;  // 8
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

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

// Block-wide max of non-negative floats (every thread gets the result).
__device__ __forceinline__ float block_max(float v, float *red) {
  const uint32_t w = __reduce_max_sync(0xffffffffu, __float_as_uint(v));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = __uint_as_float(w);
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) m = fmaxf(m, red[i]);
  __syncthreads();   // red is reused by the next tensor
  return m;
}

// Load one tensor's 8 rows of this thread (zeros past C).
__device__ __forceinline__ void load_rows(const __nv_bfloat16 *src, int row0, int C, int Hh,
                                          int d, int h, int cv, uint4 (&raw)[kPasses]) {
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int n = row0 + i * kRowsPerPass;
    raw[i] = n < C ? ld_stream(src + (static_cast<size_t>(n) * Hh + h) * d + cv * 8)
                   : make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ void widen(const uint4 &u, float *f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Rotate the 4 pairs whose first dimension is dim0, for the token at (t, y, x):
// (a c - b s, a s + b c), each product and sum rounded once to fp32.
__device__ __forceinline__ void rope8(float *v, int dim0, int t, int y, int x,
                                      const PublishParams &p) {
  const int h0 = p.split0 >> 1, h1 = p.split1 >> 1, h2 = p.split2 >> 1;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int pr = (dim0 >> 1) + i;
    float2 cs;
    if (pr < h0) cs = __ldg(p.rope_t + t * h0 + pr);
    else if (pr < h0 + h1) cs = __ldg(p.rope_h + y * h1 + (pr - h0));
    else cs = __ldg(p.rope_w + x * h2 + (pr - h0 - h1));
    const float a = v[2 * i], b = v[2 * i + 1];
    v[2 * i] = __fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y));
    v[2 * i + 1] = __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(b, cs.x));
  }
}

__global__ void __launch_bounds__(kThreads) publish_fp8_kernel(const PublishParams p) {
  __shared__ float red[kWarps];
  const int li = blockIdx.y;
  const int j = blockIdx.x / p.Hh;
  const int h = blockIdx.x - j * p.Hh;
  const int slot = p.live.slot[li];
  const int pos = __ldg(p.table + kTabSlotPos + slot);
  int phys = pos < 0 ? -1 : __ldg(p.table + kTabPages + pos * p.npc + j);
  if (phys >= p.num_pages) phys = -1;
  if (phys < 0 && threadIdx.x == 0) record_status(p.status, WF_ERR_BAD_PAGE);

  const int cv = threadIdx.x & (kTPR - 1);       // 16-byte vector of the head row
  const int r0 = threadIdx.x / kTPR;             // first row of this thread
  const int row0 = j * kRows + r0;               // token of pass 0
  const size_t slot_off = static_cast<size_t>(slot) * p.C * p.Hh * p.d;

  // Rotary positions of this thread's 8 tokens.
  int tp[kPasses], yp[kPasses], xp[kPasses];
  if (p.rope) {
    const int hw = p.gh * p.gw;
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
      int n = row0 + i * kRowsPerPass;
      if (n >= p.C) n = 0;
      const int f = n / hw, yx = n - f * hw;
      tp[i] = p.F * p.live.chunk[li] + f;
      yp[i] = yx / p.gw;
      xp[i] = yx - yp[i] * p.gw;
    }
  }

  // tensor 0 = q (to q_rot), 1 = k, 2 = v (to the page)
#pragma unroll 1
  for (int t = 0; t < 3; ++t) {
    const __nv_bfloat16 *src =
        static_cast<const __nv_bfloat16 *>(t == 0 ? p.q : (t == 1 ? p.k : p.v)) + slot_off;
    uint4 raw[kPasses];
    load_rows(src, row0, p.C, p.Hh, p.d, h, cv, raw);
    float x[kPasses][8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
      widen(raw[i], x[i]);
      // rows past C stay +0 (zero codes): rotating them could turn +0 into -0
      if (t < 2 && p.rope && row0 + i * kRowsPerPass < p.C)
        rope8(x[i], cv * 8, tp[i], yp[i], xp[i], p);
#pragma unroll
      for (int c = 0; c < 8; ++c) amax = fmaxf(amax, fabsf(x[i][c]));
    }
    const int e = scale_exponent(block_max(amax, red));
    const float mul = exp2i(-e);
    uint8_t *dst;
    size_t row_stride;
    if (t == 0) {
      dst = static_cast<uint8_t *>(p.q_rot) + slot_off + static_cast<size_t>(h) * p.d + cv * 8;
      row_stride = static_cast<size_t>(p.Hh) * p.d;
      if (threadIdx.x == 0) p.q_scale[(static_cast<size_t>(slot) * p.npc + j) * p.Hh + h] = exp2i(e);
    } else {
      if (phys < 0) continue;
      const size_t blk = (static_cast<size_t>(phys) * 2 + (t - 1)) * p.Hh + h;
      dst = reinterpret_cast<uint8_t *>(p.pages) + blk * p.P * p.d + cv * 8;
      row_stride = p.d;
      if (threadIdx.x == 0) p.kv_scale[blk] = exp2i(e);
    }
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
      const int r = r0 + i * kRowsPerPass;        // row inside the block
      const int n = j * kRows + r;
      if (t == 0 && n >= p.C) continue;           // q_rot has C rows
      uint2 w;
      w.x = pack_e4m3x4(x[i][0] * mul, x[i][1] * mul, x[i][2] * mul, x[i][3] * mul);
      w.y = pack_e4m3x4(x[i][4] * mul, x[i][5] * mul, x[i][6] * mul, x[i][7] * mul);
      const size_t row_off = t == 0 ? static_cast<size_t>(n) * row_stride
                                    : static_cast<size_t>(r) * row_stride;
      *reinterpret_cast<uint2 *>(dst + row_off) = w;
    }
  }
  if (phys >= 0 && h == 0 && threadIdx.x == 0) p.tags[phys] = p.live.tag[li];
}

}  // namespace

cudaError_t launch_publish_fp8(const PublishParams &p, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  if (p.d != 128 || p.P != kRows) return cudaErrorInvalidValue;
  const int64_t bx = static_cast<int64_t>(p.npc) * p.Hh;
  if (bx > 0x7fffffff) return cudaErrorInvalidValue;
  publish_fp8_kernel<<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(p.live.n)),
                       kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace wf
