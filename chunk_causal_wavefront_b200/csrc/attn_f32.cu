// Round attention, fp32 CUDA-core path.
//
// "Wave Forcing: Towards Speed-of-Light Streaming Video Generation", Method
// section: full attention inside each chunk and chunk-wise causal attention
// across chunks, M_WF(s, j) = 1[j >= s]. Query slot s reads the prefix of the
// ordered context (anchor, history, store, slots S-1 .. s) that ends at its own
// entry; the masked (s, j) chunk pairs are never visited.
//
// fp32 cannot use the bf16 tensor cores, and TF32 would not meet a 1e-5
// tolerance, so this path runs on FP32 FMA units. A block handles 32 query
// rows of one (slot, head); each warp owns 8 rows. Keys are processed in
// sub-tiles of 32 (one per lane): lane l scores key l against each row, the
// row max and sum of the online softmax are warp-shuffle reductions, and each
// lane accumulates the output dimensions l, l+32, ... of every row.
#include <cfloat>

#include "wf_internal.h"

namespace wf {
namespace {

constexpr int kRows = 32;          // query rows per block
constexpr int kWarps = 4;
constexpr int kRowsPerWarp = kRows / kWarps;
constexpr int kMaxDim = 128;
constexpr int kDimPerLane = kMaxDim / 32;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kWarps * 32) attn_f32_kernel(const AttnParams p) {
  extern __shared__ float smem[];
  const int D = p.d;
  const int ldk = D + 1;                       // padded K rows: conflict-free lane-per-key reads
  float *Qs = smem;                            // [kRows][D]
  float *Ks = Qs + kRows * D;                  // [32][D + 1]
  float *Vs = Ks + 32 * ldk;                   // [32][D]

  const int tiles_per_slot = (p.C + kRows - 1) / kRows;
  int item = blockIdx.x;
  const int tile = item % tiles_per_slot;
  item /= tiles_per_slot;
  const int h = item % p.Hh;
  const int li = item / p.Hh;
  const int slot = p.live.slot[li];
  const int npos = p.live.npos[li];

  const int st = check_context_pages(p.table, p.tags, p.n_pos, p.npc, p.num_pages);
  if (st != WF_OK) {
    if (threadIdx.x == 0) record_status(p.status, st);
    return;
  }

  const float *q = static_cast<const float *>(p.q_rot);
  float *out = static_cast<float *>(p.out);
  const float *pages = reinterpret_cast<const float *>(p.pages);
  const size_t page_elems = static_cast<size_t>(2) * p.Hh * p.P * D;
  const size_t row_stride = static_cast<size_t>(p.Hh) * D;
  const int row0 = tile * kRows;

  for (int i = threadIdx.x; i < kRows * D; i += blockDim.x) {
    const int r = i / D, c = i - r * D;
    const int n = row0 + r;
    Qs[i] = n < p.C ? q[(static_cast<size_t>(slot) * p.C + n) * row_stride + h * D + c] : 0.0f;
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][kDimPerLane];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.0f;
#pragma unroll
    for (int i = 0; i < kDimPerLane; ++i) o[r][i] = 0.0f;
  }

  for (int pos = 0; pos < npos; ++pos) {
    for (int j = 0; j < p.npc; ++j) {
      const int phys = __ldcg(p.table + kTabPages + pos * p.npc + j);
      const int valid = (j == p.npc - 1) ? p.C - j * p.P : p.P;
      const float *kp = pages + phys * page_elems + static_cast<size_t>(h) * p.P * D;
      const float *vp = kp + static_cast<size_t>(p.Hh) * p.P * D;
      for (int kb = 0; kb < valid; kb += 32) {
        const int nk = valid - kb < 32 ? valid - kb : 32;
        __syncthreads();
        for (int i = threadIdx.x; i < 32 * D; i += blockDim.x) {
          const int r = i / D, c = i - r * D;
          const bool ok = r < nk;
          Ks[r * ldk + c] = ok ? kp[static_cast<size_t>(kb + r) * D + c] : 0.0f;
          Vs[i] = ok ? vp[static_cast<size_t>(kb + r) * D + c] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const float *qr = Qs + (warp * kRowsPerWarp + r) * D;
          float s = -INFINITY;
          if (lane < nk) {
            const float *kr = Ks + lane * ldk;
            float acc = 0.0f;
            for (int c = 0; c < D; ++c) acc = fmaf(qr[c], kr[c], acc);
            s = acc * p.scale;
          }
          const float m_new = fmaxf(m[r], warp_max(s));
          const float alpha = expf(m[r] - m_new);            // 0 on the first tile
          const float pr = expf(s - m_new);                  // 0 for masked keys
          l[r] = l[r] * alpha + warp_sum(pr);
#pragma unroll
          for (int i = 0; i < kDimPerLane; ++i) o[r][i] *= alpha;
          for (int key = 0; key < nk; ++key) {
            const float pk = __shfl_sync(0xffffffffu, pr, key);
#pragma unroll
            for (int i = 0; i < kDimPerLane; ++i) {
              const int c = lane + 32 * i;
              if (c < D) o[r][i] = fmaf(pk, Vs[key * D + c], o[r][i]);
            }
          }
          m[r] = m_new;
        }
      }
    }
  }

#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int n = row0 + warp * kRowsPerWarp + r;
    if (n >= p.C) continue;
    const float inv = 1.0f / l[r];
    float *dst = out + (static_cast<size_t>(slot) * p.C + n) * row_stride + h * D;
#pragma unroll
    for (int i = 0; i < kDimPerLane; ++i) {
      const int c = lane + 32 * i;
      if (c < D) dst[c] = o[r][i] * inv;
    }
  }
}

}  // namespace

cudaError_t launch_attention_f32(const AttnParams &p, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  if (p.d > kMaxDim) return cudaErrorInvalidValue;
  const size_t smem = (static_cast<size_t>(kRows) * p.d + 32 * (p.d + 1) + 32 * p.d) * 4;
  cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = (p.C + kRows - 1) / kRows;
  const int64_t blocks = static_cast<int64_t>(tiles) * p.Hh * p.live.n;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  attn_f32_kernel<<<static_cast<unsigned>(blocks), kWarps * 32, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace wf
