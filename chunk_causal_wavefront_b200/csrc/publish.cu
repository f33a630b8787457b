// Early K/V publication: rotary embedding + scatter into the paged pool.
//
// "Wave Forcing: Towards Speed-of-Light Streaming Video Generation", Method
// section: K/V are published right after the QKV projection and RoPE, and
// paged delivery writes them directly into ordered attention slots, followed
// by a ready signal. Here the "slots" are the pages that the device page table
// assigns to each live slot; the ready signal is a per-page tag.
//
// One launch covers every live slot of the round (grid row = slot). A thread
// owns one 16-byte vector column (8 bf16 or 4 fp32 values = 4 or 2 rotary
// pairs) of the [C][heads][d] token rows and walks the block's tokens: it
// loads q, k and v with streaming 16-byte loads, rotates q and k in fp32 with
// (cos, sin) tables computed on the host in fp64, rounds once to the storage
// type and issues 16-byte stores to q_rot and to the K and V pages.
// Consecutive threads cover consecutive vectors of a token row, so loads are
// fully coalesced; a warp's page stores cover two contiguous 256-byte head
// rows. HBM-bound: 3 reads + 3 writes of every element.
#include <cuda_bf16.h>

#include "wf_internal.h"

namespace wf {
namespace {

template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };
template <> struct Vec<float> { static constexpr int N = 4; };

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ void unpack(const uint4 &u, float *f, __nv_bfloat16) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void unpack(const uint4 &u, float *f, float) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}

__device__ __forceinline__ uint4 pack(const float *f, __nv_bfloat16) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);   // RNE
    w[i] = *reinterpret_cast<uint32_t *>(&b);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ uint4 pack(const float *f, float) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}

// Rotate the pairs of one vector whose first element is dimension dim0.
template <int N>
__device__ __forceinline__ void rope_vec(float *x, int dim0, int tpos, int ypos, int xpos,
                                         const PublishParams &p) {
  const int h0 = p.split0 >> 1, h1 = p.split1 >> 1, h2 = p.split2 >> 1;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const int pr = (dim0 >> 1) + i;   // pair index inside head_dim
    float2 cs;
    if (pr < h0) cs = __ldg(p.rope_t + tpos * h0 + pr);
    else if (pr < h0 + h1) cs = __ldg(p.rope_h + ypos * h1 + (pr - h0));
    else cs = __ldg(p.rope_w + xpos * h2 + (pr - h0 - h1));
    const float a = x[2 * i], b = x[2 * i + 1];
    x[2 * i] = a * cs.x - b * cs.y;
    x[2 * i + 1] = a * cs.y + b * cs.x;
  }
}

constexpr int kTok = 16;   // tokens per block

// Grid: (token blocks + tail blocks, live slots); block = one thread per
// 16-byte vector column (head, vector) of a token row, looping over columns
// when a row has more vectors than the block has threads. A block first puts
// its tokens' rotary positions and page rows in shared memory, so the inner
// loop has no integer division: per token and column it issues three
// streaming 16-byte loads (two tokens at a time), rotates q and k in fp32,
// rounds once and issues three 16-byte stores. Tail blocks zero the rows past
// C in the chunk's last page.
template <typename T>
__global__ void __launch_bounds__(640) publish_kernel(const PublishParams p, int main_blocks) {
  constexpr int N = Vec<T>::N;
  __shared__ int s_pos[3][kTok];       // t, y, x of the block's tokens
  __shared__ int s_page[kTok];         // physical page of each token (-1: bad table entry)
  __shared__ int s_row[kTok];          // row of each token inside its page
  const int li = blockIdx.y;
  const int slot = p.live.slot[li];
  const int pos = __ldg(p.table + kTabSlotPos + slot);
  const int vpr = p.d / N;                                   // vectors per head row
  const int vpt = p.Hh * vpr;                                // vectors per token
  const size_t kv_elems = static_cast<size_t>(p.Hh) * p.P * p.d;   // K -> V distance
  const size_t page_elems = 2 * kv_elems;
  T *pages = reinterpret_cast<T *>(p.pages);

  if (blockIdx.x < main_blocks) {
    const int n0 = blockIdx.x * kTok;
    const int ntok = min(kTok, p.C - n0);
    if (threadIdx.x < ntok) {
      const int n = n0 + threadIdx.x;
      if (p.rope) {
        const int hw = p.gh * p.gw;
        s_pos[0][threadIdx.x] = p.F * p.live.chunk[li] + n / hw;
        s_pos[1][threadIdx.x] = (n / p.gw) % p.gh;
        s_pos[2][threadIdx.x] = n % p.gw;
      }
      const int j = n / p.P, row = n - j * p.P;
      const int phys = pos < 0 ? -1 : __ldg(p.table + kTabPages + pos * p.npc + j);
      s_row[threadIdx.x] = row;
      if (phys < 0 || phys >= p.num_pages) {
        record_status(p.status, WF_ERR_BAD_PAGE);
        s_page[threadIdx.x] = -1;
      } else {
        s_page[threadIdx.x] = phys;
        if (row == 0) p.tags[phys] = p.live.tag[li];
      }
    }
    __syncthreads();
    const size_t slot_off = static_cast<size_t>(slot) * p.C * p.Hh * p.d;
    for (int col = threadIdx.x; col < vpt; col += blockDim.x) {
      const int h = col / vpr, e = col - h * vpr;
      const size_t col_off = static_cast<size_t>(h) * p.d + e * N;   // inside a token row
      const size_t page_col = static_cast<size_t>(h) * p.P * p.d + e * N;
      for (int i = 0; i < ntok; i += 2) {
        const bool two = i + 1 < ntok;
        const size_t src0 = slot_off + static_cast<size_t>(n0 + i) * p.Hh * p.d + col_off;
        const size_t src1 = src0 + static_cast<size_t>(p.Hh) * p.d;
        const uint4 q0 = ld_stream(static_cast<const T *>(p.q) + src0);
        const uint4 k0 = ld_stream(static_cast<const T *>(p.k) + src0);
        const uint4 v0 = ld_stream(static_cast<const T *>(p.v) + src0);
        uint4 q1 = make_uint4(0, 0, 0, 0), k1 = q1, v1 = q1;
        if (two) {
          q1 = ld_stream(static_cast<const T *>(p.q) + src1);
          k1 = ld_stream(static_cast<const T *>(p.k) + src1);
          v1 = ld_stream(static_cast<const T *>(p.v) + src1);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (u == 1 && !two) break;
          const int t = i + u;
          float q[N], k[N];
          unpack(u ? q1 : q0, q, T());
          unpack(u ? k1 : k0, k, T());
          if (p.rope) {
            rope_vec<N>(q, e * N, s_pos[0][t], s_pos[1][t], s_pos[2][t], p);
            rope_vec<N>(k, e * N, s_pos[0][t], s_pos[1][t], s_pos[2][t], p);
          }
          *reinterpret_cast<uint4 *>(static_cast<T *>(p.q_rot) + (u ? src1 : src0)) = pack(q, T());
          const int phys = s_page[t];
          if (phys < 0) continue;
          T *kdst = pages + phys * page_elems + page_col + static_cast<size_t>(s_row[t]) * p.d;
          *reinterpret_cast<uint4 *>(kdst) = pack(k, T());
          *reinterpret_cast<uint4 *>(kdst + kv_elems) = u ? v1 : v0;
        }
      }
    }
  } else {
    // Zero the rows past C in the chunk's last page: (K|V, head, row, vector).
    const int tail_rows = p.npc * p.P - p.C;
    const int total = 2 * p.Hh * tail_rows * vpr;
    const int phys = pos < 0 ? -1 : __ldg(p.table + kTabPages + pos * p.npc + (p.npc - 1));
    if (phys < 0 || phys >= p.num_pages) {
      if (threadIdx.x == 0) record_status(p.status, WF_ERR_BAD_PAGE);
      return;
    }
    const int tb = blockIdx.x - main_blocks, ntb = gridDim.x - main_blocks;
    for (int v = tb * blockDim.x + threadIdx.x; v < total; v += ntb * blockDim.x) {
      int r = v;
      const int e = r % vpr;
      r /= vpr;
      const int row = p.P - tail_rows + r % tail_rows;
      r /= tail_rows;
      const int h = r % p.Hh;
      const int kv = r / p.Hh;
      T *dst = pages + phys * page_elems + kv * kv_elems +
               (static_cast<size_t>(h) * p.P + row) * p.d + e * N;
      *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
}

template <typename T>
cudaError_t launch(const PublishParams &p, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  constexpr int N = Vec<T>::N;
  const int vpt = p.Hh * (p.d / N);
  const int threads = vpt >= 640 ? 640 : ((vpt + 31) / 32) * 32;
  const int main_blocks = (p.C + kTok - 1) / kTok;
  const int64_t tail_vecs = 2LL * p.Hh * (p.npc * p.P - p.C) * (p.d / N);
  const int tail_blocks = tail_vecs == 0 ? 0 : static_cast<int>((tail_vecs + threads - 1) / threads);
  const int64_t per_slot = static_cast<int64_t>(p.C) * vpt + tail_vecs;
  if (per_slot >= (int64_t(1) << 30)) return cudaErrorInvalidValue;   // int32 vector indices
  publish_kernel<T><<<dim3(main_blocks + tail_blocks, p.live.n), threads, 0, st>>>(p, main_blocks);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_publish_bf16(const PublishParams &p, cudaStream_t st) {
  return launch<__nv_bfloat16>(p, st);
}
cudaError_t launch_publish_f32(const PublishParams &p, cudaStream_t st) {
  return launch<float>(p, st);
}

}  // namespace wf
