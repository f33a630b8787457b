// Early K/V publication: rotary embedding + scatter into the paged pool.
//
// "Wave Forcing: Towards Speed-of-Light Streaming Video Generation", Method
// section: K/V are published right after the QKV projection and RoPE, and
// paged delivery writes them directly into ordered attention slots, followed
// by a ready signal. Here the "slots" are the pages that the device page table
// assigns to each live slot; the ready signal is a per-page tag.
//
// One launch covers every live slot of the round. Each thread owns one
// 16-byte vector (8 bf16 or 4 fp32 values = 4 or 2 rotary pairs) of one
// (slot, token, head) row: it loads q, k and v with streaming 16-byte loads,
// rotates q and k in fp32 with (cos, sin) tables computed on the host in fp64,
// rounds once to the storage type and issues 16-byte stores to q_rot and to
// the K and V pages. Consecutive threads cover consecutive 16-byte vectors of
// the [C][heads][d] input rows, so loads are fully coalesced; a warp's page
// stores cover two contiguous 256-byte head rows. HBM-bound: 3 reads + 3
// writes of every element.
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

template <typename T>
__global__ void __launch_bounds__(256) publish_kernel(const PublishParams p) {
  constexpr int N = Vec<T>::N;
  const int vpr = p.d / N;                                   // vectors per head row
  const int64_t per_slot = static_cast<int64_t>(p.C) * p.Hh * vpr;
  const int64_t main_n = per_slot * p.live.n;
  const int tail_rows = p.npc * p.P - p.C;                   // zero rows of the last page
  const int64_t tail_per_slot = static_cast<int64_t>(2) * p.Hh * tail_rows * vpr;
  const int64_t total = main_n + tail_per_slot * p.live.n;
  const size_t page_elems = static_cast<size_t>(2) * p.Hh * p.P * p.d;
  T *pages = reinterpret_cast<T *>(p.pages);

  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (idx < main_n) {
      const int li = static_cast<int>(idx / per_slot);
      int64_t r = idx - li * per_slot;
      const int e = static_cast<int>(r % vpr);
      r /= vpr;
      const int h = static_cast<int>(r % p.Hh);
      const int n = static_cast<int>(r / p.Hh);
      const int slot = p.live.slot[li];
      const int pos = __ldg(p.table + kTabSlotPos + slot);
      const int j = n / p.P, row = n - j * p.P;
      const int phys = pos < 0 ? -1 : __ldg(p.table + kTabPages + pos * p.npc + j);
      const size_t src = ((static_cast<size_t>(slot) * p.C + n) * p.Hh + h) * p.d + e * N;
      float q[N], k[N];
      unpack(ld_stream(static_cast<const T *>(p.q) + src), q, T());
      unpack(ld_stream(static_cast<const T *>(p.k) + src), k, T());
      const uint4 v = ld_stream(static_cast<const T *>(p.v) + src);
      if (p.rope) {
        const int chunk = p.live.chunk[li];
        const int hw = p.gh * p.gw;
        const int tpos = p.F * chunk + n / hw;
        const int ypos = (n / p.gw) % p.gh;
        const int xpos = n % p.gw;
        rope_vec<N>(q, e * N, tpos, ypos, xpos, p);
        rope_vec<N>(k, e * N, tpos, ypos, xpos, p);
      }
      *reinterpret_cast<uint4 *>(static_cast<T *>(p.q_rot) + src) = pack(q, T());
      if (phys < 0 || phys >= p.num_pages) {
        record_status(p.status, WF_ERR_BAD_PAGE);
        continue;
      }
      T *kdst = pages + phys * page_elems + (static_cast<size_t>(h) * p.P + row) * p.d + e * N;
      T *vdst = kdst + static_cast<size_t>(p.Hh) * p.P * p.d;
      *reinterpret_cast<uint4 *>(kdst) = pack(k, T());
      *reinterpret_cast<uint4 *>(vdst) = v;
      if (row == 0 && h == 0 && e == 0) p.tags[phys] = p.live.tag[li];
    } else {
      int64_t r = idx - main_n;
      const int li = static_cast<int>(r / tail_per_slot);
      r -= li * tail_per_slot;
      const int e = static_cast<int>(r % vpr);
      r /= vpr;
      const int row = p.P - tail_rows + static_cast<int>(r % tail_rows);
      r /= tail_rows;
      const int h = static_cast<int>(r % p.Hh);
      const int kv = static_cast<int>(r / p.Hh);
      const int slot = p.live.slot[li];
      const int pos = __ldg(p.table + kTabSlotPos + slot);
      const int phys = pos < 0 ? -1 : __ldg(p.table + kTabPages + pos * p.npc + (p.npc - 1));
      if (phys < 0 || phys >= p.num_pages) {
        record_status(p.status, WF_ERR_BAD_PAGE);
        continue;
      }
      T *dst = pages + phys * page_elems +
               ((static_cast<size_t>(kv) * p.Hh + h) * p.P + row) * p.d + e * N;
      *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
}

template <typename T>
cudaError_t launch(const PublishParams &p, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  constexpr int N = Vec<T>::N;
  const int64_t vpr = p.d / N;
  const int64_t total = static_cast<int64_t>(p.live.n) *
                        (static_cast<int64_t>(p.C) * p.Hh * vpr +
                         2LL * p.Hh * (p.npc * p.P - p.C) * vpr);
  int sms = 148;
  int dev;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 8;   // 8 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  publish_kernel<T><<<static_cast<int>(blocks), 256, 0, st>>>(p);
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
