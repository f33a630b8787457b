// Early K/V publication: rotary embedding + scatter into the paged pool.
//
// "Wave Forcing: Towards Speed-of-Light Streaming Video Generation", Method
// section: K/V are published right after the QKV projection and RoPE, and
// paged delivery writes them directly into ordered attention slots, followed
// by a ready signal. Here the "slots" are the pages that the device page table
// assigns to each live slot; the ready signal is a per-page tag.
//
// This kernel serves fp32 pools (any head_dim that is a multiple of 4 up to
// 128, pages of up to 256 tokens); bf16 pools, whose head_dim and pages are
// 128, publish through the TMA ring of publish_tma.cu.
//
// One launch covers every live slot of the round (grid row = slot). A thread
// handles 16-byte vectors (4 fp32 values = 2 rotary pairs) of (slot, token,
// head) rows, two per iteration: it loads q, k and v with streaming 16-byte
// loads, rotates q and k in fp32 (each product and sum rounded once) with
// (cos, sin) tables computed on the host in fp64 and rounded to fp32, and issues 16-byte stores to q_rot and to the K and V pages. Consecutive
// threads cover consecutive 16-byte vectors of the [C][heads][d] input rows,
// so loads are fully coalesced. HBM-bound: 3 reads + 3 writes of every
// element.

#include "wf_internal.h"

namespace wf {
namespace {

// Division by a runtime-invariant divisor d (1 <= d < 2^31) for dividends
// n < 2^31 with one multiply-high and a shift (Granlund and Montgomery,
// "Division by Invariant Integers using Multiplication", 1994): with
// p = 31 + ceil(log2 d) and m = ceil(2^p / d), floor(n / d) = (n * m) >> p,
// exact because m - 2^p / d < 1 keeps the error below 1 / d.
struct FastDiv {
  uint32_t d, m, shift;   // shift = p - 32 (d >= 2); d == 1 is the identity
  __host__ __device__ FastDiv() : d(1), m(0), shift(0) {}
  __host__ explicit FastDiv(uint32_t div) : d(div), m(0), shift(0) {
    if (d > 1) {
      uint32_t l = 0;
      while ((uint64_t(1) << l) < d) ++l;                 // ceil(log2 d)
      const uint64_t p2 = uint64_t(1) << (31 + l);
      m = static_cast<uint32_t>((p2 + d - 1) / d);
      shift = 31 + l - 32;
    }
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    return d == 1 ? n : (__umulhi(n, m) >> shift);
  }
  __device__ __forceinline__ void divmod(uint32_t n, uint32_t &q, uint32_t &r) const {
    q = div(n);
    r = n - q * d;
  }
};

struct PublishDivs {
  FastDiv vpt, vpr, P, hw, gw, tail_rows, Hh;
};

template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; };

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ void unpack(const uint4 &u, float *f, float) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
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
    x[2 * i] = __fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y));     // no FMA contraction
    x[2 * i + 1] = __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(b, cs.x));
  }
}

// Physical page holding page j of live slot li's chunk (-1 if the table is bad).
__device__ __forceinline__ int slot_page(const PublishParams &p, int pos, int j) {
  const int phys = pos < 0 ? -1 : __ldg(p.table + kTabPages + pos * p.npc + j);
  return (phys < 0 || phys >= p.num_pages) ? -1 : phys;
}

// One main-part vector: rotate q and k, write q_rot and the K/V page rows.
template <typename T>
__device__ __forceinline__ void publish_vector(const PublishParams &p, const PublishDivs &dv,
                                               int li, int pos, int n, int h, int e,
                                               const uint4 &qv, const uint4 &kv,
                                               const uint4 &vv, size_t src) {
  constexpr int N = Vec<T>::N;
  float q[N], k[N];
  unpack(qv, q, T());
  unpack(kv, k, T());
  if (p.rope) {
    // n = f * (gh * gw) + y * gw + x: frame f of the chunk, row y, column x
    uint32_t f, yx, y, x;
    dv.hw.divmod(n, f, yx);
    dv.gw.divmod(yx, y, x);
    const int tpos = p.F * p.live.chunk[li] + static_cast<int>(f);
    rope_vec<N>(q, e * N, tpos, static_cast<int>(y), static_cast<int>(x), p);
    rope_vec<N>(k, e * N, tpos, static_cast<int>(y), static_cast<int>(x), p);
  }
  *reinterpret_cast<uint4 *>(static_cast<T *>(p.q_rot) + src) = pack(q, T());
  uint32_t ju, rowu;
  dv.P.divmod(n, ju, rowu);
  const int j = static_cast<int>(ju), row = static_cast<int>(rowu);
  const int phys = slot_page(p, pos, j);
  if (phys < 0) {
    record_status(p.status, WF_ERR_BAD_PAGE);
    return;
  }
  const size_t page_elems = static_cast<size_t>(2) * p.Hh * p.P * p.d;
  T *kdst = reinterpret_cast<T *>(p.pages) + phys * page_elems +
            (static_cast<size_t>(h) * p.P + row) * p.d + e * N;
  T *vdst = kdst + static_cast<size_t>(p.Hh) * p.P * p.d;
  *reinterpret_cast<uint4 *>(kdst) = pack(k, T());
  *reinterpret_cast<uint4 *>(vdst) = vv;
  if (row == 0 && h == 0 && e == 0) p.tags[phys] = p.live.tag[li];
}

// Grid: (blocks, live slots). Each thread walks its slot's vectors with a
// grid stride, two at a time so that six 16-byte loads are in flight before
// the first one is used. Vector v < C * heads * d/N is (token n, head h,
// vector e) of the [C][heads][d] rows; the remaining vectors zero the rows
// past C in the chunk's last page (K then V, head-major, row, vector).
template <typename T>
__global__ void __launch_bounds__(256) publish_kernel(const PublishParams p, const PublishDivs dv) {
  constexpr int N = Vec<T>::N;
  const int li = blockIdx.y;
  const int slot = p.live.slot[li];
  const int pos = __ldg(p.table + kTabSlotPos + slot);
  const int vpr = p.d / N;                                   // vectors per head row
  const int vpt = p.Hh * vpr;                                // vectors per token
  const int main_n = p.C * vpt;
  const int tail_rows = p.npc * p.P - p.C;
  const int total = main_n + 2 * p.Hh * tail_rows * vpr;
  const size_t slot_off = static_cast<size_t>(slot) * p.C * p.Hh * p.d;
  const T *qs = static_cast<const T *>(p.q) + slot_off;
  const T *ks = static_cast<const T *>(p.k) + slot_off;
  const T *vs = static_cast<const T *>(p.v) + slot_off;
  const int stride = gridDim.x * blockDim.x;

  for (int v0 = blockIdx.x * blockDim.x + threadIdx.x; v0 < total; v0 += 2 * stride) {
    const int v1 = v0 + stride;
    const bool m0 = v0 < main_n, m1 = v1 < main_n;
    uint4 q0, k0, w0, q1, k1, w1;
    if (m0) {
      q0 = ld_stream(qs + static_cast<size_t>(v0) * N);
      k0 = ld_stream(ks + static_cast<size_t>(v0) * N);
      w0 = ld_stream(vs + static_cast<size_t>(v0) * N);
    }
    if (m1) {
      q1 = ld_stream(qs + static_cast<size_t>(v1) * N);
      k1 = ld_stream(ks + static_cast<size_t>(v1) * N);
      w1 = ld_stream(vs + static_cast<size_t>(v1) * N);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int v = u ? v1 : v0;
      if (v >= total) break;
      if (u ? m1 : m0) {
        uint32_t n, rem, h, e;
        dv.vpt.divmod(v, n, rem);
        dv.vpr.divmod(rem, h, e);
        publish_vector<T>(p, dv, li, pos, n, h, e, u ? q1 : q0, u ? k1 : k0, u ? w1 : w0,
                          slot_off + static_cast<size_t>(v) * N);
      } else {
        uint32_t r1, e, r2, rr, kv, h;
        dv.vpr.divmod(v - main_n, r1, e);
        dv.tail_rows.divmod(r1, r2, rr);
        dv.Hh.divmod(r2, kv, h);
        const int row = p.P - tail_rows + static_cast<int>(rr);
        const int phys = slot_page(p, pos, p.npc - 1);
        if (phys < 0) {
          record_status(p.status, WF_ERR_BAD_PAGE);
          continue;
        }
        T *dst = reinterpret_cast<T *>(p.pages) +
                 phys * (static_cast<size_t>(2) * p.Hh * p.P * p.d) +
                 ((static_cast<size_t>(kv) * p.Hh + h) * p.P + row) * p.d + e * N;
        *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
      }
    }
  }
}

template <typename T>
cudaError_t launch(const PublishParams &p, cudaStream_t st) {
  if (p.live.n == 0) return cudaSuccess;
  constexpr int N = Vec<T>::N;
  const int64_t vpr = p.d / N;
  const int64_t per_slot = static_cast<int64_t>(p.C) * p.Hh * vpr +
                           2LL * p.Hh * (p.npc * p.P - p.C) * vpr;
  if (per_slot >= (int64_t(1) << 30)) return cudaErrorInvalidValue;   // int32 vector indices
  int sms = 148, dev = 0, per_sm = 4;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, publish_kernel<T>, 256, 0);
  PublishDivs dv;
  dv.vpt = FastDiv(static_cast<uint32_t>(p.Hh * (p.d / N)));
  dv.vpr = FastDiv(static_cast<uint32_t>(p.d / N));
  dv.P = FastDiv(static_cast<uint32_t>(p.P));
  dv.hw = FastDiv(static_cast<uint32_t>(p.gh * p.gw));
  dv.gw = FastDiv(static_cast<uint32_t>(p.gw));
  dv.tail_rows = FastDiv(static_cast<uint32_t>(p.npc * p.P - p.C > 0 ? p.npc * p.P - p.C : 1));
  dv.Hh = FastDiv(static_cast<uint32_t>(p.Hh));
  if (per_sm < 1) per_sm = 1;
  // One wave: every resident block slot of the GPU, spread over the live slots.
  int64_t bx = (static_cast<int64_t>(sms) * per_sm) / p.live.n;
  const int64_t need = (per_slot + 511) / 512;            // two vectors per thread
  if (bx > need) bx = need;
  if (bx < 1) bx = 1;
  publish_kernel<T><<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(p.live.n)), 256, 0, st>>>(p, dv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_publish_f32(const PublishParams &p, cudaStream_t st) {
  return launch<float>(p, st);
}

}  // namespace wf
