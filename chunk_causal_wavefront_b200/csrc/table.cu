// Stream-ordered writes of the device page table.
//
// The new table travels inside the kernel's parameter block, so the host
// buffer it came from can be reused as soon as the launch returns and the
// write lands in stream order between the kernels of two rounds.
#include "wf_internal.h"

namespace wf {
namespace {

constexpr int kWordsPerLaunch = 960;   // keeps the parameter block under 4 KB

struct TablePayload {
  int32_t n;
  int32_t w[kWordsPerLaunch];
};

__global__ void table_upload_kernel(int32_t *dst, const TablePayload payload) {
  for (int i = threadIdx.x; i < payload.n; i += blockDim.x) dst[i] = payload.w[i];
}

__global__ void poke_kernel(int32_t *dst, int32_t value) { *dst = value; }

}  // namespace

cudaError_t launch_table_upload(int32_t *dst, const int32_t *src, int n_words, cudaStream_t st) {
  for (int base = 0; base < n_words; base += kWordsPerLaunch) {
    TablePayload p;
    p.n = n_words - base < kWordsPerLaunch ? n_words - base : kWordsPerLaunch;
    for (int i = 0; i < p.n; ++i) p.w[i] = src[base + i];
    table_upload_kernel<<<1, 256, 0, st>>>(dst + base, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_poke(int32_t *dst, int32_t value, cudaStream_t st) {
  poke_kernel<<<1, 1, 0, st>>>(dst, value);
  return cudaGetLastError();
}

}  // namespace wf
