// Wave Parallelism's one-way K/V delivery into receiver pages, followed by a
// ready signal.
//
// "Wave Forcing: Towards Speed-of-Light Streaming Video Generation", Method
// section and Figure 3c: each stage runs on its own GPU; a stage publishes its
// chunk's K/V right after the QKV projection and RoPE and delivers them
// directly into the ordered attention slots of the stages that read them,
// followed by a ready signal; there is no reverse edge (thelatestinai listing,
// Table 10). Here every rank keeps a full pool whose bookkeeping is the same
// on all ranks (same config, page order and rounds), so a slot's pages have
// the same physical ids everywhere: delivery copies the slot's (page, K|V,
// head) tiles of one layer into the receiver's pool at the same ids, then
// stamps the receiver's ready tags.
//
// Two stream-ordered kernels:
//   * deliver_copy_kernel: one CTA per (page of the slot's chunk, K|V, head)
//     tile; 16-byte loads from this pool, 16-byte stores into the receiver's
//     pool (a peer device's memory over NVLink, or this device's); FP8 pools
//     also copy the tile's block scale. A system-scope fence ends each CTA.
//     Each CTA first checks the receiver's pool signature (config and page
//     order, written at pool creation) and its own page: an id in range whose
//     ready tag in this pool is this round's. A foreign receiver records
//     WF_ERR_INVALID_ARG, a bad id WF_ERR_BAD_PAGE, a stale tag
//     WF_ERR_NOT_READY, and the CTA writes nothing.
//   * deliver_tags_kernel: checks every page of the slot the same way, and
//     only if all pass writes the receiver's ready tags of the slot's pages
//     (stream order after the copy kernel, so after every tile has landed).
// So a receiver's tags are stamped only for a slot whose every page was
// published in this round and copied; a slot that was not published at all
// leaves the receiver untouched.
#include "wf_internal.h"

namespace wf {
namespace {

constexpr int kThreads = 256;

// 0 if page j of the slot is in range and carries the expected tag, else the
// status to record.
__device__ __forceinline__ int check_page(const DeliverParams &p, int pos, int j) {
  const int pg = __ldcg(p.table + kTabPages + pos * p.npc + j);
  if (pg < 0 || pg >= p.num_pages) return WF_ERR_BAD_PAGE;
  if (__ldcg(p.src_tags + pg) != p.tag) return WF_ERR_NOT_READY;
  return 0;
}

__global__ void __launch_bounds__(kThreads) deliver_copy_kernel(const DeliverParams p) {
  const int j = blockIdx.x;                  // page of the slot's chunk
  const int kvh = blockIdx.y;                // K|V x head: kv * heads + h
  __shared__ int verdict;
  if (threadIdx.x == 0) {
    const int pos = __ldcg(p.table + kTabSlotPos + p.slot);
    int st = 0;
    if (*reinterpret_cast<const volatile uint64_t *>(p.dst_signature) != p.signature)
      st = WF_ERR_INVALID_ARG;
    else if (pos < 0)
      st = WF_ERR_BAD_PAGE;
    else
      st = check_page(p, pos, j);
    // one CTA per page records its page's problem (the K|V x head CTAs agree)
    if (st && kvh == 0) record_status(p.status, st);
    verdict = st ? -1 : __ldcg(p.table + kTabPages + pos * p.npc + j);
  }
  __syncthreads();
  const int phys = verdict;
  if (phys < 0) return;
  const size_t tile = static_cast<size_t>(phys) * 2 * p.Hh + kvh;
  const uint4 *src = reinterpret_cast<const uint4 *>(p.src_pages + tile * p.tile_bytes);
  uint4 *dst = reinterpret_cast<uint4 *>(p.dst_pages + tile * p.tile_bytes);
  const int nvec = static_cast<int>(p.tile_bytes / 16);
  for (int i = threadIdx.x; i < nvec; i += kThreads) dst[i] = __ldcg(src + i);
  if (p.src_kv_scale && threadIdx.x == 0) p.dst_kv_scale[tile] = __ldcg(p.src_kv_scale + tile);
  __threadfence_system();
}

__global__ void __launch_bounds__(kThreads) deliver_tags_kernel(const DeliverParams p) {
  if (*reinterpret_cast<const volatile uint64_t *>(p.dst_signature) != p.signature) return;
  const int pos = __ldcg(p.table + kTabSlotPos + p.slot);
  if (pos < 0) return;                       // recorded by the copy kernel
  int bad = 0;
  for (int j = threadIdx.x; j < p.npc; j += kThreads) bad |= check_page(p, pos, j);
  if (__syncthreads_or(bad)) return;         // idem
  for (int j = threadIdx.x; j < p.npc; j += kThreads)
    p.dst_tags[__ldcg(p.table + kTabPages + pos * p.npc + j)] = p.tag;
  __threadfence_system();
}

}  // namespace

cudaError_t launch_deliver(const DeliverParams &p, cudaStream_t st) {
  if (p.npc <= 0 || p.Hh <= 0 || p.tile_bytes <= 0 || p.tile_bytes % 16 != 0)
    return cudaErrorInvalidValue;
  deliver_copy_kernel<<<dim3(static_cast<unsigned>(p.npc), static_cast<unsigned>(2 * p.Hh)),
                        kThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  deliver_tags_kernel<<<1, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace wf
