// Internal declarations shared by the libwf sources (host pool + kernels).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "wf.h"

namespace wf {

constexpr int kMaxSlots = WF_MAX_STAGES + 1;
constexpr int kMaxPositions = 1 + WF_MAX_HISTORY + WF_MAX_STAGES + 1;

// Device page table, rewritten (stream-ordered) on every round advance.
// int32 words at these offsets inside the table region of the pool memory:
//   [kTabRound]               round k
//   [kTabNumPos]              number of positions in the ordered context
//   [kTabSlotPos + s]         position index of slot s (store = S), -1 if idle
//   [kTabSlotChunk + s]       chunk index held by slot s, -1 if idle
//   [kTabPosTag + p]          ready tag expected for every page of position p
//   [kTabPosChunk + p]        chunk index of position p
//   [kTabPages + p*npc + j]   physical page of the j-th page of position p
constexpr int kTabRound = 0;
constexpr int kTabNumPos = 1;
constexpr int kTabSlotPos = 2;
constexpr int kTabSlotChunk = kTabSlotPos + kMaxSlots;
constexpr int kTabPosTag = kTabSlotChunk + kMaxSlots;
constexpr int kTabPosChunk = kTabPosTag + kMaxPositions;
constexpr int kTabPages = kTabPosChunk + kMaxPositions;

// Work description of one launch, built on the host from the host mirror.
struct LiveSlots {
  int32_t n;                       // live query slots this round
  int32_t slot[kMaxSlots];         // slot ids (store = S)
  int32_t chunk[kMaxSlots];        // chunk each holds
  int32_t tag[kMaxSlots];          // ready tag its publish writes
  int32_t npos[kMaxSlots];         // context prefix length it reads
};

struct PublishParams {
  const void *q, *k, *v;
  void *q_rot;
  char *pages;                // this layer's page region
  int32_t *tags;              // this layer's ready tags [num_pages]
  const int32_t *table;       // device page table
  int32_t *status;            // sticky status word
  const float2 *rope_t, *rope_h, *rope_w;  // (cos, sin) per position x pair
  float *kv_scale;            // FP8 pool: this layer's [num_pages][2][heads] block scales
  float *q_scale;             // FP8 pool: this layer's [S+1][npc][heads] query-tile scales
  int32_t S1, C, Hh, d, P, npc, num_pages;
  int32_t rope, F, gh, gw, split0, split1, split2;
  LiveSlots live;
};

struct AttnParams {
  const void *q_rot;
  void *out;
  const char *pages;          // this layer's page region
  const int32_t *tags;        // this layer's ready tags
  const int32_t *table;
  int32_t *status;
  int32_t S1, C, Hh, d, P, npc, num_pages, n_pos;
  int64_t layer_row0;         // first pool row of this layer (pool tensor map)
  const float *kv_scale;      // FP8 pool: this layer's [num_pages][2][heads] block scales
  const float *q_scale;       // FP8 pool: this layer's [S+1][npc][heads] query-tile scales
  float scale_log2;           // log2(e) / sqrt(d)
  float scale;                // 1 / sqrt(d)
  long long wait_limit;       // cycles before a bounded wait gives up (tensor-core path)
  int32_t skip_key_tile;      // test hook: key tile whose K load is never issued, else -1
  LiveSlots live;
};

struct ProjectParams {
  void *q_rot;
  char *pages;                // this layer's page region
  int32_t *tags;              // this layer's ready tags
  const int32_t *table;
  int32_t *status;
  const float2 *rope_t, *rope_h, *rope_w;
  int32_t S1, C, Hh, d, P, npc, num_pages, hidden;
  int32_t rope, F, gh, gw, split0, split1, split2;
  int64_t layer_row0;         // first pool row of this layer (pool store tensor map)
  LiveSlots live;
};

// One slot's pages of one layer, copied from this pool into a receiver pool of
// the same geometry (same physical page ids), then the receiver's ready tags.
struct DeliverParams {
  const char *src_pages;      // this pool's page region of the layer
  char *dst_pages;            // the receiver's page region of the layer
  const int32_t *src_tags;    // this pool's ready tags of the layer
  int32_t *dst_tags;          // the receiver's ready tags of the layer
  const float *src_kv_scale;  // FP8 pools: this layer's [num_pages][2][heads] scales, else null
  float *dst_kv_scale;        // FP8 pools: the receiver's, else null
  const int32_t *table;       // this pool's device page table
  int32_t *status;            // this pool's sticky status word
  const uint64_t *dst_signature;   // the receiver's pool signature word
  uint64_t signature;         // this pool's signature (config and page order)
  int32_t slot, npc, Hh, num_pages, tag;   // tag: the slot's ready tag this round
  int64_t tile_bytes;         // one (page, K|V, head) tile: P * d * element size
};

// Byte offset, inside the pool memory's 256-byte status region, of the 64-bit
// signature of the pool's config and page order, written at creation.
constexpr size_t kSignatureOffset = 8;

// Launchers (return a cudaError_t from the launch).
cudaError_t launch_publish_f32(const PublishParams &p, cudaStream_t st);
// The FP8 publish takes unswizzled tensor maps of q, k and v over
// [S+1][C][heads][d] bf16 with a box of 128 dims x 1 head x 128 rows.
cudaError_t launch_publish_fp8(const PublishParams &p, const void *tmap_q, const void *tmap_k,
                               const void *tmap_v, cudaStream_t st);
// The bf16 publish for d = 128 and 128-token pages takes unswizzled maps of q,
// k, v and q_rot over [S+1][C][heads][d] bf16 with a box of 128 dims x 1 head x
// 64 rows, and an unswizzled 2D map over the layer's pool rows
// ([pages x 2 x heads x 128 rows][d] bf16, box 128 x 64).
cudaError_t launch_publish_bf16_tma(const PublishParams &p, const void *tmap_q, const void *tmap_k,
                                    const void *tmap_v, const void *tmap_qrot,
                                    const void *tmap_pages, cudaStream_t st);
cudaError_t launch_attention_f32(const AttnParams &p, cudaStream_t st);
cudaError_t launch_deliver(const DeliverParams &p, cudaStream_t st);
// The bf16 tensor-core path takes the encoded tensor maps (opaque 128-byte
// CUtensorMap objects) of q_rot (box 64 x 1 x 128 rows), the pool's K/V pages
// (box 64 x 128) and out (box 64 x 1 x 32 rows).
cudaError_t launch_attention_bf16(const AttnParams &p, const void *tmap_q,
                                  const void *tmap_kv, const void *tmap_out,
                                  cudaStream_t st);
// The FP8 path: q_rot and the pages are E4M3 bytes (q box 128 x 1 x 128 rows,
// page box 128 x 128), out is bf16 (box 64 x 1 x 32 rows).
cudaError_t launch_attention_fp8(const AttnParams &p, const void *tmap_q,
                                 const void *tmap_kv, const void *tmap_out, cudaStream_t st);
// Fused QKV projection: tensor maps of x (3D: hidden x C x S+1, box 64 x 256 x 1)
// and w_qkv (2D: hidden x 3*hidden, box 64 x 256) for the operands, and the two
// store maps of the epilogue: q_rot (4D [S+1][C][heads][d], box 64 x 1 x 32 x 1)
// and the pool's K/V rows (2D [rows][d], box 64 x 32), all 128-byte swizzled.
cudaError_t launch_project_bf16(const ProjectParams &p, const void *tmap_x, const void *tmap_w,
                                const void *tmap_q, const void *tmap_kv, cudaStream_t st);
cudaError_t launch_table_upload(int32_t *dst, const int32_t *src, int n_words,
                                cudaStream_t st);
cudaError_t launch_poke(int32_t *dst, int32_t value, cudaStream_t st);

#ifdef __CUDACC__
// Record the first device-side error in the sticky status word.
__device__ __forceinline__ void record_status(int32_t *status, int32_t code) {
  atomicCAS(status, 0, code);
}

// Readiness and bounds check of every page in context positions [0, n_pos):
// returns WF_OK, WF_ERR_BAD_PAGE or WF_ERR_NOT_READY (block-uniform).
// Every thread of the block must call it.
__device__ __forceinline__ int check_context_pages(const int32_t *table, const int32_t *tags,
                                                   int n_pos, int npc, int num_pages) {
  int bad_page = 0, stale = 0;
  const int total = n_pos * npc;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int p = i / npc;
    const int pg = __ldcg(table + kTabPages + i);
    if (pg < 0 || pg >= num_pages) {
      bad_page = 1;
    } else if (__ldcg(tags + pg) != __ldcg(table + kTabPosTag + p)) {
      stale = 1;
    }
  }
  if (__syncthreads_or(bad_page)) return WF_ERR_BAD_PAGE;
  if (__syncthreads_or(stale)) return WF_ERR_NOT_READY;
  return WF_OK;
}
#endif

}  // namespace wf
