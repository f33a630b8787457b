// Host side of libwf: the paged K/V pool, its page table and the round state,
// plus the C entry points that launch the kernels.
//
// Round state follows "Wave Forcing: Towards Speed-of-Light Streaming Video
// Generation": Method section (round k = i + s, M_WF(s, j) = 1[j >= s], early
// publication after QKV + RoPE, paged delivery into ordered attention slots
// with a ready signal), the ordered context anchor || bounded clean history ||
// store || denoising K/V ("Como funciona", e-cogni article) and the Table 3
// notation (stage S is the store). Page allocation is this library's own
// policy: a FIFO free list seeded by the caller's page order; denoising slots
// own their pages for good, the store takes fresh pages each round, and the
// history chunk that falls out of the window returns its pages to the list.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <deque>
#include <mutex>
#include <new>
#include <vector>

#include "wf_internal.h"

using namespace wf;

namespace {

enum PosKind { kAnchor = 0, kHistory = 1, kStore = 2, kSlot = 3 };

struct Position {
  int kind;
  int chunk;
  int slot;   // -1 for anchor / history
  int tag;
  std::vector<int32_t> pages;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int32_t tag_of(int S, int64_t round, int slot) {
  return static_cast<int32_t>(round * (S + 1) + slot + 1);
}

struct Geometry {
  int npc = 0, max_pos = 0;
  int64_t num_pages = 0;
  size_t elt = 0;
  size_t status_off = 0, table_off = 0, table_words = 0;
  size_t rope_t_off = 0, rope_h_off = 0, rope_w_off = 0;
  size_t rope_t_n = 0, rope_h_n = 0, rope_w_n = 0;   // float2 entries
  size_t tags_off = 0, pages_off = 0, page_bytes = 0, total = 0;
  size_t kv_scale_off = 0, q_scale_off = 0;           // FP8 pools only (else 0)
  size_t kv_scale_per_layer = 0, q_scale_per_layer = 0;   // floats
};

wf_status validate(const wf_pool_config &c) {
  if (c.num_stages < 1 || c.num_stages > WF_MAX_STAGES) return WF_ERR_INVALID_ARG;
  if (c.chunk_tokens < 1 || c.num_heads < 1 || c.head_dim < 1) return WF_ERR_INVALID_ARG;
  if (c.anchor_chunks != 0 && c.anchor_chunks != 1) return WF_ERR_INVALID_ARG;
  if (c.history_chunks < 0 || c.history_chunks > WF_MAX_HISTORY) return WF_ERR_INVALID_ARG;
  if (c.page_tokens < 1 || c.num_layers < 1 || c.max_rounds < 1) return WF_ERR_INVALID_ARG;
  if (c.num_pages < 0) return WF_ERR_INVALID_ARG;
  if (c.mask_mode != WF_MASK_WF && c.mask_mode != WF_MASK_RF) return WF_ERR_INVALID_ARG;
  if (c.dtype == WF_DTYPE_BF16 || c.dtype == WF_DTYPE_FP8_E4M3) {
    if (c.head_dim != 128 || c.page_tokens != 128) return WF_ERR_UNSUPPORTED;
  } else if (c.dtype == WF_DTYPE_F32) {
    if (c.head_dim % 4 != 0 || c.head_dim > 128) return WF_ERR_UNSUPPORTED;
    if (c.page_tokens > 256) return WF_ERR_UNSUPPORTED;
  } else {
    return WF_ERR_INVALID_ARG;
  }
  if (c.rope == WF_ROPE_3D) {
    if (c.frames_per_chunk < 1 || c.grid_h < 1 || c.grid_w < 1) return WF_ERR_INVALID_ARG;
    if (static_cast<int64_t>(c.frames_per_chunk) * c.grid_h * c.grid_w != c.chunk_tokens)
      return WF_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
      if (c.rope_split[i] < 0 || c.rope_split[i] % 2 != 0) return WF_ERR_INVALID_ARG;
    if (c.rope_split[0] + c.rope_split[1] + c.rope_split[2] != c.head_dim)
      return WF_ERR_INVALID_ARG;
    if (!(c.rope_base > 0.0f)) return WF_ERR_INVALID_ARG;
    if (static_cast<int64_t>(c.max_rounds) * c.frames_per_chunk > (1 << 24))
      return WF_ERR_INVALID_ARG;
  } else if (c.rope != WF_ROPE_OFF) {
    return WF_ERR_INVALID_ARG;
  }
  if (static_cast<int64_t>(c.max_rounds) * (c.num_stages + 1) >= (int64_t(1) << 31))
    return WF_ERR_INVALID_ARG;
  return WF_OK;
}

wf_status geometry(const wf_pool_config &c, Geometry *g) {
  wf_status st = validate(c);
  if (st != WF_OK) return st;
  g->npc = (c.chunk_tokens + c.page_tokens - 1) / c.page_tokens;
  g->max_pos = c.anchor_chunks + c.history_chunks + c.num_stages + 1;
  const int64_t min_pages =
      static_cast<int64_t>(c.num_stages + 1 + c.anchor_chunks + c.history_chunks) * g->npc;
  g->num_pages = c.num_pages == 0 ? min_pages : c.num_pages;
  if (g->num_pages < min_pages) return WF_ERR_OUT_OF_PAGES;
  g->elt = c.dtype == WF_DTYPE_BF16 ? 2 : (c.dtype == WF_DTYPE_F32 ? 4 : 1);
  // Pool rows (one row = one token of one head of K or V) must fit int32 for
  // the tensor-map coordinates of the bf16 path.
  const int64_t rows = static_cast<int64_t>(c.num_layers) * g->num_pages * 2 * c.num_heads *
                       c.page_tokens;
  if (rows >= (int64_t(1) << 31)) return WF_ERR_INVALID_ARG;
  size_t off = 0;
  g->status_off = off;
  off += 256;
  g->table_off = off;
  g->table_words = kTabPages + static_cast<size_t>(g->max_pos) * g->npc;
  off = align_up(off + g->table_words * 4, 256);
  if (c.rope == WF_ROPE_3D) {
    g->rope_t_n = static_cast<size_t>(c.max_rounds) * c.frames_per_chunk * (c.rope_split[0] / 2);
    g->rope_h_n = static_cast<size_t>(c.grid_h) * (c.rope_split[1] / 2);
    g->rope_w_n = static_cast<size_t>(c.grid_w) * (c.rope_split[2] / 2);
    g->rope_t_off = off;
    off = align_up(off + g->rope_t_n * 8, 256);
    g->rope_h_off = off;
    off = align_up(off + g->rope_h_n * 8, 256);
    g->rope_w_off = off;
    off = align_up(off + g->rope_w_n * 8, 256);
  }
  g->tags_off = off;
  off = align_up(off + static_cast<size_t>(c.num_layers) * g->num_pages * 4, 256);
  if (c.dtype == WF_DTYPE_FP8_E4M3) {
    g->kv_scale_per_layer = static_cast<size_t>(g->num_pages) * 2 * c.num_heads;
    g->q_scale_per_layer = static_cast<size_t>(c.num_stages + 1) * g->npc * c.num_heads;
    g->kv_scale_off = off;
    off = align_up(off + c.num_layers * g->kv_scale_per_layer * 4, 256);
    g->q_scale_off = off;
    off = align_up(off + c.num_layers * g->q_scale_per_layer * 4, 256);
  }
  off = align_up(off, 1024);
  g->pages_off = off;
  g->page_bytes = 2 * static_cast<size_t>(c.num_heads) * c.page_tokens * c.head_dim * g->elt;
  off += static_cast<size_t>(c.num_layers) * g->num_pages * g->page_bytes;
  g->total = align_up(off, 256);
  return WF_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 128-byte-swizzled tiled map over bf16 elements or raw bytes (E4M3 codes).
bool encode_map(CUtensorMap *map, CUtensorMapDataType type, void *base, int rank,
                const cuuint64_t *dims, const cuuint64_t *strides_bytes, const cuuint32_t *box) {
  auto fn = get_encode();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, type, rank, base, dims, strides_bytes, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Unswizzled tiled map over bf16 elements (rows of the box land contiguously).
bool encode_plain_bf16_map(CUtensorMap *map, void *base, int rank, const cuuint64_t *dims,
                           const cuuint64_t *strides_bytes, const cuuint32_t *box) {
  auto fn = get_encode();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides_bytes, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_bf16_map(CUtensorMap *map, void *base, int rank, const cuuint64_t *dims,
                     const cuuint64_t *strides_bytes, const cuuint32_t *box) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box);
}

// 64-bit FNV-1a over the bytes of the config (its fields, one by one, so
// that struct padding does not enter), the initial page order and the pool
// size: pools that deliver into each other must agree on all three.
uint64_t pool_signature(const wf_pool_config &c, const std::vector<int32_t> &order, size_t total) {
  uint64_t h = 1469598103934665603ULL;
  auto mix = [&h](const void *data, size_t n) {
    const unsigned char *b = static_cast<const unsigned char *>(data);
    for (size_t i = 0; i < n; ++i) {
      h ^= b[i];
      h *= 1099511628211ULL;
    }
  };
  const int32_t words[] = {c.num_stages, c.chunk_tokens, c.num_heads, c.head_dim,
                           c.anchor_chunks, c.history_chunks, c.page_tokens, c.num_layers,
                           c.dtype, c.rope, c.frames_per_chunk, c.grid_h, c.grid_w,
                           c.rope_split[0], c.rope_split[1], c.rope_split[2], c.max_rounds,
                           c.num_pages, c.mask_mode};
  mix(words, sizeof(words));
  mix(&c.rope_base, sizeof(c.rope_base));
  mix(order.data(), order.size() * sizeof(int32_t));
  const uint64_t t = total;
  mix(&t, sizeof(t));
  return h ? h : 1;
}

}  // namespace

struct wf_pool {
  wf_pool_config cfg{};
  Geometry g;
  uint64_t signature = 0;   // config + page order, also stored in the device memory
  bool host_only = false;
  char *dev = nullptr;
  int device = -1;
  int64_t k = 0;
  std::deque<int32_t> free_list;
  std::vector<std::vector<int32_t>> slot_pages;   // S denoising slots
  std::vector<int32_t> store_pages;
  bool has_store = false;
  bool has_anchor = false;
  std::vector<int32_t> anchor_pages;
  std::deque<std::pair<int, std::vector<int32_t>>> history;
  std::vector<Position> layout;                   // current ordered context
  CUtensorMap kv_map;                             // bf16 / E4M3 pages, 2D rows x d
  // Test hook (wf_pool_debug_stall_next_attention), consumed by the next
  // tensor-core attention launch.
  int32_t stall_key_tile = -1;
  long long stall_wait_limit = 0;
};

namespace {

// Ordered context of the pool's current round from its host state.
void build_layout(wf_pool *p) {
  const int S = p->cfg.num_stages;
  const int64_t k = p->k;
  p->layout.clear();
  if (p->has_anchor) {
    p->layout.push_back({kAnchor, 0, -1, tag_of(S, 0 + S, S), p->anchor_pages});
  }
  for (auto &h : p->history) {
    p->layout.push_back({kHistory, h.first, -1, tag_of(S, h.first + S, S), h.second});
  }
  if (p->has_store) {
    p->layout.push_back({kStore, static_cast<int>(k - S), S, tag_of(S, k, S), p->store_pages});
  }
  for (int s = S - 1; s >= 0; --s) {
    if (k - s >= 0) p->layout.push_back({kSlot, static_cast<int>(k - s), s, tag_of(S, k, s),
                                         p->slot_pages[s]});
  }
}

std::vector<int32_t> table_words(const wf_pool *p) {
  std::vector<int32_t> w(p->g.table_words, 0);
  w[kTabRound] = static_cast<int32_t>(p->k);
  w[kTabNumPos] = static_cast<int32_t>(p->layout.size());
  for (int s = 0; s < kMaxSlots; ++s) {
    w[kTabSlotPos + s] = -1;
    w[kTabSlotChunk + s] = -1;
  }
  for (size_t i = 0; i < p->layout.size(); ++i) {
    const Position &q = p->layout[i];
    if (q.slot >= 0) {
      w[kTabSlotPos + q.slot] = static_cast<int32_t>(i);
      w[kTabSlotChunk + q.slot] = q.chunk;
    }
    w[kTabPosTag + i] = q.tag;
    w[kTabPosChunk + i] = q.chunk;
    for (int j = 0; j < p->g.npc; ++j) w[kTabPages + i * p->g.npc + j] = q.pages[j];
  }
  return w;
}

wf_status upload_table(wf_pool *p, cudaStream_t st) {
  if (p->host_only) return WF_OK;
  std::vector<int32_t> w = table_words(p);
  cudaError_t e = launch_table_upload(reinterpret_cast<int32_t *>(p->dev + p->g.table_off),
                                      w.data(), static_cast<int>(w.size()), st);
  return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

LiveSlots live_slots(const wf_pool *p) {
  LiveSlots l{};
  for (size_t i = 0; i < p->layout.size(); ++i) {
    const Position &q = p->layout[i];
    if (q.slot < 0) continue;
    l.slot[l.n] = q.slot;
    l.chunk[l.n] = q.chunk;
    l.tag[l.n] = q.tag;
    // WF: the context prefix up to its own entry; RF: the whole context.
    l.npos[l.n] = p->cfg.mask_mode == WF_MASK_RF ? static_cast<int32_t>(p->layout.size())
                                                  : static_cast<int32_t>(i) + 1;
    ++l.n;
  }
  return l;
}

// Keep only `slot` in the live list (slot < 0 keeps every slot); false if the
// slot is not live in the current round.
bool select_slot(LiveSlots &l, int32_t slot) {
  if (slot < 0) return true;
  for (int i = 0; i < l.n; ++i) {
    if (l.slot[i] != slot) continue;
    LiveSlots one{};
    one.n = 1;
    one.slot[0] = l.slot[i];
    one.chunk[0] = l.chunk[i];
    one.tag[0] = l.tag[i];
    one.npos[0] = l.npos[i];
    l = one;
    return true;
  }
  return false;
}

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool on_pool_device(const wf_pool *p) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == p->device;
}

}  // namespace

extern "C" {

const char *wf_status_string(wf_status s) {
  switch (s) {
    case WF_OK: return "WF_OK";
    case WF_ERR_INVALID_ARG: return "WF_ERR_INVALID_ARG: invalid argument";
    case WF_ERR_OUT_OF_PAGES: return "WF_ERR_OUT_OF_PAGES: pool has too few pages";
    case WF_ERR_NOT_READY: return "WF_ERR_NOT_READY: K/V page read before it was published";
    case WF_ERR_BAD_PAGE: return "WF_ERR_BAD_PAGE: page id outside the pool";
    case WF_ERR_CALL_ORDER: return "WF_ERR_CALL_ORDER: call not allowed in this pool state";
    case WF_ERR_CUDA: return "WF_ERR_CUDA: CUDA call failed";
    case WF_ERR_UNSUPPORTED: return "WF_ERR_UNSUPPORTED: shape/dtype not supported";
    case WF_ERR_TIMEOUT: return "WF_ERR_TIMEOUT: a bounded device wait ran out";
  }
  return "unknown wf_status";
}

wf_status wf_kv_pool_bytes(const wf_pool_config *cfg, size_t *bytes) {
  if (!cfg || !bytes) return WF_ERR_INVALID_ARG;
  Geometry g;
  wf_status st = geometry(*cfg, &g);
  if (st != WF_OK) return st;
  *bytes = g.total;
  return WF_OK;
}

wf_status wf_kv_pool_create(const wf_pool_config *cfg, void *dev_mem, size_t bytes,
                            const int32_t *page_order, wf_stream_t stream, wf_pool **out) {
  if (!cfg || !out) return WF_ERR_INVALID_ARG;
  *out = nullptr;
  Geometry g;
  wf_status st = geometry(*cfg, &g);
  if (st != WF_OK) return st;
  const bool host_only = dev_mem == nullptr;
  if (!host_only) {
    if (bytes < g.total) return WF_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(dev_mem) & 255u) return WF_ERR_INVALID_ARG;
  }
  std::vector<int32_t> order(static_cast<size_t>(g.num_pages));
  if (page_order) {
    std::vector<char> seen(order.size(), 0);
    for (size_t i = 0; i < order.size(); ++i) {
      const int32_t v = page_order[i];
      if (v < 0 || v >= g.num_pages || seen[v]) return WF_ERR_INVALID_ARG;
      seen[v] = 1;
      order[i] = v;
    }
  } else {
    for (size_t i = 0; i < order.size(); ++i) order[i] = static_cast<int32_t>(i);
  }

  wf_pool *p = new (std::nothrow) wf_pool();
  if (!p) return WF_ERR_INVALID_ARG;
  p->cfg = *cfg;
  p->g = g;
  p->host_only = host_only;
  p->dev = static_cast<char *>(dev_mem);
  p->signature = pool_signature(*cfg, order, g.total);
  p->free_list.assign(order.begin(), order.end());
  const int S = cfg->num_stages;
  p->slot_pages.resize(S);
  for (int s = 0; s < S; ++s)
    for (int j = 0; j < g.npc; ++j) {
      p->slot_pages[s].push_back(p->free_list.front());
      p->free_list.pop_front();
    }
  build_layout(p);

  if (!host_only) {
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (cudaGetDevice(&p->device) != cudaSuccess) { delete p; return WF_ERR_CUDA; }
    cudaError_t e = cudaMemsetAsync(p->dev, 0, g.pages_off, cs);   // status, table, tags
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(p->dev + g.status_off + kSignatureOffset, &p->signature,
                          sizeof(p->signature), cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);   // the signature's source is on this stack
    if (e == cudaSuccess && cfg->rope == WF_ROPE_3D) {
      // (cos, sin) of angle = pos * base^(-2m / width), in float64, rounded to fp32.
      const int widths[3] = {cfg->rope_split[0], cfg->rope_split[1], cfg->rope_split[2]};
      const size_t npos[3] = {static_cast<size_t>(cfg->max_rounds) * cfg->frames_per_chunk,
                              static_cast<size_t>(cfg->grid_h),
                              static_cast<size_t>(cfg->grid_w)};
      const size_t offs[3] = {g.rope_t_off, g.rope_h_off, g.rope_w_off};
      std::vector<float> tab;
      for (int a = 0; a < 3 && e == cudaSuccess; ++a) {
        const int half = widths[a] / 2;
        tab.assign(npos[a] * half * 2, 0.0f);
        for (size_t pos = 0; pos < npos[a]; ++pos)
          for (int m = 0; m < half; ++m) {
            const double inv = std::pow(static_cast<double>(cfg->rope_base),
                                        -2.0 * m / static_cast<double>(widths[a]));
            const double ang = static_cast<double>(pos) * inv;
            tab[(pos * half + m) * 2 + 0] = static_cast<float>(std::cos(ang));
            tab[(pos * half + m) * 2 + 1] = static_cast<float>(std::sin(ang));
          }
        if (!tab.empty())
          e = cudaMemcpyAsync(p->dev + offs[a], tab.data(), tab.size() * sizeof(float),
                              cudaMemcpyHostToDevice, cs);
        if (e == cudaSuccess) e = cudaStreamSynchronize(cs);   // tab is reused
      }
    }
    if (e != cudaSuccess) { delete p; return WF_ERR_CUDA; }
    if (upload_table(p, cs) != WF_OK || cudaStreamSynchronize(cs) != cudaSuccess) {
      delete p;
      return WF_ERR_CUDA;
    }
    if (cfg->dtype == WF_DTYPE_BF16 || cfg->dtype == WF_DTYPE_FP8_E4M3) {
      // One pool row = one token of one head of K or V: 128 elements.
      const bool f8 = cfg->dtype == WF_DTYPE_FP8_E4M3;
      const cuuint64_t rows = static_cast<cuuint64_t>(cfg->num_layers) * g.num_pages * 2 *
                              cfg->num_heads * cfg->page_tokens;
      const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cfg->head_dim), rows};
      const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cfg->head_dim) * g.elt};
      const cuuint32_t box[2] = {f8 ? 128u : 64u, static_cast<cuuint32_t>(cfg->page_tokens)};
      if (!encode_map(&p->kv_map, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                      p->dev + g.pages_off, 2, dims, strides, box)) {
        delete p;
        return WF_ERR_CUDA;
      }
    }
  }
  *out = p;
  return WF_OK;
}

}  // extern "C"

namespace {

// Publication of every live slot (only_slot < 0) or of one live slot.
wf_status publish_impl(wf_pool *p, int32_t layer, const void *q, const void *k, const void *v,
                       void *q_rot, int32_t only_slot, wf_stream_t stream) {
  if (!p) return WF_ERR_INVALID_ARG;
  if (p->host_only) return WF_ERR_CALL_ORDER;
  const wf_pool_config &c = p->cfg;
  if (layer < 0 || layer >= c.num_layers) return WF_ERR_INVALID_ARG;
  if (!q || !k || !v || !q_rot) return WF_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_rot))
    return WF_ERR_INVALID_ARG;
  if (q_rot == q || q_rot == k || q_rot == v) return WF_ERR_INVALID_ARG;
  if (!on_pool_device(p)) return WF_ERR_INVALID_ARG;
  PublishParams pp{};
  pp.q = q; pp.k = k; pp.v = v; pp.q_rot = q_rot;
  pp.pages = p->dev + p->g.pages_off + static_cast<size_t>(layer) * p->g.num_pages * p->g.page_bytes;
  pp.tags = reinterpret_cast<int32_t *>(p->dev + p->g.tags_off) +
            static_cast<size_t>(layer) * p->g.num_pages;
  pp.table = reinterpret_cast<const int32_t *>(p->dev + p->g.table_off);
  pp.status = reinterpret_cast<int32_t *>(p->dev + p->g.status_off);
  if (c.rope == WF_ROPE_3D) {
    pp.rope_t = reinterpret_cast<const float2 *>(p->dev + p->g.rope_t_off);
    pp.rope_h = reinterpret_cast<const float2 *>(p->dev + p->g.rope_h_off);
    pp.rope_w = reinterpret_cast<const float2 *>(p->dev + p->g.rope_w_off);
  }
  pp.S1 = c.num_stages + 1; pp.C = c.chunk_tokens; pp.Hh = c.num_heads; pp.d = c.head_dim;
  pp.P = c.page_tokens; pp.npc = p->g.npc; pp.num_pages = static_cast<int32_t>(p->g.num_pages);
  pp.rope = c.rope; pp.F = c.frames_per_chunk; pp.gh = c.grid_h; pp.gw = c.grid_w;
  pp.split0 = c.rope_split[0]; pp.split1 = c.rope_split[1]; pp.split2 = c.rope_split[2];
  pp.live = live_slots(p);
  if (only_slot > c.num_stages) return WF_ERR_INVALID_ARG;
  if (!select_slot(pp.live, only_slot)) return WF_ERR_CALL_ORDER;
  if (c.dtype == WF_DTYPE_FP8_E4M3) {
    pp.kv_scale = reinterpret_cast<float *>(p->dev + p->g.kv_scale_off) +
                  static_cast<size_t>(layer) * p->g.kv_scale_per_layer;
    pp.q_scale = reinterpret_cast<float *>(p->dev + p->g.q_scale_off) +
                 static_cast<size_t>(layer) * p->g.q_scale_per_layer;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (c.dtype == WF_DTYPE_FP8_E4M3 || c.dtype == WF_DTYPE_BF16) {   // d = P = 128 (validate)
    // [S+1][C][heads][d] bf16; one box is a 128-row (FP8 publish) or 64-row
    // (bf16 publish) tile of one head.
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(c.head_dim),
                                static_cast<cuuint64_t>(c.num_heads),
                                static_cast<cuuint64_t>(c.chunk_tokens),
                                static_cast<cuuint64_t>(c.num_stages + 1)};
    const cuuint64_t row = static_cast<cuuint64_t>(c.head_dim) * 2;
    const cuuint64_t strides[3] = {row, row * c.num_heads, row * c.num_heads * c.chunk_tokens};
    const cuuint32_t box[4] = {128, 1, c.dtype == WF_DTYPE_FP8_E4M3 ? 128u : 64u, 1};
    CUtensorMap mq, mk, mv;
    if (!encode_plain_bf16_map(&mq, const_cast<void *>(q), 4, dims, strides, box) ||
        !encode_plain_bf16_map(&mk, const_cast<void *>(k), 4, dims, strides, box) ||
        !encode_plain_bf16_map(&mv, const_cast<void *>(v), 4, dims, strides, box))
      return WF_ERR_CUDA;
    if (c.dtype == WF_DTYPE_FP8_E4M3) {
      e = launch_publish_fp8(pp, &mq, &mk, &mv, cs);
    } else {
      // q_rot as the inputs; the layer's pages as [pages x 2 x heads x P rows][d],
      // box 64 rows.
      const cuuint64_t pdims[2] = {static_cast<cuuint64_t>(c.head_dim),
                                   static_cast<cuuint64_t>(p->g.num_pages) * 2 * c.num_heads *
                                       c.page_tokens};
      const cuuint64_t pstrides[1] = {row};
      const cuuint32_t pbox[2] = {128, 64};
      CUtensorMap mqr, mpg;
      if (!encode_plain_bf16_map(&mqr, q_rot, 4, dims, strides, box) ||
          !encode_plain_bf16_map(&mpg, pp.pages, 2, pdims, pstrides, pbox))
        return WF_ERR_CUDA;
      e = launch_publish_bf16_tma(pp, &mq, &mk, &mv, &mqr, &mpg, cs);
    }
  } else {
    e = launch_publish_f32(pp, cs);
  }
  return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

// Round attention of every live slot (only_slot < 0) or of one live slot, whose
// readiness check then covers only the context prefix it reads.
wf_status attention_impl(wf_pool *p, int32_t layer, const void *q_rot, void *out,
                         int32_t only_slot, wf_stream_t stream) {
  if (!p) return WF_ERR_INVALID_ARG;
  if (p->host_only) return WF_ERR_CALL_ORDER;
  const wf_pool_config &c = p->cfg;
  if (layer < 0 || layer >= c.num_layers) return WF_ERR_INVALID_ARG;
  if (!q_rot || !out || !aligned16(q_rot) || !aligned16(out)) return WF_ERR_INVALID_ARG;
  if (q_rot == out) return WF_ERR_INVALID_ARG;
  if (!on_pool_device(p)) return WF_ERR_INVALID_ARG;
  AttnParams ap{};
  ap.q_rot = q_rot; ap.out = out;
  ap.pages = p->dev + p->g.pages_off + static_cast<size_t>(layer) * p->g.num_pages * p->g.page_bytes;
  ap.tags = reinterpret_cast<const int32_t *>(p->dev + p->g.tags_off) +
            static_cast<size_t>(layer) * p->g.num_pages;
  ap.table = reinterpret_cast<const int32_t *>(p->dev + p->g.table_off);
  ap.status = reinterpret_cast<int32_t *>(p->dev + p->g.status_off);
  ap.S1 = c.num_stages + 1; ap.C = c.chunk_tokens; ap.Hh = c.num_heads; ap.d = c.head_dim;
  ap.P = c.page_tokens; ap.npc = p->g.npc; ap.num_pages = static_cast<int32_t>(p->g.num_pages);
  ap.n_pos = static_cast<int32_t>(p->layout.size());
  ap.layer_row0 = static_cast<int64_t>(layer) * p->g.num_pages * 2 * c.num_heads * c.page_tokens;
  ap.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(c.head_dim)));
  ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.head_dim)));
  ap.live = live_slots(p);
  if (only_slot > c.num_stages) return WF_ERR_INVALID_ARG;
  if (!select_slot(ap.live, only_slot)) return WF_ERR_CALL_ORDER;
  if (only_slot >= 0) ap.n_pos = ap.live.npos[0];
  ap.wait_limit = 2000000000LL;   // ~1 s at 2 GHz
  ap.skip_key_tile = -1;
  if (p->stall_key_tile >= 0 && c.dtype != WF_DTYPE_F32) {
    ap.skip_key_tile = p->stall_key_tile;
    ap.wait_limit = p->stall_wait_limit;
    p->stall_key_tile = -1;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (c.dtype == WF_DTYPE_BF16 || c.dtype == WF_DTYPE_FP8_E4M3) {
    const bool f8 = c.dtype == WF_DTYPE_FP8_E4M3;
    // [S+1][C][heads][d] activations; q_rot in the pool's element type, out bf16.
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(c.head_dim),
                                static_cast<cuuint64_t>(c.num_heads),
                                static_cast<cuuint64_t>(c.chunk_tokens),
                                static_cast<cuuint64_t>(c.num_stages + 1)};
    auto strides_of = [&](cuuint64_t elt, cuuint64_t *st) {
      st[0] = static_cast<cuuint64_t>(c.head_dim) * elt;
      st[1] = st[0] * c.num_heads;
      st[2] = st[1] * c.chunk_tokens;
    };
    cuuint64_t qstr[3], ostr[3];
    strides_of(p->g.elt, qstr);
    strides_of(2, ostr);
    CUtensorMap qmap, omap;
    const cuuint32_t qbox[4] = {f8 ? 128u : 64u, 1, 128, 1};
    if (!encode_map(&qmap, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    const_cast<void *>(q_rot), 4, dims, qstr, qbox))
      return WF_ERR_CUDA;
    const cuuint32_t obox[4] = {64, 1, 32, 1};
    if (!encode_bf16_map(&omap, out, 4, dims, ostr, obox)) return WF_ERR_CUDA;
    if (f8) {
      ap.kv_scale = reinterpret_cast<const float *>(p->dev + p->g.kv_scale_off) +
                    static_cast<size_t>(layer) * p->g.kv_scale_per_layer;
      ap.q_scale = reinterpret_cast<const float *>(p->dev + p->g.q_scale_off) +
                   static_cast<size_t>(layer) * p->g.q_scale_per_layer;
      e = launch_attention_fp8(ap, &qmap, &p->kv_map, &omap, cs);
    } else {
      e = launch_attention_bf16(ap, &qmap, &p->kv_map, &omap, cs);
    }
  } else {
    e = launch_attention_f32(ap, cs);
  }
  return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

}  // namespace

extern "C" {

wf_status wf_publish_kv(wf_pool *p, int32_t layer, const void *q, const void *k, const void *v,
                        void *q_rot, wf_stream_t stream) {
  return publish_impl(p, layer, q, k, v, q_rot, -1, stream);
}

wf_status wf_publish_kv_slot(wf_pool *p, int32_t layer, int32_t slot, const void *q,
                             const void *k, const void *v, void *q_rot, wf_stream_t stream) {
  if (slot < 0) return WF_ERR_INVALID_ARG;
  return publish_impl(p, layer, q, k, v, q_rot, slot, stream);
}

wf_status wf_round_attention(wf_pool *p, int32_t layer, const void *q_rot, void *out,
                             wf_stream_t stream) {
  return attention_impl(p, layer, q_rot, out, -1, stream);
}

wf_status wf_round_attention_slot(wf_pool *p, int32_t layer, int32_t slot, const void *q_rot,
                                  void *out, wf_stream_t stream) {
  if (slot < 0) return WF_ERR_INVALID_ARG;
  return attention_impl(p, layer, q_rot, out, slot, stream);
}

wf_status wf_deliver_kv(const wf_pool *p, int32_t layer, int32_t slot, void *dst_pool_mem,
                        size_t dst_pool_bytes, wf_stream_t stream) {
  if (!p || !dst_pool_mem) return WF_ERR_INVALID_ARG;
  if (p->host_only) return WF_ERR_CALL_ORDER;
  if (dst_pool_bytes != p->g.total) return WF_ERR_INVALID_ARG;
  const wf_pool_config &c = p->cfg;
  if (layer < 0 || layer >= c.num_layers) return WF_ERR_INVALID_ARG;
  if (slot < 0 || slot > c.num_stages) return WF_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(dst_pool_mem) & 255u) != 0) return WF_ERR_INVALID_ARG;
  if (dst_pool_mem == p->dev) return WF_ERR_INVALID_ARG;
  if (!on_pool_device(p)) return WF_ERR_INVALID_ARG;
  LiveSlots l = live_slots(p);
  if (!select_slot(l, slot)) return WF_ERR_CALL_ORDER;
  char *dst = static_cast<char *>(dst_pool_mem);
  const size_t page_off = p->g.pages_off + static_cast<size_t>(layer) * p->g.num_pages * p->g.page_bytes;
  const size_t tag_off = p->g.tags_off + static_cast<size_t>(layer) * p->g.num_pages * sizeof(int32_t);
  DeliverParams dp{};
  dp.src_pages = p->dev + page_off;
  dp.dst_pages = dst + page_off;
  dp.src_tags = reinterpret_cast<const int32_t *>(p->dev + tag_off);
  dp.dst_tags = reinterpret_cast<int32_t *>(dst + tag_off);
  if (c.dtype == WF_DTYPE_FP8_E4M3) {
    const size_t sc_off = p->g.kv_scale_off + static_cast<size_t>(layer) * p->g.kv_scale_per_layer * sizeof(float);
    dp.src_kv_scale = reinterpret_cast<const float *>(p->dev + sc_off);
    dp.dst_kv_scale = reinterpret_cast<float *>(dst + sc_off);
  }
  dp.table = reinterpret_cast<const int32_t *>(p->dev + p->g.table_off);
  dp.status = reinterpret_cast<int32_t *>(p->dev + p->g.status_off);
  dp.dst_signature = reinterpret_cast<const uint64_t *>(dst + p->g.status_off + kSignatureOffset);
  dp.signature = p->signature;
  dp.slot = slot; dp.npc = p->g.npc; dp.Hh = c.num_heads;
  dp.num_pages = static_cast<int32_t>(p->g.num_pages); dp.tag = l.tag[0];
  dp.tile_bytes = static_cast<int64_t>(c.page_tokens) * c.head_dim * p->g.elt;
  const cudaError_t e = launch_deliver(dp, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

wf_status wf_project_publish(wf_pool *p, int32_t layer, const void *x, const void *w_qkv,
                             void *q_rot, wf_stream_t stream) {
  if (!p) return WF_ERR_INVALID_ARG;
  if (p->host_only) return WF_ERR_CALL_ORDER;
  const wf_pool_config &c = p->cfg;
  if (c.dtype != WF_DTYPE_BF16) return WF_ERR_UNSUPPORTED;
  const int hidden = c.num_heads * c.head_dim;
  if (hidden % 256 != 0 || c.page_tokens != 128) return WF_ERR_UNSUPPORTED;
  if (layer < 0 || layer >= c.num_layers) return WF_ERR_INVALID_ARG;
  if (!x || !w_qkv || !q_rot || !aligned16(x) || !aligned16(w_qkv) || !aligned16(q_rot))
    return WF_ERR_INVALID_ARG;
  if (q_rot == x || q_rot == w_qkv) return WF_ERR_INVALID_ARG;
  if (!on_pool_device(p)) return WF_ERR_INVALID_ARG;
  ProjectParams pp{};
  pp.q_rot = q_rot;
  pp.pages = p->dev + p->g.pages_off + static_cast<size_t>(layer) * p->g.num_pages * p->g.page_bytes;
  pp.tags = reinterpret_cast<int32_t *>(p->dev + p->g.tags_off) +
            static_cast<size_t>(layer) * p->g.num_pages;
  pp.table = reinterpret_cast<const int32_t *>(p->dev + p->g.table_off);
  pp.status = reinterpret_cast<int32_t *>(p->dev + p->g.status_off);
  if (c.rope == WF_ROPE_3D) {
    pp.rope_t = reinterpret_cast<const float2 *>(p->dev + p->g.rope_t_off);
    pp.rope_h = reinterpret_cast<const float2 *>(p->dev + p->g.rope_h_off);
    pp.rope_w = reinterpret_cast<const float2 *>(p->dev + p->g.rope_w_off);
  }
  pp.S1 = c.num_stages + 1; pp.C = c.chunk_tokens; pp.Hh = c.num_heads; pp.d = c.head_dim;
  pp.P = c.page_tokens; pp.npc = p->g.npc; pp.num_pages = static_cast<int32_t>(p->g.num_pages);
  pp.hidden = hidden;
  pp.rope = c.rope; pp.F = c.frames_per_chunk; pp.gh = c.grid_h; pp.gw = c.grid_w;
  pp.split0 = c.rope_split[0]; pp.split1 = c.rope_split[1]; pp.split2 = c.rope_split[2];
  pp.layer_row0 = static_cast<int64_t>(layer) * p->g.num_pages * 2 * c.num_heads * c.page_tokens;
  pp.live = live_slots(p);
  CUtensorMap xmap, wmap, qmap, kvmap;
  const cuuint64_t xd[3] = {static_cast<cuuint64_t>(hidden), static_cast<cuuint64_t>(c.chunk_tokens),
                            static_cast<cuuint64_t>(c.num_stages + 1)};
  const cuuint64_t xs[2] = {static_cast<cuuint64_t>(hidden) * 2,
                            static_cast<cuuint64_t>(hidden) * 2 * c.chunk_tokens};
  const cuuint32_t xb[3] = {64, 128, 1};   // one page per CTA of a pair
  if (!encode_bf16_map(&xmap, const_cast<void *>(x), 3, xd, xs, xb)) return WF_ERR_CUDA;
  const cuuint64_t wd[2] = {static_cast<cuuint64_t>(hidden), static_cast<cuuint64_t>(3 * hidden)};
  const cuuint64_t ws[1] = {static_cast<cuuint64_t>(hidden) * 2};
  const cuuint32_t wb[2] = {64, 128};      // half of a tile's features per CTA
  if (!encode_bf16_map(&wmap, const_cast<void *>(w_qkv), 2, wd, ws, wb)) return WF_ERR_CUDA;
  // Epilogue stores: q_rot [S+1][C][heads][d] and the pool's K/V rows, 32 rows per box.
  const cuuint64_t qd[4] = {static_cast<cuuint64_t>(c.head_dim), static_cast<cuuint64_t>(c.num_heads),
                            static_cast<cuuint64_t>(c.chunk_tokens),
                            static_cast<cuuint64_t>(c.num_stages + 1)};
  const cuuint64_t qs[3] = {static_cast<cuuint64_t>(c.head_dim) * 2,
                            static_cast<cuuint64_t>(c.head_dim) * 2 * c.num_heads,
                            static_cast<cuuint64_t>(c.head_dim) * 2 * c.num_heads * c.chunk_tokens};
  const cuuint32_t qb[4] = {64, 1, 32, 1};
  if (!encode_bf16_map(&qmap, q_rot, 4, qd, qs, qb)) return WF_ERR_CUDA;
  const cuuint64_t kd[2] = {static_cast<cuuint64_t>(c.head_dim),
                            static_cast<cuuint64_t>(c.num_layers) * p->g.num_pages * 2 *
                                c.num_heads * c.page_tokens};
  const cuuint64_t ks[1] = {static_cast<cuuint64_t>(c.head_dim) * 2};
  const cuuint32_t kb[2] = {64, 32};
  if (!encode_bf16_map(&kvmap, p->dev + p->g.pages_off, 2, kd, ks, kb)) return WF_ERR_CUDA;
  cudaError_t e = launch_project_bf16(pp, &xmap, &wmap, &qmap, &kvmap,
                                      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

wf_status wf_advance_round(wf_pool *p, wf_stream_t stream) {
  if (!p) return WF_ERR_INVALID_ARG;
  const int S = p->cfg.num_stages;
  if (p->k + 1 >= p->cfg.max_rounds) return WF_ERR_CALL_ORDER;
  if (!p->host_only && !on_pool_device(p)) return WF_ERR_INVALID_ARG;
  if (p->has_store) {
    const int c = static_cast<int>(p->k - S);
    if (p->cfg.anchor_chunks == 1 && c == 0) {
      p->anchor_pages = p->store_pages;
      p->has_anchor = true;
    } else {
      p->history.emplace_back(c, p->store_pages);
      if (static_cast<int>(p->history.size()) > p->cfg.history_chunks) {
        for (int32_t pg : p->history.front().second) p->free_list.push_back(pg);
        p->history.pop_front();
      }
    }
    p->store_pages.clear();
    p->has_store = false;
  }
  p->k += 1;
  if (p->k >= S) {
    if (static_cast<int>(p->free_list.size()) < p->g.npc) return WF_ERR_OUT_OF_PAGES;
    for (int j = 0; j < p->g.npc; ++j) {
      p->store_pages.push_back(p->free_list.front());
      p->free_list.pop_front();
    }
    p->has_store = true;
  }
  build_layout(p);
  return upload_table(p, reinterpret_cast<cudaStream_t>(stream));
}

wf_status wf_pool_check_status(wf_pool *p, wf_stream_t stream) {
  if (!p) return WF_ERR_INVALID_ARG;
  if (p->host_only) return WF_OK;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return WF_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, p->dev + p->g.status_off, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return WF_ERR_CUDA;
  if (v != 0) {
    if (cudaMemset(p->dev + p->g.status_off, 0, 4) != cudaSuccess) return WF_ERR_CUDA;
  }
  return static_cast<wf_status>(v);
}

wf_status wf_pool_destroy(wf_pool *p) {
  if (!p) return WF_ERR_INVALID_ARG;
  delete p;
  return WF_OK;
}

int64_t wf_pool_round(const wf_pool *p) { return p ? p->k : -1; }

wf_status wf_pool_get_geometry(const wf_pool *p, wf_pool_geometry *geom) {
  if (!p || !geom) return WF_ERR_INVALID_ARG;
  geom->num_pages = p->g.num_pages;
  geom->pages_per_chunk = p->g.npc;
  geom->max_positions = p->g.max_pos;
  geom->status_offset = p->g.status_off;
  geom->tags_offset = p->g.tags_off;
  geom->pages_offset = p->g.pages_off;
  geom->page_bytes = p->g.page_bytes;
  geom->total_bytes = p->g.total;
  geom->kv_scale_offset = p->g.kv_scale_off;
  geom->q_scale_offset = p->g.q_scale_off;
  return WF_OK;
}

wf_status wf_pool_get_layout(const wf_pool *p, int32_t *n_positions, int32_t *kinds,
                             int32_t *chunks, int32_t *slots, int32_t *tags, int32_t *pages,
                             int32_t cap) {
  if (!p) return WF_ERR_INVALID_ARG;
  const int n = static_cast<int>(p->layout.size());
  if (n_positions) *n_positions = n;
  for (int i = 0; i < n && i < cap; ++i) {
    const Position &q = p->layout[i];
    if (kinds) kinds[i] = q.kind;
    if (chunks) chunks[i] = q.chunk;
    if (slots) slots[i] = q.slot;
    if (tags) tags[i] = q.tag;
    if (pages)
      for (int j = 0; j < p->g.npc; ++j) pages[i * p->g.npc + j] = q.pages[j];
  }
  return WF_OK;
}

wf_status wf_pool_debug_stall_next_attention(wf_pool *p, int32_t key_tile,
                                             int64_t wait_limit_cycles) {
  if (!p) return WF_ERR_INVALID_ARG;
  if (p->host_only) return WF_ERR_CALL_ORDER;
  if (p->cfg.dtype == WF_DTYPE_F32) return WF_ERR_UNSUPPORTED;
  if (key_tile < 0 || wait_limit_cycles < 1000 || wait_limit_cycles > 2000000000LL)
    return WF_ERR_INVALID_ARG;
  p->stall_key_tile = key_tile;
  p->stall_wait_limit = wait_limit_cycles;
  return WF_OK;
}

wf_status wf_pool_debug_poke_page(wf_pool *p, int32_t position, int32_t j, int32_t physical,
                                  wf_stream_t stream) {
  if (!p) return WF_ERR_INVALID_ARG;
  if (p->host_only) return WF_ERR_CALL_ORDER;
  if (position < 0 || position >= p->g.max_pos || j < 0 || j >= p->g.npc)
    return WF_ERR_INVALID_ARG;
  int32_t *dst = reinterpret_cast<int32_t *>(p->dev + p->g.table_off) + kTabPages +
                 position * p->g.npc + j;
  return launch_poke(dst, physical, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? WF_OK
             : WF_ERR_CUDA;
}

}  // extern "C"
