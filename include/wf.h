/*
 * wf.h - C ABI of libwf: one causal-wavefront round of chunk-wise causal
 * attention (Wave Forcing), on one NVIDIA B200 (sm_100a).
 *
 * Source: "Wave Forcing: Towards Speed-of-Light Streaming Video Generation"
 * (arXiv 2611.00859). The method, as the pages state it:
 *   - Method section (hyper.ai summary): a stage-s update of chunk i runs in
 *     round k = i + s; full attention inside each chunk, chunk-wise causal
 *     attention across chunks, mask M_WF(s, j) = 1[j >= s] (query slot s reads
 *     itself and every cleaner slot j, never a noisier one); K/V are published
 *     right after the QKV projection and RoPE, readiness is checked just before
 *     attention, and paged delivery writes K/V straight into ordered attention
 *     slots followed by a ready signal.
 *   - "Como funciona" (e-cogni article): the ordered context of a layer is
 *     anchor (initial chunk) || bounded clean history || live store ||
 *     denoising K/V.
 *   - Appendix Table 3: stages 0 <= s < S, the store is stage S; B_i = Z_i(S).
 *
 * Conventions for every call:
 *   - Pointers named q, k, v, q_rot, out and dev_mem are DEVICE pointers on the
 *     current CUDA device; dst_pool_mem (wf_deliver_kv) is a device pointer
 *     addressable from it (its own memory or a peer device's); config structs
 *     and page_order are HOST pointers.
 *   - Activations are laid out [S+1][C][num_heads][head_dim], row-major, in the
 *     pool's dtype (bf16 or fp32; FP8 pools: see WF_DTYPE_FP8_E4M3): slot-major,
 *     then token, head, dimension.
 *     Slot s < S holds the chunk at denoising stage s; slot S is the store.
 *   - Every call that takes a stream enqueues its device work on that stream
 *     (NULL = legacy default stream) and returns without synchronising, except
 *     wf_kv_pool_create (synchronises once, at set-up) and
 *     wf_pool_check_status. No call allocates device memory.
 *   - Errors found on the host return at once and enqueue nothing. Errors found
 *     by a kernel (a slot read before it was published, a page id out of range)
 *     are recorded in a sticky status word inside the pool memory; the kernel
 *     that found them writes no output, and the next wf_pool_check_status
 *     returns (and clears) the first one recorded.
 *   - A pool is not thread-safe; calls on one pool must be issued in program
 *     order on one stream (or streams ordered by the caller).
 */
#ifndef WF_H_
#define WF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *wf_stream_t;

typedef enum {
  WF_OK = 0,
  WF_ERR_INVALID_ARG = 1,   /* bad config, pointer, size, layer or alignment */
  WF_ERR_OUT_OF_PAGES = 2,  /* num_pages below the minimum the schedule needs */
  WF_ERR_NOT_READY = 3,     /* attention found a page whose ready tag is stale */
  WF_ERR_BAD_PAGE = 4,      /* a page-table entry points outside the pool */
  WF_ERR_CALL_ORDER = 5,    /* call not allowed in the pool's current state */
  WF_ERR_CUDA = 6,          /* a CUDA runtime/driver call failed */
  WF_ERR_UNSUPPORTED = 7,   /* valid but not implemented shape/dtype combo */
  WF_ERR_TIMEOUT = 8        /* a bounded device-side wait ran out (kernel gave up) */
} wf_status;

/* Storage / compute type of a pool.
 * BF16: pages, q, k, v, q_rot and out are bf16; tensor-core attention.
 * F32:  all fp32; CUDA-core attention.
 * FP8_E4M3: the K/V payload plus scale factors of Appendix Table 8 ("FP8 K/V
 *   communication"), with 8-bit attention operands as in the Sage backends of
 *   Tables 4-6. Pages hold E4M3 codes (1 byte per element, round to nearest
 *   even); every (page, K|V, head) block of 128 x d codes has a power-of-two
 *   fp32 scale 2^e, e the smallest integer with amax * 2^-e <= 448 (clamped
 *   below at -100). wf_publish_kv reads bf16 q, k, v, rotates q and k in fp32
 *   (each product and sum rounded once), and writes q_rot as E4M3 codes
 *   [S+1][C][heads][d] with one scale per (slot, 128-row tile, head) kept in
 *   the pool. wf_round_attention reads those codes and scales and writes bf16
 *   out. Needs head_dim 128 and page_tokens 128. */
enum { WF_DTYPE_BF16 = 0, WF_DTYPE_F32 = 1, WF_DTYPE_FP8_E4M3 = 2 };
enum { WF_ROPE_OFF = 0, WF_ROPE_3D = 1 };
/* Which (query slot, key slot) pairs are visible.
 * WF: M_WF(s, j) = 1[j >= s] (Method section of the hyper.ai summary), plus
 *     anchor and history; masked pairs are never computed.
 * RF: every live slot sees every other (bidirectional live window), the
 *     Rolling Forcing graph that the pages contrast WF with ("Contexto",
 *     e-cogni article); also sees anchor and history. */
enum { WF_MASK_WF = 0, WF_MASK_RF = 1 };

/* Limits of this implementation. */
#define WF_MAX_STAGES 16
#define WF_MAX_HISTORY 64

typedef struct {
  int32_t num_stages;      /* S, 1..WF_MAX_STAGES; slots 0..S-1 plus the store */
  int32_t chunk_tokens;    /* C, tokens per chunk (full attention inside) */
  int32_t num_heads;       /* attention heads (K/V heads = Q heads) */
  int32_t head_dim;        /* d; bf16 attention: 128; fp32: multiple of 4, <= 128 */
  int32_t anchor_chunks;   /* 0 or 1: keep chunk 0 as the anchor */
  int32_t history_chunks;  /* H, bounded clean history window, 0..WF_MAX_HISTORY */
  int32_t page_tokens;     /* P, tokens per page; bf16 attention: 128 */
  int32_t num_layers;      /* layers sharing the page table (one pool region each) */
  int32_t dtype;           /* WF_DTYPE_BF16, WF_DTYPE_F32 or WF_DTYPE_FP8_E4M3 */
  int32_t rope;            /* WF_ROPE_OFF or WF_ROPE_3D */
  int32_t frames_per_chunk;/* F: latent frames per chunk (3D rotary only) */
  int32_t grid_h, grid_w;  /* patch grid per frame; C == F * grid_h * grid_w */
  int32_t rope_split[3];   /* rotary band widths over t, h, w; even, sum = d */
  float rope_base;         /* rotary base (10000) */
  int32_t max_rounds;      /* rounds the pool may run (sizes the t table) */
  int32_t num_pages;       /* physical pages per layer; 0 = the minimum */
  int32_t mask_mode;       /* WF_MASK_WF (default, 0) or WF_MASK_RF */
} wf_pool_config;

typedef struct wf_pool wf_pool;

/* Where things live inside the caller's pool memory (for tests and tools). */
typedef struct {
  int64_t num_pages;        /* physical pages per layer */
  int32_t pages_per_chunk;  /* ceil(C / P) */
  int32_t max_positions;    /* A + H + S + 1 */
  size_t status_offset;     /* int32 sticky status word */
  size_t tags_offset;       /* int32 [num_layers][num_pages] ready tags */
  size_t pages_offset;      /* [num_layers][num_pages][2 (K,V)][heads][P][d] */
  size_t page_bytes;        /* bytes of one (layer, page): 2 * heads * P * d * elt */
  size_t total_bytes;       /* == wf_kv_pool_bytes */
  size_t kv_scale_offset;   /* FP8: fp32 [num_layers][num_pages][2 (K,V)][heads]; else 0 */
  size_t q_scale_offset;    /* FP8: fp32 [num_layers][S+1][pages_per_chunk][heads]
                               (scale of q_rot rows [128 t, 128 t + 128)); else 0 */
} wf_pool_geometry;

/* Bytes of device memory a pool with this config needs (the caller allocates
 * them, 256-byte aligned, and keeps them alive until wf_pool_destroy).
 * Returns WF_ERR_INVALID_ARG / WF_ERR_OUT_OF_PAGES / WF_ERR_UNSUPPORTED for a
 * config that wf_kv_pool_create would reject. */
wf_status wf_kv_pool_bytes(const wf_pool_config *cfg, size_t *bytes);

/* Create the paged K/V pool: page table, free list, ordered slots, ready tags
 * (paged delivery into ordered attention slots, Method section; the bounded
 * history window of "Como funciona").
 *   dev_mem, bytes : caller-owned device memory of wf_kv_pool_bytes bytes,
 *                    256-byte aligned; NULL/0 creates a host-only pool that
 *                    runs the bookkeeping (advance, layout queries) with no
 *                    device work, for dry runs and CPU tests.
 *   page_order     : host array of num_pages distinct ids in [0, num_pages)
 *                    giving the initial free-list order, or NULL (identity).
 *   stream         : stream for the set-up writes; the call synchronises it.
 * On success *out owns the host state; the pool starts at round 0. */
wf_status wf_kv_pool_create(const wf_pool_config *cfg, void *dev_mem, size_t bytes,
                            const int32_t *page_order, wf_stream_t stream, wf_pool **out);

/* Publish one layer's K/V for every live slot of the current round (early
 * publication after QKV + RoPE, Method section): applies the 3D rotary
 * embedding to q and k (fp32 math with each product and sum rounded once,
 * (cos, sin) from the host's float64 cos and sin rounded to fp32; then one
 * rounding to the pool's dtype), writes q_rot, scatters
 * rotated K and V into the slots' pages (rows past C in a chunk's last page
 * are zeroed) and stamps each written page's ready tag.
 *   q, k, v : inputs, [S+1][C][heads][d]; rows of slots that are not live in
 *             this round are not read.
 *   q_rot   : output, same layout; only live slots' rows are written.
 * FP8_E4M3 pools: q, k, v are bf16; q_rot receives E4M3 codes (1 byte per
 * element) and the pool records the block scales of q_rot, K and V.
 * Pointers must be 16-byte aligned; q_rot must not alias q, k or v. */
wf_status wf_publish_kv(wf_pool *pool, int32_t layer, const void *q, const void *k,
                        const void *v, void *q_rot, wf_stream_t stream);

/* Round attention for one layer (M_WF mask, full attention inside chunks):
 * for every live query slot s and head h,
 *     out[s] = softmax(q_rot[s] K_s^T / sqrt(d)) V_s
 * where K_s, V_s are the keys slot s may read: under WF_MASK_WF the
 * ordered-context prefix (anchor, history, store, slots S-1 .. s), under
 * WF_MASK_RF the whole context. Before reading, the kernel checks
 * every page's ready tag against the round's expected tag; any mismatch sets
 * WF_ERR_NOT_READY in the status word and the launch writes no output.
 *   q_rot : [S+1][C][heads][d] rotated queries (as written by wf_publish_kv);
 *   out   : [S+1][C][heads][d]; rows of non-live slots are left untouched.
 * bf16 pools need head_dim == 128 and page_tokens == 128 (tensor-core path);
 * fp32 pools run a CUDA-core path. FP8_E4M3 pools read q_rot codes as written
 * by wf_publish_kv in this round for this layer (their scales live in the
 * pool), run E4M3 tensor-core MMAs (P rounded to E4M3 too) and write bf16 out.
 * Pointers must be 16-byte aligned. */
wf_status wf_round_attention(wf_pool *pool, int32_t layer, const void *q_rot, void *out,
                             wf_stream_t stream);

/* Wave Parallelism (Method section, Figure 3c; thelatestinai listing, Table
 * 10): one GPU per stage, each running one query slot per round, with one-way
 * K/V delivery into the pages of the stages that read them and a ready signal.
 * Every rank keeps a full pool created with the same config and page_order and
 * advanced through the same rounds, so the page tables (and the physical ids
 * of every slot's pages) are the same on all ranks. A round on rank r, owner
 * of slot r (the store rank owns slot S):
 *   wf_publish_kv_slot(r) -> wf_deliver_kv(r) to each reader ->
 *   wf_round_attention_slot(r) once the deliveries into this pool have landed
 *   (the caller orders them, e.g. with a barrier or an IPC event);
 * readers of slot j are the live slots s < j under WF_MASK_WF, every live slot
 * under WF_MASK_RF, and every rank for the store (its chunk becomes anchor or
 * history for all later rounds). wave_plan() in the Python binding lists them.
 *
 * Ordering across rounds is the caller's too: a delivery of round k + 1
 * overwrites the receiver's pages of the same slot (and the recycled store
 * pages), so a sender must not deliver round k + 1 into a receiver until that
 * receiver's round-k wf_round_attention_slot has finished reading them (for
 * example an event the receiver records after its attention, or a barrier
 * between rounds). The readiness check reads the tags once, when the
 * attention kernel starts, so it cannot catch an overwrite that lands while
 * the kernel runs; the output would then be silently wrong.
 *
 * wf_publish_kv_slot: wf_publish_kv restricted to one live slot: reads only
 * that slot's rows of q, k, v ([S+1][C][heads][d] buffers), writes its q_rot
 * rows, its pages and their ready tags. WF_ERR_CALL_ORDER if the slot is not
 * live in this round. */
wf_status wf_publish_kv_slot(wf_pool *pool, int32_t layer, int32_t slot, const void *q,
                             const void *k, const void *v, void *q_rot, wf_stream_t stream);

/* wf_round_attention restricted to one live query slot: writes only that
 * slot's rows of out, and checks the ready tags of only the context prefix the
 * slot reads (under WF_MASK_RF, the whole context). WF_ERR_CALL_ORDER if the
 * slot is not live in this round. */
wf_status wf_round_attention_slot(wf_pool *pool, int32_t layer, int32_t slot, const void *q_rot,
                                  void *out, wf_stream_t stream);

/* Deliver one live slot's published K/V pages of one layer into a receiver's
 * pool: every (page, K|V, head) tile of the slot's chunk (and, for FP8_E4M3
 * pools, its block scale) is copied to the same physical page of the
 * receiver, then the receiver's ready tags of those pages are set to the
 * slot's tag of this round.
 *   dst_pool_mem   : the receiver pool's device buffer (as passed to its
 *                    wf_kv_pool_create), 256-byte aligned and addressable from
 *                    the current device: a buffer on this device, a peer
 *                    device's buffer with peer access enabled, or a buffer of
 *                    another process opened with wf_ipc_open_mem (the copy
 *                    stores go over NVLink when it is on another GPU).
 *   dst_pool_bytes : the receiver's pool size; WF_ERR_INVALID_ARG unless it
 *                    equals this pool's wf_kv_pool_bytes.
 * The receiver must have this pool's config, page order and round. Every pool
 * stores a 64-bit signature of its config and page order in its memory at
 * creation; the kernels compare the receiver's with this pool's and, if they
 * differ, record WF_ERR_INVALID_ARG in this pool's status word and write
 * nothing. Each copy CTA then checks its own page in this pool: an id out of
 * range records WF_ERR_BAD_PAGE, a ready tag from another round
 * WF_ERR_NOT_READY (the slot was not published in this round), and that
 * page's tiles are not copied. The tag kernel, in stream order after the
 * copy, checks every page of the slot the same way and stamps the receiver's
 * tags only if all pass, so the receiver never sees a ready tag for a slot
 * that was not wholly published and copied; a slot not published at all
 * leaves the receiver untouched. WF_ERR_CALL_ORDER if the slot is not live;
 * WF_ERR_INVALID_ARG for a NULL, misaligned or self receiver buffer. */
wf_status wf_deliver_kv(const wf_pool *pool, int32_t layer, int32_t slot, void *dst_pool_mem,
                        size_t dst_pool_bytes, wf_stream_t stream);

/* Inter-process access to a pool buffer, for Wave Parallelism with one
 * process per stage GPU (Method section and Figure 3c: each stage writes its
 * K/V straight into the ordered slots of the stages that read it).
 *
 * wf_ipc_get_mem_handle: export the device allocation that holds dev_ptr
 * (a receiver's pool buffer, on the current device) as an opaque handle that
 * another process can open, plus dev_ptr's byte offset inside that
 * allocation. WF_ERR_INVALID_ARG if dev_ptr is not device memory of this
 * process, WF_ERR_CUDA if CUDA refuses the export.
 * wf_ipc_open_mem: map an exported allocation into this process (on the
 * current device; peer access to the owner's device is enabled on demand) and
 * return the pointer at `offset` inside it, to pass to wf_deliver_kv as
 * dst_pool_mem. WF_ERR_CUDA if the handle cannot be opened (a handle cannot
 * be opened by the process that exported it).
 * wf_ipc_close_mem: unmap a pointer returned by wf_ipc_open_mem (same
 * offset). The exporting process keeps ownership of the memory and must keep
 * it allocated until every importer has closed it. None of these calls
 * allocates device memory. */
typedef struct { unsigned char bytes[64]; } wf_ipc_handle;
wf_status wf_ipc_get_mem_handle(const void *dev_ptr, wf_ipc_handle *handle, size_t *offset);
wf_status wf_ipc_open_mem(const wf_ipc_handle *handle, size_t offset, void **dev_ptr);
wf_status wf_ipc_close_mem(void *dev_ptr, size_t offset);

/* Fused QKV projection + publication for one layer (Method section: the local
 * QKV projection runs without waiting for remote K/V, and K/V are published
 * right after the projection and RoPE, written straight into the ordered
 * slots). For every live slot s and token n:
 *     [q | k | v][s][n] = x[s][n] . w_qkv^T        (fp32 accumulation)
 * then q and k are rotated by the 3D rotary embedding exactly as in
 * wf_publish_kv, and the results are written as wf_publish_kv writes them:
 * q_rot rows, K and V page rows (rows past C zeroed), ready tags.
 *   x     : [S+1][C][hidden] bf16 activations, hidden = num_heads * head_dim;
 *           rows of slots that are not live are not read.
 *   w_qkv : [3 * hidden][hidden] bf16, the q, k, v output features stacked
 *           (row f holds the weights of output feature f).
 *   q_rot : [S+1][C][heads][d] bf16; only live slots' rows are written.
 * bf16 pools only, with head_dim 128, page_tokens 128 and hidden a multiple of
 * 256 (WF_ERR_UNSUPPORTED otherwise, FP8 pools included). Pointers must be 16-byte aligned. */
wf_status wf_project_publish(wf_pool *pool, int32_t layer, const void *x, const void *w_qkv,
                             void *q_rot, wf_stream_t stream);

/* Move the pool to the next round (k -> k + 1, Table 3): the store's chunk
 * becomes the anchor (chunk 0, when kept) or the newest history chunk; history
 * beyond H returns its pages to the free list; the next store takes pages
 * from the free list; the device page table is rewritten on the stream.
 * Returns WF_ERR_CALL_ORDER when max_rounds would be exceeded. */
wf_status wf_advance_round(wf_pool *pool, wf_stream_t stream);

/* Synchronise the stream, then return and clear the pool's sticky device
 * status (WF_OK if no kernel recorded an error). */
wf_status wf_pool_check_status(wf_pool *pool, wf_stream_t stream);

/* Free the host state. Does not touch dev_mem (the caller owns it). */
wf_status wf_pool_destroy(wf_pool *pool);

const char *wf_status_string(wf_status status);

/* Current round k, or -1 for a NULL pool. */
int64_t wf_pool_round(const wf_pool *pool);

/* Region offsets inside dev_mem. */
wf_status wf_pool_get_geometry(const wf_pool *pool, wf_pool_geometry *geom);

/* The current round's ordered context, from the host mirror of the page table.
 * Writes *n_positions and, for each position p < cap: kinds[p] (0 anchor,
 * 1 history, 2 store, 3 denoising slot), chunks[p], slots[p] (-1 for anchor
 * and history), tags[p] (expected ready tag) and
 * pages[p * pages_per_chunk + j] (physical page of the chunk's j-th page).
 * Any output pointer may be NULL. */
wf_status wf_pool_get_layout(const wf_pool *pool, int32_t *n_positions, int32_t *kinds,
                             int32_t *chunks, int32_t *slots, int32_t *tags,
                             int32_t *pages, int32_t cap);

/* Fault-injection hook for tests: overwrite one entry of the DEVICE page table
 * (position, j) with `physical` (which may be out of range), without changing
 * the host mirror. The next publish/attention sees it; kernels bounds-check
 * page ids and record WF_ERR_BAD_PAGE instead of accessing memory. */
wf_status wf_pool_debug_poke_page(wf_pool *pool, int32_t position, int32_t j,
                                  int32_t physical, wf_stream_t stream);

/* Test hook for the bounded waits of the tensor-core attention kernel
 * (readiness is checked just before attention, Method section; a kernel whose
 * wait for a copy or an MMA runs out gives up instead of spinning): the NEXT
 * wf_round_attention / wf_round_attention_slot call on this pool issues no
 * load of K for key tile `key_tile` of any query tile (key tiles count the
 * 128-token pages of the slot's context in order, from 0), so the waits for it
 * can only run out, and every bounded wait of that launch gives up after
 * `wait_limit_cycles` SM clock cycles (1000 .. 2e9; the default is 2e9, about
 * a second). The waits that drain a CTA's own in-flight copies and MMAs keep
 * their fixed, longer bound. A CTA that gives up records WF_ERR_TIMEOUT,
 * writes none of its output rows, and frees its tensor memory; CTAs whose
 * context is shorter than key_tile + 1 tiles run normally. Later launches are
 * unaffected. bf16 and FP8_E4M3 pools only (WF_ERR_UNSUPPORTED for fp32). */
wf_status wf_pool_debug_stall_next_attention(wf_pool *pool, int32_t key_tile,
                                             int64_t wait_limit_cycles);

#ifdef __cplusplus
}
#endif
#endif /* WF_H_ */
