/*
 * paged_kv_cache_frame_b200 -- C-ABI for per-frame paged-KV prefill attention
 * on NVIDIA B200 (sm_100a).
 *
 * The operation, from the LingBot-Map pages:
 *   [P1] "How the Paged KV Cache Attention Mechanism Enables Long Sequence
 *        Inference in LingBot-Map"
 *   [P2] "KV Cache Mechanism in LingBot-Map for Streaming Inference: A Deep Dive"
 *   [P3] "FlashInfer Paged KV Cache Performance Benefits in LingBot-Map:
 *        Technical Implementation and Benchmarks"
 *   [P4] "How LingBot-Map Achieves ~20 FPS Inference with Its KV Cache"
 *
 * Each video frame brings T = NS + P tokens (NS special tokens: camera,
 * register, scale; P patch tokens). Per transformer block the frame's K/V are
 * appended to a paged pool and the frame's T queries attend, with no mask,
 * over every visible token: the S scale frames, the latest W window frames
 * (the current one included) and the whole append-only special stream.
 *
 * Conventions for every call:
 *   - Return value: KV_OK (0) or a negative KV_ERR_* code. Nothing aborts;
 *     kv_last_error() gives a one-line detail of the last failure on the
 *     calling thread.
 *   - Device buffers (pool, q, k, v, out, workspace) belong to the caller. The
 *     library never allocates device memory. Host state (kv_cache_t,
 *     kv_plan_t) belongs to the library and is released by kv_destroy /
 *     kv_plan_free.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Device work is
 *     enqueued asynchronously on it; errors raised later inside a kernel are
 *     reported by kv_check_device.
 *   - Token order inside a frame, for q, k, v and out alike: tokens 0..NS-1
 *     are the special tokens, NS..T-1 the patch tokens. Tensors [T, H, D] are
 *     contiguous, 16-byte aligned, in the cache's dtype.
 *   - Frame step rule. The first kv_append_frame of a frame step (any block)
 *     advances the page state: it takes a patch page and NS special slots for
 *     the new frame. Every other block must then be appended exactly once in
 *     the same step before its kv_run. A step is complete when all blocks are
 *     appended; the next append opens a new step. A pending (deferred) frame
 *     must be committed or rolled back before the next step.
 *   - Not thread-safe: one host thread drives a cache and its plans.
 */
#ifndef PAGED_KV_CACHE_FRAME_B200_KV_H
#define PAGED_KV_CACHE_FRAME_B200_KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  KV_OK = 0,
  KV_ERR_ARG = -1,          /* null/out-of-range argument, misaligned pointer, bad shape */
  KV_ERR_CAPACITY = -2,     /* pool too small, no free patch page, special stream full,
                               workspace too small, too many streams in one plan */
  KV_ERR_ORDER = -3,        /* call out of order (frame step rule above) */
  KV_ERR_NO_PENDING = -4,   /* commit or rollback without a deferred frame */
  KV_ERR_NOT_APPENDED = -5, /* kv_run for a block not appended in the current step */
  KV_ERR_EMPTY = -6,        /* kv_plan before the first frame, or with no visible token */
  KV_ERR_CUDA = -7,         /* a CUDA runtime or driver call failed */
  KV_ERR_DEVICE_CHECK = -8, /* a kernel set the device error word (bounded wait expired
                               or an index check failed) */
  KV_ERR_UNSUPPORTED = -9,  /* no kernel for this head_dim/dtype (head_dim must be 64 or 128) */
  KV_ERR_STALE_PLAN = -10   /* the cache state changed after the plan was built */
};

enum { KV_BF16 = 0, KV_FP16 = 1 };

/* Upper bound on the streams (requests) batched in one plan. */
#define KV_MAX_STREAMS 32

typedef struct kv_cache kv_cache_t; /* one video stream's cache, all blocks */
typedef struct kv_plan kv_plan_t;   /* one frame step's execution plan */

/* get_cache_stats ([P3] "Monitoring Cache Statistics").
 *   frame_count    frames appended since init/reset and not rolled back
 *                  (a pending frame counts)
 *   scale_pages    resident scale-frame patch pages (<= scale_frames)
 *   live_pages     resident window patch pages, a pending frame's page included
 *   free_pages     patch pages on the free list
 *   special_tokens tokens in the special stream (NS per frame_count)
 * scale_pages + live_pages + free_pages == patch pages, always. */
typedef struct kv_stats {
  int frame_count;
  int scale_pages;
  int live_pages;
  int free_pages;
  int special_tokens;
} kv_stats;

/* A cache's configuration as kv_init fixed it (patch_pages resolved). */
typedef struct kv_config {
  int max_pages, page_size, num_heads, head_dim, scale_frames, window, num_blocks, num_special, dtype;
  int patch_pages;          /* patch pages [0, patch_pages) (shared in a group) */
  int special_base;         /* this stream's special pages [special_base, special_base + special_pages) */
  int special_pages;
  int tokens_per_frame;     /* T = page_size + num_special: rows of k, v, q and out */
  int cross_frame_special;  /* 1 while the special tokens of evicted frames stay visible */
  int camera_only;          /* 1 while attention sees only the camera tokens */
} kv_config;

/* Execution-plan summary, for tests and benchmarks. */
typedef struct kv_plan_stats {
  int n_streams;      /* requests in the plan */
  int n_ctas;         /* CTAs of the attention launch (work units) */
  int n_split_units;  /* (stream, head, q-tile) units split across CTAs */
  int n_kv_tiles;     /* 128-token K/V tiles summed over streams */
  int tiles_per_cta;  /* largest number of K/V tiles one CTA processes */
  long long visible_tokens; /* visible tokens summed over streams */
  int fused_merge;    /* 1: split units are merged by their own CTAs (the launch
                         has at most one CTA per SM and no unit more than 32
                         chunks; a CTA whose partners do not run alongside it,
                         e.g. because another launch holds SMs, leaves its share
                         to the last one), 0: by a merge launch */
  int run_launches;   /* kernel launches of one kv_run / kv_run_append (1, or 2 with
                         a merge launch) */
  int upload_launches; /* kernel launches kv_plan made to upload the tables */
} kv_plan_stats;

/* kv_init -- create one stream's cache ([P1] "Implementation Example": the
 * FlashInferKVCacheManager constructor; [P2] "Configuration Parameters").
 *   max_pages     pages per block pool: patch pages + special pages
 *   page_size     tokens per page; must equal the patch tokens per frame
 *                 ([P1] "Patch Stream (Recyclable)": one page per frame)
 *   num_heads, head_dim   H, D of K/V/Q (D = 64 or 128 for kv_run)
 *   scale_frames  S: the first S committed frames stay resident for good
 *   window        W: at most W non-scale frames stay resident
 *   num_blocks    transformer blocks (one pool each)
 *   num_special   NS special tokens per frame (6 on the pages), >= 0
 *   dtype         KV_BF16 or KV_FP16
 *   patch_pages   size of the recyclable patch pool; 0 = S + W + 1 (append takes
 *                 a page before eviction returns one). Pages [0, patch_pages) are
 *                 patch pages, [patch_pages, max_pages) special pages.
 * Errors: KV_ERR_ARG (bad value), KV_ERR_CAPACITY (max_pages < patch_pages + 1
 * when num_special > 0). No CUDA call is made. */
int kv_init(kv_cache_t** out, int max_pages, int page_size, int num_heads, int head_dim,
            int scale_frames, int window, int num_blocks, int num_special, int dtype,
            int patch_pages);

/* kv_init_group -- create n_streams caches that share one pool per block
 * ([P3] "Constant Memory with Two-Stream Paging": memory is bounded by
 * max_patch_pages + max_special_pages, here for all the streams together).
 * The patch pages [0, patch_pages) and their LIFO free list are common to the
 * streams: a stream takes a page when it appends a frame and returns it when
 * it evicts, rolls back or resets, so pages left by one stream serve another.
 * Stream i owns the special pages [patch_pages + i * special_pages,
 * patch_pages + (i + 1) * special_pages) for its special stream.
 *   out            array of n_streams handles (1 <= n_streams <= KV_MAX_STREAMS),
 *                  each released with kv_destroy
 *   patch_pages    0 = n_streams * (scale_frames + window + 1), enough for every
 *                  stream at once; fewer pages give KV_ERR_CAPACITY on an append
 *                  that finds the common list empty
 *   special_pages  per stream; 0 = (max_pages - patch_pages) / n_streams
 * Other arguments as kv_init. kv_bind_pool on any of the caches binds the
 * block's pool for all of them (and zero-fills it: bind before the first
 * append). kv_reset of one stream returns its scale pages (frame order), then
 * its window pages (oldest first), then a pending page to the common list.
 * Errors: KV_ERR_ARG, KV_ERR_CAPACITY (max_pages < patch_pages + n_streams *
 * special_pages). No CUDA call is made. */
int kv_init_group(kv_cache_t** out, int n_streams, int max_pages, int page_size, int num_heads, int head_dim,
                  int scale_frames, int window, int num_blocks, int num_special, int dtype, int patch_pages,
                  int special_pages);

/* kv_destroy -- free the host state. Pools are not touched. NULL is ignored. */
void kv_destroy(kv_cache_t* c);

/* kv_reset -- clean_kv_cache ([P2] "Manual Cache Control"): back to the state
 * kv_init left, keeping the bound pools (their contents are not cleared). */
int kv_reset(kv_cache_t* c);

/* kv_pool_bytes -- bytes of one block's pool
 * [max_pages, 2, page_size, H, D] ([P1] "Physical Memory Layout"). Dimension 1
 * is K (0) / V (1); the two streams are told apart by page-id range. */
size_t kv_pool_bytes(const kv_cache_t* c);

/* kv_bind_pool -- lend block `block` a device pool of kv_pool_bytes() bytes,
 * 16-byte aligned, owned by the caller and kept alive while the cache uses it.
 * The pool is zero-filled on `stream` (so that masked rows a kernel reads
 * past a page's end are finite) and a TMA descriptor for it is built on the
 * host. Errors: KV_ERR_ARG, KV_ERR_CUDA. */
int kv_bind_pool(kv_cache_t* c, int block, void* pool, void* stream);

/* kv_append_frame -- append_frame(block_idx, k, v) ([P1] "Appending New
 * Frames"). k, v: device [T, H, D]. Special tokens 0..NS-1 go to the special
 * stream at its current length (packed continuously, possibly across two
 * pages); patch tokens NS..T-1 fill the frame's patch page, taken from the
 * free list by the first append of the step. Launches one scatter kernel
 * with 16-byte stores on `stream`.
 * If k and v are both NULL only the page state advances and the block is
 * marked appended; nothing is written (for callers that fill the pool
 * themselves, and host-side tests).
 * Errors: KV_ERR_ARG, KV_ERR_ORDER (block appended twice in a step, or a
 * pending frame from an earlier step), KV_ERR_CAPACITY (no free patch page or
 * special stream full), KV_ERR_CUDA (the scatter launch failed). On every
 * error the page state is left unchanged: the scatter is launched before the
 * state advances, so after a failed launch the same call can be retried. */
int kv_append_frame(kv_cache_t* c, int block, const void* k, const void* v, void* stream);

/* kv_evict_frames -- evict_frames ([P1] "Evicting Stale Frames"; [P2]
 * "Sliding-Window Eviction Strategy"): while more than W window pages are
 * resident, push the oldest on the free list. Scale and special pages are
 * never touched. No-op while eviction is deferred. Idempotent. Host only. */
int kv_evict_frames(kv_cache_t* c);

/* kv_defer_eviction -- _set_defer_eviction ([P2] "Flow-Based Keyframe
 * Selection"): with on != 0 the next appended frame stays pending (visible,
 * not committed) and eviction is suspended until kv_commit_frame or
 * kv_rollback_last_frame. Turning it off while a frame is pending is
 * KV_ERR_ORDER. */
int kv_defer_eviction(kv_cache_t* c, int on);

/* kv_commit_frame -- execute_deferred_eviction ([P2] "Flow-Based Keyframe
 * Selection"): the pending frame becomes a normal frame, eviction runs, defer
 * is switched off. Errors: KV_ERR_NO_PENDING; KV_ERR_ORDER if its step has
 * not appended every block. */
int kv_commit_frame(kv_cache_t* c);

/* kv_rollback_last_frame -- rollback_last_frame ([P2] "Flow-Based Keyframe
 * Selection"; [P4] "Deferred Eviction and Rollback Mechanism"): discard the
 * pending frame: its patch page goes back on the free list, the special stream
 * shrinks by NS, defer is switched off and the step is closed. The page state
 * then equals the state before the frame's append. Pool bytes are not
 * touched. Errors: KV_ERR_NO_PENDING. */
int kv_rollback_last_frame(kv_cache_t* c);

/* kv_get_stats -- get_cache_stats ([P3] "Monitoring Cache Statistics"). */
int kv_get_stats(const kv_cache_t* c, kv_stats* out);

/* kv_get_config -- the cache's configuration, for callers that size q, k, v
 * and out ([T, H, D] per stream) from a cache handle. Errors: KV_ERR_ARG. */
int kv_get_config(const kv_cache_t* c, kv_config* out);

/* kv_get_free_list -- the free list bottom to top (the next page handed out is
 * ids[n-1]). Writes at most `cap` ids; *n gets the full length. */
int kv_get_free_list(const kv_cache_t* c, int* ids, int cap, int* n);

/* kv_workspace_bytes -- device workspace kv_plan needs for these caches
 * (plan tables, split-KV partials, the device error word). 0 on bad input. */
size_t kv_workspace_bytes(kv_cache_t* const* caches, int n_streams);

/* kv_plan -- plan() once per frame step ([P1] "FlashInfer Kernel Execution";
 * [P3] "Visible Page Table Attention"). For each cache, build the visible page
 * table ([P1] "Building the Visible Page Table"): scale pages in frame order,
 * window pages oldest to newest, the pending page, then the special pages,
 * and paged_kv_last_page_len = tokens written to the table's final page
 * (1..page_size; [P1] "Frequently Asked Questions": the exact count of valid
 * tokens in the final page). The final page is the special stream's last page
 * unless cross-frame special retention is off and hides all of its tokens;
 * the tokens that retention off hides inside a listed page are not expressible
 * in (indices, last_page_len) and are left out of the K/V tiles.
 * Split the 128-token K/V tiles over CTAs (tiles_per_split = 0: automatic
 * schedule for the SM count; > 0: at most that many tiles per CTA, which
 * forces split-KV for tests) and copy the tables into `workspace` on
 * `stream` (kernel launches whose parameters carry the tables: asynchronous,
 * no host staging buffer). Stream i's queries are rows
 * [sum_{j<i} T, sum_{j<=i} T) of kv_run's q.
 * workspace == NULL builds a host-only plan (kv_get_page_table works, kv_run
 * does not). All caches must share page_size, H, D, NS, num_blocks and dtype.
 * The plan stays valid, for every block, until a cache's page state changes.
 * Errors: KV_ERR_ARG, KV_ERR_EMPTY (a cache with no frame, or none of whose
 * tokens is visible: scale_frames = window = 0 with retention off), KV_ERR_CAPACITY
 * (workspace smaller than kv_workspace_bytes, > KV_MAX_STREAMS), KV_ERR_CUDA. */
int kv_plan(kv_plan_t** out, kv_cache_t* const* caches, int n_streams, int tiles_per_split,
            void* workspace, size_t workspace_bytes, void* stream);

/* kv_run -- run() for one block ([P1] "FlashInfer Kernel Execution"; [P3]
 * "Custom CUDA Kernel Implementation"): for every stream r, head h and query
 * row i of the frame,
 *     out[i, h] = sum_j softmax_j(q[i, h] . k_j[h] / sqrt(D)) v_j[h]
 * over the visible tokens j of block `block`'s pool, no mask. q, out: device
 * [sum T, H, D] in the cache dtype; fp32 accumulation; out rounded to nearest
 * even. Launches the attention kernel and, when the plan splits a unit and
 * its CTAs do not merge it themselves (kv_plan_stats.fused_merge), the
 * split-KV merge kernel on `stream`. Plans may run on several streams at
 * once.
 * Errors: KV_ERR_ARG, KV_ERR_STALE_PLAN, KV_ERR_NOT_APPENDED, KV_ERR_CUDA. */
int kv_run(const kv_plan_t* plan, int block, const void* q, void* out, void* stream);

/* kv_begin_frame -- open a frame step without appending a block: the new
 * frame takes its patch page and NS special slots now, as the first
 * kv_append_frame of a step would ([P1] "Appending New Frames"). Then evict,
 * plan, and append every block, each with kv_append_frame or kv_run_append.
 * Errors: KV_ERR_ORDER (the open step still has blocks to append, or a
 * pending frame of an earlier step), KV_ERR_CAPACITY (no free patch page or
 * special stream full); the state is unchanged on error. Host only. */
int kv_begin_frame(kv_cache_t* c);

/* kv_run_append -- append_frame for block `block` followed by run() for it,
 * in one kernel launch ([P1] "Appending New Frames", "FlashInfer Kernel
 * Execution"). k, v, q, out: device [sum T, H, D] in the cache dtype, the
 * streams' rows in plan order (as q for kv_run). The launch copies every
 * stream's k, v rows into the block's pool (special tokens to the special
 * stream, patch tokens to the frame's page, exactly as kv_append_frame does)
 * and computes out as kv_run does, reading the frame's own K/V from k and v.
 * The plan must have been built after the step was opened (kv_begin_frame,
 * or a kv_append_frame of another block), and `block` must not be appended
 * yet in that step; it counts as appended once the launch has been made.
 * Errors: KV_ERR_ARG, KV_ERR_STALE_PLAN, KV_ERR_ORDER (no open step for the
 * plan, or the block already appended), KV_ERR_CUDA. If the attention launch
 * fails nothing was appended; if a merge launch after it fails, the block is
 * appended and out is incomplete. */
int kv_run_append(const kv_plan_t* plan, int block, const void* k, const void* v, const void* q,
                  void* out, void* stream);

/* kv_plan_free -- release a plan's host state. NULL is ignored. */
void kv_plan_free(kv_plan_t* plan);

/* kv_get_page_table -- host copy of stream `stream_idx`'s visible page table:
 * up to `cap` page ids into `indices`, the full count into *n, and
 * paged_kv_last_page_len into *last_page_len. */
int kv_get_page_table(const kv_plan_t* plan, int stream_idx, int* indices, int cap, int* n,
                      int* last_page_len);

/* kv_get_kv_tiles -- host copy of stream `stream_idx`'s K/V tile list: the
 * visible rows of earlier frames in visible-table order, then those of the
 * open step's frame. Tile t reads pool K rows [row[t], row[t] + 128) of the
 * [max_pages * 2 * page_size]-row space (its V rows start page_size later);
 * columns [lo[t], hi[t]) of the tile are visible tokens, the rest are masked.
 * krow (may be NULL): for a tile of the open step's frame, the row of the
 * frame's k/v ([T, H, D]) that column 0 stands for (column c is row
 * krow[t] + c; it can be negative, those columns being masked), which
 * kv_run_append reads instead of the pool; INT32_MIN / 2 for other tiles.
 * step (may be NULL): 1, or with camera-only NS: of [lo, hi) only columns
 * lo, lo + step, ... are visible.
 * Writes at most `cap` entries per array; *n gets the full count. */
int kv_get_kv_tiles(const kv_plan_t* plan, int stream_idx, int* row, int* lo, int* hi, int* krow, int* step,
                    int cap, int* n);

/* kv_plan_get_stats -- summary of the plan's schedule. */
int kv_plan_get_stats(const kv_plan_t* plan, kv_plan_stats* out);

/* kv_check_device -- synchronise `stream` and read the plan's device error
 * word. KV_OK, KV_ERR_DEVICE_CHECK (bit set by a kernel) or KV_ERR_CUDA. */
int kv_check_device(const kv_plan_t* plan, void* stream);

/* kv_set_cross_frame_special -- kv_cache_cross_frame_special ([P2]
 * "Configuration Parameters"): on (1, the default) keeps the special tokens of
 * evicted frames visible; off (0) leaves visible only the special tokens of
 * frames whose patch tokens are (scale, window and pending frames). Evictions
 * take the oldest window frame, so the hidden tokens form one range of the
 * special stream and the K/V tiles skip it; kv_get_page_table then lists only
 * special pages that hold a visible token. Takes effect for the next kv_plan
 * (plans made before it become stale). include_scale_frames=False of the same
 * section is scale_frames = 0 in kv_init.
 * Errors: KV_ERR_ARG (NULL cache). */
int kv_set_cross_frame_special(kv_cache_t* cache, int on);

/* kv_set_camera_only -- kv_cache_camera_only ([P2] "Configuration
 * Parameters": restrict the cache to camera tokens, excluding patches). The
 * pages list a frame's six special tokens as camera, register and scale
 * ([P2] "Special Stream (Append-Only)"); this library reads slot 0 of each
 * frame's NS special tokens (token 0 of its k/v) as the camera token. With
 * camera-only on (1), attention sees no patch token and only the camera
 * tokens among the special tokens that would otherwise be visible (every
 * frame's with cross-frame special retention on, the scale, window and
 * pending frames' with it off); kv_get_page_table lists only the special
 * pages that hold one. The page state is unchanged: patch pages are still
 * taken, written and evicted as usual. Off (0) is the default. Takes effect
 * for the next kv_plan (plans made before it become stale).
 * Errors: KV_ERR_ARG (NULL cache). */
int kv_set_camera_only(kv_cache_t* cache, int on);

/* Size of the library-owned device array that kv_run_static uses as scratch. */
#define KV_STATIC_SCRATCH_BYTES (32u << 20)

/* kv_run_static -- kv_plan + kv_run for one block in a single call that
 * allocates no memory. The paper has no counterpart: this entry point is for
 * callers that cannot call cudaMalloc, or do not want to allocate, for
 * example a host engine that runs under a fixed memory budget, or code that
 * runs while an allocator is locked. The caller still provides the caches
 * (with their bound pools), q and out as for kv_plan and kv_run. The plan's
 * tables and the split-KV partials go into one static device array of
 * KV_STATIC_SCRATCH_BYTES that the library holds instead of a caller
 * workspace.
 *
 * Arguments are as for kv_plan followed by kv_run. check != 0 also
 * synchronises `stream` and reads the kernels' error word (below).
 * `stream` must belong to the current device.
 *
 * Memory and set-up:
 *   - The array is reserved on every device where the library's code is
 *     loaded, and it stays there until the process exits.
 *   - On the first call on a device, with that device current, the library
 *     looks up the array's device address. Make that first call before any
 *     stream capture on the device.
 *   - Each call rewrites the tables at the start of the array. Partials are
 *     written before they are read.
 *   - The array's address is looked up once per device and kept. Do not call
 *     kv_run_static on a device after cudaDeviceReset (or any other
 *     destruction of its primary context) in the same process.
 *
 * Error word: the kernels of every call on a device OR their error bits into
 * one word of the array, which starts at zero when the library is loaded.
 * No call clears it except a call with check != 0, which reads it after
 * synchronising `stream`, returns KV_ERR_DEVICE_CHECK if it is non-zero and
 * then clears it. So an error raised by a call made with check == 0 is
 * reported by the next call made with check != 0.
 *
 * Concurrency: every call on a device shares the array. Two calls that
 * overlap on the GPU (for example on two streams with no ordering between
 * them) race and corrupt each other's output. Calls on one stream are
 * ordered and safe.
 *
 * Errors: as kv_plan and kv_run, plus KV_ERR_CAPACITY when the call needs
 * more than KV_STATIC_SCRATCH_BYTES of scratch. That check runs before any
 * GPU work. A 224x224 frame (16 heads, 262 tokens, 320-frame stream) needs
 * about 15 MB with automatic splitting. */
int kv_run_static(kv_cache_t* const* caches, int n_streams, int block, int tiles_per_split,
                  const void* q, void* out, int check, void* stream);

/* kv_testing_fail_launches -- for tests of the error paths only: the next n
 * kernel launches the library makes (any call, any thread) return
 * cudaErrorLaunchFailure, and so KV_ERR_CUDA, without launching anything.
 * n <= 0 cancels. No device state is touched, so no GPU fault is involved. */
void kv_testing_fail_launches(int n);

/* kv_strerror -- static text for a status code. */
const char* kv_strerror(int status);

/* kv_last_error -- detail of the last failing call on this thread ("" if none). */
const char* kv_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* PAGED_KV_CACHE_FRAME_B200_KV_H */
