// Kernel launch interfaces (host side). Every launcher returns the CUDA error
// of the launch; no launcher allocates memory.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/kv.h"
#include "kv_layout.h"

namespace pkv {

// Tensor maps of one attention launch: q [sum T, H, D] and each request's pool
// [max_pages * 2 * page_size rows, H, D], both with 128-row x 64-column boxes
// and 128-byte swizzle.
struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k, v;    // the frame's own k, v [sum T, H, D] (launches that append it)
  CUtensorMap kv[KV_MAX_STREAMS];
  // the next block's pools: the first ring of each CTA's tiles is prefetched
  // into L2 for the next block's launch of the same plan (prefetch_next)
  CUtensorMap kv_next[KV_MAX_STREAMS];
};

struct AttnArgs {
  const void* q;       // [sum T, H, D] (the tail rows are read directly)
  const KvReq* reqs;
  const KvUnit* units;
  const KvTile* tiles;
  float* part_o;       // [slot][128][D] chunk-normalised partial outputs
  float* part_lse;     // [slot][128] log2-sum-exp of each partial row
  void* out;           // [sum T, H, D]
  uint32_t* err;       // device error word
  uint32_t* groups;    // [n_groups][4] arrivals, merge tickets, departures (and padding) of split groups
  int H;
  int fused_merge;     // the CTAs of a split group merge it themselves
  float scale_log2;    // log2(e) / sqrt(D)
  // Appending the frame in the same launch: the CTAs copy k, v into the
  // pools (each CTA a slice) and read the frame's own tiles from k, v.
  int fused_append;
  int n_reqs;
  int row_vecs;        // 16-byte vectors per token row: H * D * 2 / 16
  const void* k;       // [sum T, H, D]
  const void* v;
  int prefetch_next;   // kv_next holds the next block's pools
  void* pools[KV_MAX_STREAMS];   // this block's pool of each request
};

struct MergeArgs {
  const KvMergeItem* items;
  const float* part_o;
  const float* part_lse;
  void* out;
  int H;
  int n_items;
};

struct AppendArgs {
  const void* k;       // [T, H, D]
  const void* v;
  void* pool;          // [max_pages, 2, page_size, H, D]
  int T, NS, page_size, sp_base, max_pages;   // special token j: page sp_base + j / page_size
  int row_vecs;        // H * D * 2 / 16
  int patch_page;      // page of this frame's patch tokens
  int sp0;             // special-stream index of the frame's first special token
};

cudaError_t launch_attention(const AttnMaps& maps, const AttnArgs& a, int D, bool fp16, int n_units,
                             cudaStream_t stream);
cudaError_t launch_merge(const MergeArgs& m, int D, bool fp16, cudaStream_t stream);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);
// Copies `bytes` (a multiple of 4) of host data to device memory with
// parameter-payload kernel launches on `stream`.
cudaError_t upload_plan(void* dst, const void* src, size_t bytes, cudaStream_t stream);
// Launches upload_plan makes for `bytes`.
int upload_launches(size_t bytes);

// Attention CTAs that fit on one SM for this head_dim (used by the planner).
int attention_ctas_per_sm(int D);
// Largest tail tile the attention kernel computes inside the preceding unit
// for this head_dim (used by the planner; 0 = none).
int attention_max_tail_rows(int D);

}  // namespace pkv
