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
  CUtensorMap kv[KV_MAX_STREAMS];
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
  int H;
  float scale_log2;    // log2(e) / sqrt(D)
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
  int T, NS, page_size, Np, max_pages;
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

// Attention CTAs that fit on one SM for this head_dim (used by the planner).
int attention_ctas_per_sm(int D);
// Whether the attention kernel computes <= 16-row tail tiles inside the
// preceding unit for this head_dim (used by the planner).
bool attention_tail_ok(int D);

}  // namespace pkv
