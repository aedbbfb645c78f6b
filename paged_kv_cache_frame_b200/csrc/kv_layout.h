// Device-side plan layout shared by the host planner and the kernels.
//
// A plan lives in the caller's workspace:
//   [header | requests | work units | merge items | K/V tiles] uploaded by
//   kv_plan in one copy, then the split-KV partials (fp32 O and log2-sum-exp)
//   written by the attention kernel and read by the merge kernel.
#pragma once
#include <stdint.h>

namespace pkv {

constexpr int kTile = 128;           // query rows per CTA tile == K/V tokens per tile
constexpr int kMaxTargetCtas = 512;  // bound on CTAs the split schedule may add

// One request (video stream) of the batch.
struct KvReq {
  int32_t q_row0;     // first row of this request in q/out [sum T, H, D]
  int32_t T;          // query rows (tokens of the frame)
  int32_t page_size;  // tokens per page of this request's pool
  int32_t n_tiles;    // K/V tiles in the visible table
  // where the open step's frame goes in the pool (for a launch that appends it)
  int32_t cur_page;   // its patch page (-1: no open step)
  int32_t cur_sp0;    // its first special token in the special stream
  int32_t sp_base;    // the stream's first special page (special token j: page sp_base + j / page_size)
  int32_t NS;         // special tokens per frame
};

// 128 consecutive pool rows of one page, starting at K row `row` of the
// [pages * 2 * page_size] row space of the pool; V rows start page_size
// later. Columns [lo, hi) of the tile are visible tokens, the rest masked.
//
// Tiles of the current frame (the frame the open step appended) also carry
// krow: column c of the tile is row krow + c of the frame's own k/v
// ([T, H, D], tokens 0..NS-1 special), so a launch that appends the frame
// itself can read those rows from k/v instead of the pool. krow can be
// negative when the box is anchored before the frame's first row (those
// columns are masked, and a TMA load fills negative rows with zeros). Other
// tiles have krow = kNotCurrent.
//
// With step > 1 only every step-th column from lo on is visible (lo, lo +
// step, ... < hi): the camera tokens of the special stream when the cache is
// camera-only.
constexpr int32_t kNotCurrent = -0x40000000;   // INT32_MIN / 2
struct KvTile {
  int32_t row;
  int16_t lo;
  int16_t hi;
  int32_t krow;
  int16_t step;
  int16_t pad;
};

// One CTA of the attention launch: one or two consecutive 128-row query
// tiles of one head, optionally followed by a short tail tile (<= 16 rows),
// against a range of K/V tiles.
struct KvUnit {
  int16_t req;
  int16_t head;
  int16_t qtile;       // first query tile: rows [qtile*128, qtile*128 + 128)
  int16_t nq;          // full query tiles in the unit (1 or 2)
  int16_t tail_rows;   // rows of the tail tile qtile + nq (0 = none)
  int16_t chunk;       // this CTA's chunk of a split group (0 if not split)
  int16_t n_chunks;    // CTAs of the group (1 = not split)
  int16_t pad;
  int32_t tile_begin;  // absolute index into the tile table
  int32_t tile_end;
  int32_t slot[3];     // per query tile (tail last): -1 = write `out`, else partial slot
  int32_t group;       // split group (index of its two counters), -1 if not split
};

constexpr int kMaxTailRows = 16;   // tail rows computed with swapped operands (N = 16)

// One (request, head, q-tile) whose K/V range was split over n CTAs.
struct KvMergeItem {
  int16_t head;
  int16_t rows;        // valid query rows of the tile (at most 128)
  int16_t n;           // partial slots slot0 .. slot0 + n - 1
  int16_t pad;
  int32_t slot0;
  int32_t row0;        // row of q/out holding the tile's first query row
};

struct KvPlanHeader {
  uint32_t error;      // device error word (bit 0: bounded wait expired; bit 1: index check)
  int32_t n_reqs;
  int32_t n_units;
  int32_t n_merge;
  int32_t n_tiles;
  int32_t off_reqs, off_units, off_merge, off_tiles;  // byte offsets from the header
  int32_t upload_bytes;
  int64_t off_part_o, off_part_lse;                    // byte offsets from the header
  int32_t n_groups;      // split groups
  int32_t off_groups;    // byte offset of the groups' counters: [n_groups][4] uint32, zero
  int32_t fused_merge;   // 1: the attention CTAs of a split group merge it themselves
};

}  // namespace pkv
