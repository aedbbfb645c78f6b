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
};

// 128 consecutive pool rows of one page, starting at K row `row` of the
// [pages * 2 * page_size] row space of the pool; V rows start page_size
// later. Columns [lo, hi) of the tile are visible tokens, the rest masked.
struct KvTile {
  int32_t row;
  int16_t lo;
  int16_t hi;
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
  int16_t pad;
  int32_t tile_begin;  // absolute index into the tile table
  int32_t tile_end;
  int32_t slot[3];     // per query tile (tail last): -1 = write `out`, else partial slot
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
};

}  // namespace pkv
