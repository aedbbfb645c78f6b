// Host-side page state of one stream's paged KV cache, and the planner that
// turns the visible page tables of a batch of streams into the device plan.
// Plain C++17, no CUDA.
//
// Page state ([P1] "Two-Stream Page Design"; [P2] "Two-Stream Design: Patch vs.
// Special Tokens", "Sliding-Window Eviction Strategy", "Flow-Based Keyframe
// Selection"):
//   - patch pages [0, Np) come from a LIFO free list (initially Np-1 .. 0 from
//     bottom to top, so the first frames get pages 0, 1, 2, ...);
//   - the first S committed frames keep their pages for good (scale pages);
//   - later frames form the window, oldest first; eviction returns the oldest
//     to the free list while more than W are resident;
//   - the special stream packs NS tokens per frame back to back over pages
//     [Np, max_pages): token j sits on page Np + j / page_size, slot
//     j % page_size;
//   - a frame appended while eviction is deferred stays pending until it is
//     committed or rolled back;
//   - without cross-frame special retention ([P2] "Configuration
//     Parameters"), the special tokens of evicted frames are not visible.
//     Evictions take the oldest window frame, so the hidden tokens form one
//     range of the special stream, between the scale frames' and the
//     window's.
// (The pages are titled "How the Paged KV Cache Attention Mechanism Enables
// Long Sequence Inference in LingBot-Map" [P1] and "KV Cache Mechanism in
// LingBot-Map for Streaming Inference: A Deep Dive" [P2].)
#pragma once
#include <cstdint>
#include <deque>
#include <memory>
#include <string>
#include <vector>

#include "kv_layout.h"

namespace pkv {

struct FramePage {
  int frame;
  int page;
  int sp0;   // the frame's first token in the special stream
};

// A visible range [lo, hi) of rows of one pool page.
// Visible rows lo, lo + step, ... < hi of one pool page (step > 1: the
// camera tokens of a camera-only cache, lo being one of them).
struct PageRun {
  int page;
  int lo, hi;
  int krow = -1;   // rows of the current frame: k/v row of row lo (>= 0), else -1
  int step = 1;
};

struct Config {
  int max_pages, page_size, H, D, S, W, B, NS, dtype, Np;
  int sp_base = 0;    // this stream's special pages [sp_base, sp_base + sp_pages)
  int sp_pages = 0;   // (0, 0 at init: every page after the patch pages)
};

// Patch pages [0, Np) and their LIFO free list (back() is handed out next).
// A stream alone in its pool owns one; the streams of a group share one.
struct PatchPool {
  std::vector<int> free;
  int Np = 0;
  bool shared = false;
};

class PageState {
 public:
  Config cfg{};
  std::shared_ptr<PatchPool> patch_;   // patch pages and their free list
  std::vector<FramePage> scale_;
  std::deque<FramePage> window_;
  bool has_pending = false;
  FramePage pending_{};
  int sp_len = 0;
  int committed = 0;
  int next_frame = 0;
  bool defer = false;
  bool cross_special = true;   // special tokens of evicted frames stay visible
  bool camera_only = false;    // attention sees only the camera tokens (slot 0 of each frame's NS)
  // frame step
  bool step_open = false;
  std::vector<uint8_t> appended;
  int n_appended = 0;
  int step_page = -1;
  int step_sp0 = 0;
  uint64_t epoch = 1;   // bumped on every change of the visible table

  // Returns KV_OK or a KV_ERR_* code; `why` gets a one-line detail on error.
  // `pool`: a patch pool shared with other streams (NULL: a pool of its own).
  int init(const Config& c, std::string* why, std::shared_ptr<PatchPool> pool = nullptr);
  // Back to the initial state. In a shared pool this stream's patch pages go
  // back to the common free list: scale pages (frame order), then window
  // pages (oldest first), then a pending page.
  void reset();
  const std::vector<int>& free_list() const { return patch_->free; }
  // Marks `block` appended in the current step, opening a new step (and
  // taking a patch page and NS special slots) when needed.
  int append(int block, int* page, int* sp0, std::string* why);
  // What append(block) would return (status, page, sp0), with no change to
  // the state: lets a caller launch the scatter first and advance the state
  // only once the launch has succeeded.
  int peek_append(int block, int* page, int* sp0, std::string* why) const;
  int evict();
  int set_defer(int on, std::string* why);
  int commit(std::string* why);
  int rollback(std::string* why);
  int page_table(std::vector<int>* idx, int* last_page_len) const;
  // Hidden range [g0, g1) of the special stream (empty unless cross-frame
  // special retention is off and frames have been evicted).
  void special_gap(int* g0, int* g1) const;
  // The visible rows, page by page, in page-table order.
  int visible_runs(std::vector<PageRun>* runs) const;
  // The visible rows as the K/V tiles cover them: visible_runs with the rows
  // of the open step's frame (its patch page and its NS special tokens, those
  // that are visible) taken out and appended at the end with their k/v rows.
  int tile_runs(std::vector<PageRun>* runs) const;
  // Opens a frame step without appending a block (takes the frame's patch
  // page and NS special slots); the blocks are appended afterwards.
  int begin_frame(std::string* why);
  int special_capacity() const { return cfg.sp_pages * cfg.page_size; }
  bool is_appended(int block) const {
    return step_open && block >= 0 && block < cfg.B && appended[block];
  }
  long long visible_tokens() const;

 private:
  void commit_frame(const FramePage& fp);
  void open_step();   // the step-opening part of append (checks done by the caller)
};

struct PlanInputs {
  int num_sms;           // SMs of the device
  int ctas_per_sm;       // attention CTAs resident per SM
  int tiles_per_split;   // > 0: forced chunk size (tests); 0: automatic
  int max_tail_rows;     // the attention kernel computes tail tiles of up to this many rows in-unit
};

struct HostPlan {
  std::vector<std::vector<int>> tables;
  std::vector<int> last_page_len;
  std::vector<KvReq> reqs;
  std::vector<KvUnit> units;
  std::vector<KvMergeItem> merges;
  std::vector<KvTile> tiles;
  std::vector<uint8_t> image;   // header + tables, as uploaded
  KvPlanHeader header{};
  int max_tiles_per_cta = 0;
  int n_split_units = 0;
  long long visible = 0;
};

// Capacities that fix the workspace layout for a set of caches.
struct WorkspaceLayout {
  size_t table_bytes;   // header + tables region
  size_t slot_cap;      // split-KV partial slots
  size_t off_part_o, off_part_lse, total;
};

WorkspaceLayout workspace_layout(const std::vector<const PageState*>& st);

// Builds the K/V tile list of one stream's visible rows.
void build_tiles(const std::vector<PageRun>& runs, int page_size, std::vector<KvTile>* tiles);

int build_plan(const std::vector<const PageState*>& st, const PlanInputs& in, HostPlan* out,
               std::string* why);

}  // namespace pkv
