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
struct PageRun {
  int page;
  int lo, hi;
};

struct Config {
  int max_pages, page_size, H, D, S, W, B, NS, dtype, Np;
};

class PageState {
 public:
  Config cfg{};
  std::vector<int> free_;        // back() is the next page handed out
  std::vector<FramePage> scale_;
  std::deque<FramePage> window_;
  bool has_pending = false;
  FramePage pending_{};
  int sp_len = 0;
  int committed = 0;
  int next_frame = 0;
  bool defer = false;
  bool cross_special = true;   // special tokens of evicted frames stay visible
  // frame step
  bool step_open = false;
  std::vector<uint8_t> appended;
  int n_appended = 0;
  int step_page = -1;
  int step_sp0 = 0;
  uint64_t epoch = 1;   // bumped on every change of the visible table

  // Returns KV_OK or a KV_ERR_* code; `why` gets a one-line detail on error.
  int init(const Config& c, std::string* why);
  void reset();
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
  int special_capacity() const { return (cfg.max_pages - cfg.Np) * cfg.page_size; }
  bool is_appended(int block) const {
    return step_open && block >= 0 && block < cfg.B && appended[block];
  }
  long long visible_tokens() const;

 private:
  void commit_frame(const FramePage& fp);
};

struct PlanInputs {
  int num_sms;           // SMs of the device
  int ctas_per_sm;       // attention CTAs resident per SM
  int tiles_per_split;   // > 0: forced chunk size (tests); 0: automatic
  bool tail_ok;          // the attention kernel computes <= 16-row tail tiles in-unit
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
