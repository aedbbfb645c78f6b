// Page state machine and planner (see kv_state.h).
#include "kv_state.h"

#include <algorithm>
#include <cstring>
#include <functional>
#include <queue>

#include "../../include/kv.h"

namespace pkv {

namespace {
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }
}  // namespace

int PageState::init(const Config& c0, std::string* why, std::shared_ptr<PatchPool> pool) {
  Config c = c0;
  if (c.sp_base == 0 && c.sp_pages == 0) {
    c.sp_base = c.Np;
    c.sp_pages = c.max_pages - c.Np;
  }
  if (c.page_size < 1 || c.H < 1 || c.D < 1 || c.S < 0 || c.W < 0 || c.B < 1 || c.NS < 0 ||
      c.max_pages < 1 || (c.dtype != KV_BF16 && c.dtype != KV_FP16) || c.Np < 1) {
    *why = "kv_init: invalid argument";
    return KV_ERR_ARG;
  }
  if ((long long)c.max_pages * 2 * c.page_size > 0x7fffffffLL) {
    *why = "kv_init: pool row count exceeds int32";
    return KV_ERR_ARG;
  }
  if (c.sp_base < c.Np || c.sp_pages < (c.NS > 0 ? 1 : 0) || c.sp_base + c.sp_pages > c.max_pages) {
    *why = "kv_init: max_pages must leave at least one special page after the patch pages";
    return KV_ERR_CAPACITY;
  }
  cfg = c;
  if (pool) {
    patch_ = pool;
  } else {
    patch_ = std::make_shared<PatchPool>();
    patch_->Np = c.Np;
  }
  reset();
  return KV_OK;
}

void PageState::reset() {
  if (patch_->shared) {
    for (const auto& fp : scale_) patch_->free.push_back(fp.page);
    for (const auto& fp : window_) patch_->free.push_back(fp.page);
    if (has_pending) patch_->free.push_back(pending_.page);
  } else {
    patch_->free.clear();
    for (int p = cfg.Np - 1; p >= 0; --p) patch_->free.push_back(p);
  }
  scale_.clear();
  window_.clear();
  has_pending = false;
  sp_len = 0;
  committed = 0;
  next_frame = 0;
  defer = false;
  step_open = false;
  appended.assign(cfg.B, 0);
  n_appended = 0;
  step_page = -1;
  step_sp0 = 0;
  ++epoch;
}

void PageState::commit_frame(const FramePage& fp) {
  if ((int)scale_.size() < cfg.S)
    scale_.push_back(fp);
  else
    window_.push_back(fp);
  ++committed;
}

int PageState::peek_append(int block, int* page, int* sp0, std::string* why) const {
  if (block < 0 || block >= cfg.B) {
    *why = "append: block out of range";
    return KV_ERR_ARG;
  }
  const bool new_step = !step_open || n_appended == cfg.B;
  if (new_step) {
    if (has_pending) {
      *why = "append: the deferred frame of the previous step must be committed or rolled back";
      return KV_ERR_ORDER;
    }
    if (patch_->free.empty()) {
      *why = "append: no free patch page (patch_pages too small for S + W)";
      return KV_ERR_CAPACITY;
    }
    if (sp_len + cfg.NS > special_capacity()) {
      *why = "append: special stream full (raise max_pages)";
      return KV_ERR_CAPACITY;
    }
    *page = patch_->free.back();
    *sp0 = sp_len;
    return KV_OK;
  }
  if (appended[block]) {
    *why = "append: block already appended in this frame step";
    return KV_ERR_ORDER;
  }
  *page = step_page;
  *sp0 = step_sp0;
  return KV_OK;
}

int PageState::begin_frame(std::string* why) {
  if (step_open && n_appended < cfg.B) {
    *why = "begin_frame: the open frame step has blocks still to append";
    return KV_ERR_ORDER;
  }
  int page = 0, sp0 = 0;
  const int rc = peek_append(0, &page, &sp0, why);   // the checks of a step-opening append
  if (rc != KV_OK) return rc;
  open_step();
  return KV_OK;
}

void PageState::open_step() {
  const int pg = patch_->free.back();
  patch_->free.pop_back();
  step_sp0 = sp_len;
  sp_len += cfg.NS;
  step_page = pg;
  const FramePage fp{next_frame++, pg, step_sp0};
  if (defer) {
    has_pending = true;
    pending_ = fp;
  } else {
    commit_frame(fp);
  }
  step_open = true;
  std::fill(appended.begin(), appended.end(), 0);
  n_appended = 0;
  ++epoch;
}

int PageState::append(int block, int* page, int* sp0, std::string* why) {
  const int rc = peek_append(block, page, sp0, why);
  if (rc != KV_OK) return rc;
  if (!step_open || n_appended == cfg.B) {
    open_step();
  }
  appended[block] = 1;
  ++n_appended;
  return KV_OK;
}

int PageState::evict() {
  if (defer) return KV_OK;
  bool any = false;
  while ((int)window_.size() > cfg.W) {
    patch_->free.push_back(window_.front().page);
    window_.pop_front();
    any = true;
  }
  if (any) ++epoch;
  return KV_OK;
}

int PageState::set_defer(int on, std::string* why) {
  if (!on && has_pending) {
    *why = "defer_eviction(0): a frame is pending; commit or roll it back";
    return KV_ERR_ORDER;
  }
  defer = on != 0;
  return KV_OK;
}

int PageState::commit(std::string* why) {
  if (!has_pending) {
    *why = "commit: no deferred frame";
    return KV_ERR_NO_PENDING;
  }
  if (n_appended != cfg.B) {
    *why = "commit: not every block of the pending frame has been appended";
    return KV_ERR_ORDER;
  }
  has_pending = false;
  defer = false;
  commit_frame(pending_);
  ++epoch;
  evict();
  return KV_OK;
}

int PageState::rollback(std::string* why) {
  if (!has_pending) {
    *why = "rollback: no deferred frame";
    return KV_ERR_NO_PENDING;
  }
  patch_->free.push_back(pending_.page);
  sp_len -= cfg.NS;
  --next_frame;
  has_pending = false;
  defer = false;
  step_open = false;
  std::fill(appended.begin(), appended.end(), 0);
  n_appended = 0;
  step_page = -1;
  ++epoch;
  return KV_OK;
}

void PageState::special_gap(int* g0, int* g1) const {
  *g0 = *g1 = 0;
  if (cross_special) return;
  const int a = cfg.NS * (int)scale_.size();
  const int b = !window_.empty() ? window_.front().sp0 : has_pending ? pending_.sp0 : sp_len;
  if (b > a) {
    *g0 = a;
    *g1 = b;
  }
}

int PageState::visible_runs(std::vector<PageRun>* runs) const {
  if (committed == 0 && !has_pending) return KV_ERR_EMPTY;
  runs->clear();
  const int ps = cfg.page_size;
  if (!camera_only) {
    for (const auto& fp : scale_) runs->push_back({fp.page, 0, ps});
    for (const auto& fp : window_) runs->push_back({fp.page, 0, ps});
    if (has_pending) runs->push_back({pending_.page, 0, ps});
  }
  int g0, g1;
  special_gap(&g0, &g1);
  // camera-only: the frames' first tokens, stream indices 0, NS, 2 NS, ...
  // (every frame's run starts at a multiple of NS, and so do g0 and g1)
  const int step = camera_only && cfg.NS > 0 ? cfg.NS : 1;
  const int k = ceil_div(sp_len, ps);
  for (int i = 0; i < k; ++i) {
    const int a = i * ps, b = std::min(sp_len, a + ps);   // this page's tokens [a, b) of the stream
    // visible parts: [a, b) minus the hidden range [g0, g1)
    const bool gap = g1 > g0;
    const int pieces[2][2] = {{a, gap ? std::min(b, g0) : b}, {gap ? std::max(a, g1) : b, b}};
    for (const auto& pc : pieces) {
      const int lo = ceil_div(pc[0], step) * step;   // first visible token of the piece
      if (pc[1] > lo) runs->push_back({cfg.sp_base + i, lo - a, pc[1] - a, -1, step});
    }
  }
  return KV_OK;
}

int PageState::tile_runs(std::vector<PageRun>* runs) const {
  std::vector<PageRun> all;
  const int rc = visible_runs(&all);
  if (rc != KV_OK) return rc;
  runs->clear();
  if (!step_open) {
    *runs = all;
    return KV_OK;
  }
  const int ps = cfg.page_size;
  const int c0 = step_sp0, c1 = step_sp0 + cfg.NS;   // the frame's tokens of the special stream
  std::vector<PageRun> cur;
  for (const PageRun& r : all) {
    if (r.page == step_page) {
      cur.push_back({r.page, r.lo, r.hi, cfg.NS + r.lo, r.step});
    } else if (r.page >= cfg.sp_base) {
      // stream tokens [a, b) of this run, split around [c0, c1) (both ends
      // are multiples of NS, so each piece still starts on a visible token)
      const int a = (r.page - cfg.sp_base) * ps + r.lo, b = (r.page - cfg.sp_base) * ps + r.hi;
      const int base = a - r.lo;
      if (std::min(b, c0) > a) runs->push_back({r.page, r.lo, std::min(b, c0) - base, -1, r.step});
      if (std::min(b, c1) > std::max(a, c0))
        cur.push_back({r.page, std::max(a, c0) - base, std::min(b, c1) - base, std::max(a, c0) - c0, r.step});
      if (b > std::max(a, c1)) runs->push_back({r.page, std::max(a, c1) - base, r.hi, -1, r.step});
    } else {
      runs->push_back(r);
    }
  }
  runs->insert(runs->end(), cur.begin(), cur.end());
  return KV_OK;
}

int PageState::page_table(std::vector<int>* idx, int* last_page_len) const {
  std::vector<PageRun> runs;
  const int rc = visible_runs(&runs);
  if (rc != KV_OK) return rc;
  // nothing visible: no scale frame, no window and retention off
  if (runs.empty()) return KV_ERR_EMPTY;
  idx->clear();
  for (const PageRun& r : runs)
    if (idx->empty() || idx->back() != r.page) idx->push_back(r.page);
  // tokens written to the table's final page: the special stream's last page
  // unless retention off hides all of its tokens
  const int ps = cfg.page_size;
  const int last = idx->back();
  *last_page_len = last >= cfg.sp_base ? std::min(ps, sp_len - ps * (last - cfg.sp_base)) : ps;
  return KV_OK;
}

long long PageState::visible_tokens() const {
  std::vector<PageRun> runs;
  if (visible_runs(&runs) != KV_OK) return 0;
  long long n = 0;
  for (const PageRun& r : runs) n += ceil_div(r.hi - r.lo, r.step);
  return n;
}

void build_tiles(const std::vector<PageRun>& runs, int page_size, std::vector<KvTile>* tiles) {
  for (const PageRun& r : runs) {
    const int base = r.page * 2 * page_size;
    // a tile covers rows [s, e) of the run; the next one starts at the run's
    // next visible row (s advances by whole steps)
    const int advance = ceil_div(kTile, r.step) * r.step;
    for (int s = r.lo; s < r.hi; s += advance) {
      const int e = std::min(s + kTile, r.hi);
      KvTile t{};
      if (e - s == kTile) {
        t.row = base + s; t.lo = 0; t.hi = kTile;
      } else if (page_size >= kTile) {
        // the box stays inside the page: anchored at the run's last row when
        // it can be, else at the page's first row; rows outside [s, e) are
        // masked (for the ragged end of a long page they repeat the
        // previous tile)
        const int row0 = e >= kTile ? e - kTile : 0;
        t.row = base + row0; t.lo = (int16_t)(s - row0); t.hi = (int16_t)(e - row0);
      } else {
        // a page shorter than one tile: the box runs past it, rows >= e masked
        t.row = base; t.lo = (int16_t)s; t.hi = (int16_t)e;
      }
      // column c is pool row t.row + c and, for the current frame, k/v row
      // krow + c
      t.krow = r.krow >= 0 ? r.krow + (t.row - base) - r.lo : kNotCurrent;
      t.step = (int16_t)r.step;
      tiles->push_back(t);
    }
  }
}

static size_t header_bytes() { return align_up(sizeof(KvPlanHeader), 256); }

WorkspaceLayout workspace_layout(const std::vector<const PageState*>& st) {
  WorkspaceLayout L{};
  size_t units_base = 0, tiles_cap = 0;
  int D = 0;
  for (const PageState* s : st) {
    const Config& c = s->cfg;
    const int T = c.page_size + c.NS;
    units_base += (size_t)c.H * ceil_div(T, kTile);
    // + the retention gap's split page and the current frame's special runs
    tiles_cap += (size_t)c.max_pages * ceil_div(c.page_size, kTile) + 8;
    D = c.D;
  }
  L.slot_cap = 2 * (units_base + kMaxTargetCtas);
  const size_t units_cap = units_base + L.slot_cap;
  size_t off = header_bytes();
  off += align_up(st.size() * sizeof(KvReq), 16);
  off += align_up(units_cap * sizeof(KvUnit), 16);
  off += align_up(units_base * sizeof(KvMergeItem), 16);
  off += align_up(tiles_cap * sizeof(KvTile), 16);
  off += align_up(units_base * 4 * sizeof(uint32_t), 16);   // split groups' counters
  L.table_bytes = align_up(off, 256);
  L.off_part_o = L.table_bytes;
  L.off_part_lse = align_up(L.off_part_o + L.slot_cap * kTile * (size_t)D * 4, 256);
  L.total = align_up(L.off_part_lse + L.slot_cap * kTile * 4, 256);
  return L;
}

int build_plan(const std::vector<const PageState*>& st, const PlanInputs& in, HostPlan* out,
               std::string* why) {
  HostPlan& P = *out;
  P = HostPlan();
  const int n_req = (int)st.size();
  const Config& c0 = st[0]->cfg;
  const int H = c0.H;
  int q_row0 = 0;
  std::vector<int> tile0(n_req);
  for (int r = 0; r < n_req; ++r) {
    const PageState* s = st[r];
    std::vector<int> table;
    int lpl = 0;
    const int rc = s->page_table(&table, &lpl);
    if (rc != KV_OK) {
      *why = s->committed == 0 && !s->has_pending ? "plan: a stream has no frame yet"
                                                  : "plan: a stream has no visible token";
      return rc;
    }
    std::vector<PageRun> runs;
    s->tile_runs(&runs);
    tile0[r] = (int)P.tiles.size();
    build_tiles(runs, s->cfg.page_size, &P.tiles);
    KvReq rq;
    rq.q_row0 = q_row0;
    rq.T = s->cfg.page_size + s->cfg.NS;
    rq.page_size = s->cfg.page_size;
    rq.n_tiles = (int)P.tiles.size() - tile0[r];
    rq.cur_page = s->step_open ? s->step_page : -1;
    rq.cur_sp0 = s->step_open ? s->step_sp0 : 0;
    rq.sp_base = s->cfg.sp_base;
    rq.NS = s->cfg.NS;
    q_row0 += rq.T;
    P.reqs.push_back(rq);
    P.tables.push_back(table);
    P.last_page_len.push_back(lpl);
    P.visible += s->visible_tokens();
  }

  // Work units: (request, head, pair of query tiles) -- a lone last tile
  // forms a single unit -- each split into chunks of at most L K/V tiles so
  // that the launch fills the machine. When the kernel supports it, a last
  // query tile of at most 16 rows rides as a tail on the preceding unit,
  // which computes it with swapped operands (S^T = K Q^T, N = 16). Per K/V
  // tile a pair costs about 1.0, a single unit about 0.7, a tail 0.3 more.
  struct Group { int req, qt, nq, tail, n; double w; };
  std::vector<Group> groups;
  int n_base = 0, max_n = 0;
  for (int r = 0; r < n_req; ++r) {
    const int T = P.reqs[r].T;
    int qtiles = ceil_div(T, kTile);
    const int last_rows = T - (qtiles - 1) * kTile;
    const bool tail = qtiles >= 2 && last_rows <= in.max_tail_rows;
    if (tail) --qtiles;
    for (int qt = 0; qt < qtiles; qt += 2) {
      const int nq = std::min(2, qtiles - qt);
      const bool last = qt + nq >= qtiles;
      groups.push_back({r, qt, nq, (tail && last) ? last_rows : 0, P.reqs[r].n_tiles,
                        (nq == 2 ? 1.0 : 0.7) + ((tail && last) ? 0.3 : 0.0)});
    }
    n_base += ceil_div(qtiles, 2) * H;
    max_n = std::max(max_n, P.reqs[r].n_tiles);
  }
  const int target = std::max(1, in.num_sms * in.ctas_per_sm);
  int L;
  if (in.tiles_per_split > 0) {
    L = in.tiles_per_split;
  } else {
    // Pick the chunk size whose schedule finishes first when CTAs are handed
    // to `target` slots greedily, longest first (what the block scheduler
    // does); a CTA costs its weighted tiles plus a fixed prologue/epilogue.
    L = max_n;
    double best = 1e300;
    for (int c = 1; c <= 32; ++c) {
      const int cand = std::max(1, ceil_div(max_n, c));
      if (c > 1 && cand == ceil_div(max_n, c - 1)) continue;
      std::vector<double> costs;
      for (const Group& g : groups) {
        const int ch = std::max(1, ceil_div(g.n, cand));
        for (int k = 0; k < ch; ++k) {
          const double tiles = (double)((long long)(k + 1) * g.n / ch - (long long)k * g.n / ch);
          for (int h = 0; h < H; ++h) costs.push_back(tiles * g.w + 2.0 + (ch > 1 ? 1.0 : 0.0));
        }
      }
      if ((int)costs.size() > target + n_base) break;
      std::sort(costs.begin(), costs.end(), std::greater<double>());
      // least-loaded slot first (a min-heap; tied slots are interchangeable,
      // so the loads, and the makespan, do not depend on which one is taken)
      std::priority_queue<double, std::vector<double>, std::greater<double>> slot;
      for (size_t i = 0; i < std::min<size_t>(target, costs.size()); ++i) slot.push(0.0);
      double makespan = 0.0;
      for (double x : costs) {
        const double load = slot.top() + x;
        slot.pop();
        slot.push(load);
        makespan = std::max(makespan, load);
      }
      if (makespan < best * 0.995) {
        best = makespan;
        L = cand;
      }
      if (cand <= 2) break;
    }
  }
  const WorkspaceLayout WL = workspace_layout(st);
  int n_slots = 0, n_groups = 0;
  for (const Group& g : groups) {
    const int nt = g.n;
    const int chunks = std::max(1, ceil_div(nt, L));
    const int ntiles_q = g.nq + (g.tail ? 1 : 0);
    for (int h = 0; h < H; ++h) {
      int slot0[3] = {-1, -1, -1};
      if (chunks > 1) {
        for (int t = 0; t < ntiles_q; ++t) {
          slot0[t] = n_slots;
          n_slots += chunks;
          const KvReq& rq = P.reqs[g.req];
          KvMergeItem m{};
          m.head = (int16_t)h;
          m.rows = (int16_t)std::min(kTile, rq.T - (g.qt + t) * kTile);
          m.n = (int16_t)chunks; m.slot0 = slot0[t];
          m.row0 = rq.q_row0 + (g.qt + t) * kTile;
          P.merges.push_back(m);
          ++P.n_split_units;
        }
      }
      const int group = chunks > 1 ? n_groups++ : -1;
      for (int k = 0; k < chunks; ++k) {
        KvUnit u{};
        u.req = (int16_t)g.req; u.head = (int16_t)h; u.qtile = (int16_t)g.qt; u.nq = (int16_t)g.nq;
        u.tail_rows = (int16_t)g.tail;
        u.chunk = (int16_t)k; u.n_chunks = (int16_t)chunks; u.group = group;
        u.tile_begin = tile0[g.req] + (int)((long long)k * nt / chunks);
        u.tile_end = tile0[g.req] + (int)((long long)(k + 1) * nt / chunks);
        for (int t = 0; t < 3; ++t) u.slot[t] = (chunks > 1 && t < ntiles_q) ? slot0[t] + k : -1;
        P.max_tiles_per_cta = std::max(P.max_tiles_per_cta, u.tile_end - u.tile_begin);
        P.units.push_back(u);
      }
    }
  }
  if ((size_t)n_slots > WL.slot_cap || P.units.size() > 0x7fffffff) {
    *why = "plan: split schedule exceeds the workspace's partial slots";
    return KV_ERR_CAPACITY;
  }
  // Launch order: the block scheduler starts CTAs in index order over a few
  // microseconds, so the longest chunks go first (no two CTAs read the same
  // K/V tile, so the order costs no L2 reuse); ties keep (request, head,
  // first tile) order.
  std::stable_sort(P.units.begin(), P.units.end(), [](const KvUnit& a, const KvUnit& b) {
    const int la = a.tile_end - a.tile_begin, lb = b.tile_end - b.tile_begin;
    if (la != lb) return la > lb;
    if (a.req != b.req) return a.req < b.req;
    if (a.head != b.head) return a.head < b.head;
    if (a.tile_begin != b.tile_begin) return a.tile_begin < b.tile_begin;
    return a.qtile < b.qtile;
  });

  // Serialise.
  KvPlanHeader& Hd = P.header;
  std::memset(&Hd, 0, sizeof(Hd));
  Hd.n_reqs = n_req;
  Hd.n_units = (int)P.units.size();
  Hd.n_merge = (int)P.merges.size();
  Hd.n_tiles = (int)P.tiles.size();
  size_t off = header_bytes();
  Hd.off_reqs = (int)off;   off += align_up(P.reqs.size() * sizeof(KvReq), 16);
  Hd.off_units = (int)off;  off += align_up(P.units.size() * sizeof(KvUnit), 16);
  Hd.off_merge = (int)off;  off += align_up(P.merges.size() * sizeof(KvMergeItem), 16);
  Hd.off_tiles = (int)off;  off += align_up(P.tiles.size() * sizeof(KvTile), 16);
  Hd.off_groups = (int)off; off += align_up((size_t)n_groups * 4 * sizeof(uint32_t), 16);
  Hd.n_groups = n_groups;
  // The attention CTAs of a split group merge it themselves when the launch
  // has at most one CTA per SM slot (so the group's CTAs usually run at the
  // same time and share the merge) and no group has more than 32 chunks (the
  // kernel marks a group's shares in a 32-bit mask); otherwise a separate
  // merge launch does.
  int max_chunks = 0;
  for (const KvUnit& u : P.units) max_chunks = std::max(max_chunks, (int)u.n_chunks);
  Hd.fused_merge = (n_groups > 0 && (int)P.units.size() <= target && max_chunks <= 32) ? 1 : 0;
  Hd.upload_bytes = (int)off;
  Hd.off_part_o = (int64_t)WL.off_part_o;
  Hd.off_part_lse = (int64_t)WL.off_part_lse;
  if (off > WL.table_bytes) {
    *why = "plan: tables exceed the workspace layout";
    return KV_ERR_CAPACITY;
  }
  P.image.assign(off, 0);
  std::memcpy(P.image.data(), &Hd, sizeof(Hd));
  std::memcpy(P.image.data() + Hd.off_reqs, P.reqs.data(), P.reqs.size() * sizeof(KvReq));
  std::memcpy(P.image.data() + Hd.off_units, P.units.data(), P.units.size() * sizeof(KvUnit));
  if (!P.merges.empty())
    std::memcpy(P.image.data() + Hd.off_merge, P.merges.data(), P.merges.size() * sizeof(KvMergeItem));
  std::memcpy(P.image.data() + Hd.off_tiles, P.tiles.data(), P.tiles.size() * sizeof(KvTile));
  return KV_OK;
}

}  // namespace pkv
