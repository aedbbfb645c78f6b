// C-ABI of the paged KV cache (declared in include/kv.h): argument checks,
// host page state, plan upload, TMA descriptors and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <cstring>
#include <memory>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/kv.h"
#include "kernels.h"
#include "kv_state.h"
#include "launch.cuh"

// The device pools of one cache, or of every cache of a group (shared).
struct DevPools {
  std::vector<void*> pools;
  std::vector<CUtensorMap> maps;
  std::vector<uint8_t> bound;
};

struct kv_cache {
  pkv::PageState st;
  std::shared_ptr<DevPools> dev;
};

struct kv_plan {
  std::vector<kv_cache*> caches;
  std::vector<uint64_t> epochs;
  pkv::HostPlan hp;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int H = 0, D = 0, dtype = 0, total_T = 0;
};

namespace {

thread_local std::string g_last;

int fail(int code, const std::string& why) {
  g_last = why;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  g_last = std::string(where) + ": " + cudaGetErrorString(e);
  return KV_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Looked up once; the initialisation of a function-local static is
// thread-safe, so concurrent first calls from several threads are fine.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

// 3-D view [rows][H][D] of a row-major [rows, H, D] tensor; boxes of
// 128 rows x 1 head x 64 columns with 128-byte swizzle (the UMMA K-major /
// MN-major canonical layout).
int encode_rows_map(CUtensorMap* m, const void* base, int H, int D, long long rows, int dtype) {
  auto fn = encode_fn();
  if (!fn) return fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (no CUDA driver)");
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)pkv::kTile};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dtype == KV_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return KV_OK;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

}  // namespace

namespace pkv {
std::atomic<int> g_fail_launches{0};
}

extern "C" {

void kv_testing_fail_launches(int n) { pkv::g_fail_launches.store(n > 0 ? n : 0); }

const char* kv_strerror(int status) {
  switch (status) {
    case KV_OK: return "ok";
    case KV_ERR_ARG: return "invalid argument";
    case KV_ERR_CAPACITY: return "capacity exceeded";
    case KV_ERR_ORDER: return "call out of order";
    case KV_ERR_NO_PENDING: return "no pending (deferred) frame";
    case KV_ERR_NOT_APPENDED: return "block not appended in this frame step";
    case KV_ERR_EMPTY: return "cache holds no frame or no visible token";
    case KV_ERR_CUDA: return "CUDA error";
    case KV_ERR_DEVICE_CHECK: return "device-side check failed";
    case KV_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case KV_ERR_STALE_PLAN: return "plan is stale (cache state changed)";
    default: return "unknown status";
  }
}

const char* kv_last_error(void) { return g_last.c_str(); }

int kv_init(kv_cache_t** out, int max_pages, int page_size, int num_heads, int head_dim, int scale_frames,
            int window, int num_blocks, int num_special, int dtype, int patch_pages) {
  if (!out) return fail(KV_ERR_ARG, "kv_init: out is NULL");
  *out = nullptr;
  if (head_dim % 8 != 0) return fail(KV_ERR_ARG, "kv_init: head_dim must be a multiple of 8");
  pkv::Config c{max_pages, page_size, num_heads, head_dim, scale_frames, window, num_blocks, num_special, dtype,
                patch_pages > 0 ? patch_pages : scale_frames + window + 1};
  if (patch_pages < 0) return fail(KV_ERR_ARG, "kv_init: patch_pages < 0");
  kv_cache* k = new kv_cache();
  std::string why;
  const int rc = k->st.init(c, &why);
  if (rc != KV_OK) {
    delete k;
    return fail(rc, why);
  }
  k->dev = std::make_shared<DevPools>();
  k->dev->pools.assign(num_blocks, nullptr);
  k->dev->maps.assign(num_blocks, CUtensorMap{});
  k->dev->bound.assign(num_blocks, 0);
  *out = k;
  return KV_OK;
}

int kv_init_group(kv_cache_t** out, int n_streams, int max_pages, int page_size, int num_heads, int head_dim,
                  int scale_frames, int window, int num_blocks, int num_special, int dtype, int patch_pages,
                  int special_pages) {
  if (!out) return fail(KV_ERR_ARG, "kv_init_group: out is NULL");
  if (n_streams < 1 || n_streams > KV_MAX_STREAMS) return fail(KV_ERR_ARG, "kv_init_group: n_streams out of range");
  for (int i = 0; i < n_streams; ++i) out[i] = nullptr;
  if (head_dim % 8 != 0) return fail(KV_ERR_ARG, "kv_init_group: head_dim must be a multiple of 8");
  if (patch_pages < 0 || special_pages < 0) return fail(KV_ERR_ARG, "kv_init_group: negative page count");
  const int Np = patch_pages > 0 ? patch_pages : n_streams * (scale_frames + window + 1);
  const int sp = special_pages > 0 ? special_pages : (max_pages - Np) / n_streams;
  if ((long long)Np + (long long)n_streams * sp > max_pages || sp < (num_special > 0 ? 1 : 0))
    return fail(KV_ERR_CAPACITY, "kv_init_group: max_pages < patch_pages + n_streams * special_pages");
  auto pool = std::make_shared<pkv::PatchPool>();
  pool->Np = Np;
  pool->shared = true;
  for (int p = Np - 1; p >= 0; --p) pool->free.push_back(p);
  auto dev = std::make_shared<DevPools>();
  dev->pools.assign(num_blocks, nullptr);
  dev->maps.assign(num_blocks, CUtensorMap{});
  dev->bound.assign(num_blocks, 0);
  for (int i = 0; i < n_streams; ++i) {
    pkv::Config c{max_pages, page_size, num_heads, head_dim, scale_frames, window, num_blocks, num_special, dtype,
                  Np, Np + i * sp, sp};
    kv_cache* k = new kv_cache();
    std::string why;
    const int rc = k->st.init(c, &why, pool);
    if (rc != KV_OK) {
      delete k;
      for (int j = 0; j < i; ++j) {
        delete out[j];
        out[j] = nullptr;
      }
      return fail(rc, why);
    }
    k->dev = dev;
    out[i] = k;
  }
  return KV_OK;
}

void kv_destroy(kv_cache_t* c) { delete c; }

int kv_reset(kv_cache_t* c) {
  if (!c) return fail(KV_ERR_ARG, "kv_reset: NULL cache");
  c->st.reset();
  return KV_OK;
}

size_t kv_pool_bytes(const kv_cache_t* c) {
  if (!c) return 0;
  const pkv::Config& g = c->st.cfg;
  return (size_t)g.max_pages * 2 * g.page_size * g.H * g.D * 2;
}

int kv_bind_pool(kv_cache_t* c, int block, void* pool, void* stream) {
  if (!c || !pool) return fail(KV_ERR_ARG, "kv_bind_pool: NULL argument");
  if (block < 0 || block >= c->st.cfg.B) return fail(KV_ERR_ARG, "kv_bind_pool: block out of range");
  if (!aligned16(pool)) return fail(KV_ERR_ARG, "kv_bind_pool: pool not 16-byte aligned");
  const pkv::Config& g = c->st.cfg;
  cudaError_t e = cudaMemsetAsync(pool, 0, kv_pool_bytes(c), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kv_bind_pool: memset");
  if (g.D % 64 == 0) {
    const int rc = encode_rows_map(&c->dev->maps[block], pool, g.H, g.D, (long long)g.max_pages * 2 * g.page_size,
                                   g.dtype);
    if (rc != KV_OK) return rc;
  }
  c->dev->pools[block] = pool;
  c->dev->bound[block] = 1;
  return KV_OK;
}

int kv_append_frame(kv_cache_t* c, int block, const void* k, const void* v, void* stream) {
  if (!c) return fail(KV_ERR_ARG, "kv_append_frame: NULL cache");
  if ((k == nullptr) != (v == nullptr)) return fail(KV_ERR_ARG, "kv_append_frame: k and v must both be set or both NULL");
  const pkv::Config& g = c->st.cfg;
  if (block < 0 || block >= g.B) return fail(KV_ERR_ARG, "kv_append_frame: block out of range");
  if (k) {
    if (!c->dev->bound[block]) return fail(KV_ERR_ARG, "kv_append_frame: no pool bound for this block");
    if (!aligned16(k) || !aligned16(v)) return fail(KV_ERR_ARG, "kv_append_frame: k/v not 16-byte aligned");
  }
  // The scatter is launched before the page state advances, so a failed
  // launch leaves the cache exactly as it was.
  int page = -1, sp0 = 0;
  std::string why;
  int rc = c->st.peek_append(block, &page, &sp0, &why);
  if (rc != KV_OK) return fail(rc, why);
  if (k) {
    pkv::AppendArgs a;
    a.k = k;
    a.v = v;
    a.pool = c->dev->pools[block];
    a.T = g.page_size + g.NS;
    a.NS = g.NS;
    a.page_size = g.page_size;
    a.sp_base = g.sp_base;
    a.max_pages = g.max_pages;
    a.row_vecs = g.H * g.D * 2 / 16;
    a.patch_page = page;
    a.sp0 = sp0;
    cudaError_t e = pkv::launch_append(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kv_append_frame: scatter launch");
  }
  rc = c->st.append(block, &page, &sp0, &why);
  return rc == KV_OK ? KV_OK : fail(rc, why);
}

int kv_evict_frames(kv_cache_t* c) {
  if (!c) return fail(KV_ERR_ARG, "kv_evict_frames: NULL cache");
  return c->st.evict();
}

int kv_defer_eviction(kv_cache_t* c, int on) {
  if (!c) return fail(KV_ERR_ARG, "kv_defer_eviction: NULL cache");
  std::string why;
  const int rc = c->st.set_defer(on, &why);
  return rc == KV_OK ? rc : fail(rc, why);
}

int kv_commit_frame(kv_cache_t* c) {
  if (!c) return fail(KV_ERR_ARG, "kv_commit_frame: NULL cache");
  std::string why;
  const int rc = c->st.commit(&why);
  return rc == KV_OK ? rc : fail(rc, why);
}

int kv_rollback_last_frame(kv_cache_t* c) {
  if (!c) return fail(KV_ERR_ARG, "kv_rollback_last_frame: NULL cache");
  std::string why;
  const int rc = c->st.rollback(&why);
  return rc == KV_OK ? rc : fail(rc, why);
}

int kv_get_config(const kv_cache_t* c, kv_config* out) {
  if (!c || !out) return fail(KV_ERR_ARG, "kv_get_config: NULL argument");
  const pkv::Config& g = c->st.cfg;
  out->max_pages = g.max_pages;
  out->page_size = g.page_size;
  out->num_heads = g.H;
  out->head_dim = g.D;
  out->scale_frames = g.S;
  out->window = g.W;
  out->num_blocks = g.B;
  out->num_special = g.NS;
  out->dtype = g.dtype;
  out->patch_pages = g.Np;
  out->special_base = g.sp_base;
  out->special_pages = g.sp_pages;
  out->tokens_per_frame = g.page_size + g.NS;
  out->cross_frame_special = c->st.cross_special ? 1 : 0;
  out->camera_only = c->st.camera_only ? 1 : 0;
  return KV_OK;
}

int kv_get_stats(const kv_cache_t* c, kv_stats* out) {
  if (!c || !out) return fail(KV_ERR_ARG, "kv_get_stats: NULL argument");
  const pkv::PageState& s = c->st;
  const int pend = s.has_pending ? 1 : 0;
  out->frame_count = s.committed + pend;
  out->scale_pages = (int)s.scale_.size();
  out->live_pages = (int)s.window_.size() + pend;
  out->free_pages = (int)s.free_list().size();
  out->special_tokens = s.sp_len;
  return KV_OK;
}

int kv_set_cross_frame_special(kv_cache_t* c, int on) {
  if (!c) return fail(KV_ERR_ARG, "kv_set_cross_frame_special: NULL cache");
  const bool v = on != 0;
  if (c->st.cross_special != v) {
    c->st.cross_special = v;
    ++c->st.epoch;
  }
  return KV_OK;
}

int kv_set_camera_only(kv_cache_t* c, int on) {
  if (!c) return fail(KV_ERR_ARG, "kv_set_camera_only: NULL cache");
  const bool v = on != 0;
  if (c->st.camera_only != v) {
    c->st.camera_only = v;
    ++c->st.epoch;
  }
  return KV_OK;
}

int kv_get_free_list(const kv_cache_t* c, int* ids, int cap, int* n) {
  if (!c || !n || cap < 0 || (cap > 0 && !ids)) return fail(KV_ERR_ARG, "kv_get_free_list: bad argument");
  const auto& f = c->st.free_list();
  *n = (int)f.size();
  for (int i = 0; i < (int)f.size() && i < cap; ++i) ids[i] = f[i];
  return KV_OK;
}

static int check_batch(kv_cache_t* const* caches, int n, std::vector<const pkv::PageState*>* st) {
  if (!caches || n < 1) return fail(KV_ERR_ARG, "plan: no caches");
  if (n > KV_MAX_STREAMS) return fail(KV_ERR_CAPACITY, "plan: more than KV_MAX_STREAMS streams");
  for (int i = 0; i < n; ++i) {
    if (!caches[i]) return fail(KV_ERR_ARG, "plan: NULL cache");
    const pkv::Config& a = caches[0]->st.cfg;
    const pkv::Config& b = caches[i]->st.cfg;
    if (a.page_size != b.page_size || a.H != b.H || a.D != b.D || a.NS != b.NS || a.B != b.B || a.dtype != b.dtype)
      return fail(KV_ERR_ARG, "plan: caches differ in page_size/H/D/NS/num_blocks/dtype");
    st->push_back(&caches[i]->st);
  }
  return KV_OK;
}

size_t kv_workspace_bytes(kv_cache_t* const* caches, int n_streams) {
  std::vector<const pkv::PageState*> st;
  if (check_batch(caches, n_streams, &st) != KV_OK) return 0;
  return pkv::workspace_layout(st).total;
}

int kv_plan(kv_plan_t** out, kv_cache_t* const* caches, int n_streams, int tiles_per_split, void* workspace,
            size_t workspace_bytes, void* stream) {
  if (!out) return fail(KV_ERR_ARG, "kv_plan: out is NULL");
  *out = nullptr;
  if (tiles_per_split < 0) return fail(KV_ERR_ARG, "kv_plan: tiles_per_split < 0");
  std::vector<const pkv::PageState*> st;
  int rc = check_batch(caches, n_streams, &st);
  if (rc != KV_OK) return rc;
  const pkv::Config& g = st[0]->cfg;
  if (workspace) {
    if (!aligned16(workspace)) return fail(KV_ERR_ARG, "kv_plan: workspace not 16-byte aligned");
    if (workspace_bytes < pkv::workspace_layout(st).total)
      return fail(KV_ERR_CAPACITY, "kv_plan: workspace smaller than kv_workspace_bytes()");
  }
  pkv::PlanInputs in;
  in.num_sms = workspace ? device_sms() : 148;
  in.ctas_per_sm = pkv::attention_ctas_per_sm(g.D);
  in.tiles_per_split = tiles_per_split;
  in.max_tail_rows = pkv::attention_max_tail_rows(g.D);
  kv_plan_t* p = new kv_plan_t();
  std::string why;
  rc = pkv::build_plan(st, in, &p->hp, &why);
  if (rc != KV_OK) {
    delete p;
    return fail(rc, why);
  }
  for (int i = 0; i < n_streams; ++i) {
    p->caches.push_back(caches[i]);
    p->epochs.push_back(caches[i]->st.epoch);
    p->total_T += g.page_size + g.NS;
  }
  p->H = g.H;
  p->D = g.D;
  p->dtype = g.dtype;
  p->ws = workspace;
  p->ws_bytes = workspace_bytes;
  if (workspace) {
    cudaError_t e = pkv::upload_plan(workspace, p->hp.image.data(), p->hp.image.size(), (cudaStream_t)stream);
    if (e != cudaSuccess) {
      delete p;
      return cuda_fail(e, "kv_plan: upload");
    }
  }
  *out = p;
  return KV_OK;
}

void kv_plan_free(kv_plan_t* plan) { delete plan; }

}  // extern "C"

namespace {

// kv_run, and kv_run_append when k and v are given: the launch then also
// writes the open step's frame (block `block`'s K/V) into every request's pool
// and reads that frame's tiles from k and v. Marks the block appended once
// the attention launch has succeeded.
int run_impl(const kv_plan_t* p, int block, const void* q, void* out, const void* k, const void* v,
             void* stream, const char* who) {
  const std::string w(who);
  const bool append = k != nullptr;
  if (!p || !q || !out) return fail(KV_ERR_ARG, w + ": NULL argument");
  if (append != (v != nullptr)) return fail(KV_ERR_ARG, w + ": k and v must both be set");
  if (!p->ws) return fail(KV_ERR_ARG, w + ": host-only plan (built without a workspace)");
  if (p->D != 64 && p->D != 128) return fail(KV_ERR_UNSUPPORTED, w + ": head_dim must be 64 or 128");
  if (!aligned16(q) || !aligned16(out)) return fail(KV_ERR_ARG, w + ": q/out not 16-byte aligned");
  if (append && (!aligned16(k) || !aligned16(v))) return fail(KV_ERR_ARG, w + ": k/v not 16-byte aligned");
  const int B = p->caches[0]->st.cfg.B;
  if (block < 0 || block >= B) return fail(KV_ERR_ARG, w + ": block out of range");
  pkv::AttnMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  pkv::AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  for (size_t r = 0; r < p->caches.size(); ++r) {
    const kv_cache* c = p->caches[r];
    if (c->st.epoch != p->epochs[r]) return fail(KV_ERR_STALE_PLAN, w + ": cache state changed after kv_plan");
    if (!c->dev->bound[block]) return fail(KV_ERR_ARG, w + ": no pool bound for this block");
    if (append) {
      // the plan's frame step must be open with this block still to append
      const pkv::PageState& st = c->st;
      if (!st.step_open || st.n_appended == st.cfg.B || p->hp.reqs[r].cur_page != st.step_page)
        return fail(KV_ERR_ORDER, w + ": no open frame step for this plan (call kv_begin_frame before kv_plan)");
      if (st.appended[block]) return fail(KV_ERR_ORDER, w + ": block already appended in this frame step");
      a.pools[r] = c->dev->pools[block];
    } else if (!c->st.is_appended(block)) {
      return fail(KV_ERR_NOT_APPENDED, w + ": block not appended in this step");
    }
    maps.kv[r] = c->dev->maps[block];
  }
  // Blocks run in order in a frame step, all on this plan: the CTAs prefetch
  // the first tiles of their units from the next block's pools into L2 once
  // their own loads are issued, so the next launch starts on L2 hits. Only
  // while a launch's K/V fits well inside L2 (126 MB): a larger launch evicts
  // the prefetched tiles before the next one reads them.
  const double kv_bytes = 2.0 * (double)p->hp.visible * p->H * p->D * 2.0;
  a.prefetch_next = block + 1 < B && kv_bytes <= 80.0 * (1 << 20);
  for (size_t r = 0; r < p->caches.size() && a.prefetch_next; ++r) {
    const kv_cache* c = p->caches[r];
    if (!c->dev->bound[block + 1]) a.prefetch_next = 0;
    else maps.kv_next[r] = c->dev->maps[block + 1];
  }
  int rc = encode_rows_map(&maps.q, q, p->H, p->D, p->total_T, p->dtype);
  if (rc == KV_OK && append) rc = encode_rows_map(&maps.k, k, p->H, p->D, p->total_T, p->dtype);
  if (rc == KV_OK && append) rc = encode_rows_map(&maps.v, v, p->H, p->D, p->total_T, p->dtype);
  if (rc != KV_OK) return rc;
  uint8_t* ws = static_cast<uint8_t*>(p->ws);
  const pkv::KvPlanHeader& hd = p->hp.header;
  a.q = q;
  a.reqs = reinterpret_cast<const pkv::KvReq*>(ws + hd.off_reqs);
  a.units = reinterpret_cast<const pkv::KvUnit*>(ws + hd.off_units);
  a.tiles = reinterpret_cast<const pkv::KvTile*>(ws + hd.off_tiles);
  a.part_o = reinterpret_cast<float*>(ws + hd.off_part_o);
  a.part_lse = reinterpret_cast<float*>(ws + hd.off_part_lse);
  a.out = out;
  a.err = reinterpret_cast<uint32_t*>(ws);
  a.groups = reinterpret_cast<uint32_t*>(ws + hd.off_groups);
  a.fused_merge = hd.fused_merge;
  a.H = p->H;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->D));
  a.fused_append = append ? 1 : 0;
  a.n_reqs = (int)p->caches.size();
  a.row_vecs = p->H * p->D * 2 / 16;
  a.k = k;
  a.v = v;
  cudaError_t e = pkv::launch_attention(maps, a, p->D, p->dtype == KV_FP16, hd.n_units, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, (w + ": attention launch").c_str());
  if (append) {
    // the launch writes the frame into the pools: the block is appended
    for (kv_cache* c : p->caches) {
      int page = 0, sp0 = 0;
      std::string why;
      c->st.append(block, &page, &sp0, &why);
    }
  }
  if (hd.n_merge > 0 && !hd.fused_merge) {
    pkv::MergeArgs m;
    m.items = reinterpret_cast<const pkv::KvMergeItem*>(ws + hd.off_merge);
    m.part_o = a.part_o;
    m.part_lse = a.part_lse;
    m.out = out;
    m.H = p->H;
    m.n_items = hd.n_merge;
    e = pkv::launch_merge(m, p->D, p->dtype == KV_FP16, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, (w + ": merge launch").c_str());
  }
  return KV_OK;
}

}  // namespace

extern "C" {

int kv_run(const kv_plan_t* p, int block, const void* q, void* out, void* stream) {
  return run_impl(p, block, q, out, nullptr, nullptr, stream, "kv_run");
}

int kv_run_append(const kv_plan_t* p, int block, const void* k, const void* v, const void* q, void* out,
                  void* stream) {
  if (!k || !v) return fail(KV_ERR_ARG, "kv_run_append: NULL k/v");
  return run_impl(p, block, q, out, k, v, stream, "kv_run_append");
}

int kv_begin_frame(kv_cache_t* c) {
  if (!c) return fail(KV_ERR_ARG, "kv_begin_frame: NULL cache");
  std::string why;
  const int rc = c->st.begin_frame(&why);
  return rc == KV_OK ? rc : fail(rc, why);
}

int kv_get_page_table(const kv_plan_t* p, int stream_idx, int* indices, int cap, int* n, int* last_page_len) {
  if (!p || !n || !last_page_len || cap < 0 || (cap > 0 && !indices))
    return fail(KV_ERR_ARG, "kv_get_page_table: bad argument");
  if (stream_idx < 0 || stream_idx >= (int)p->hp.tables.size())
    return fail(KV_ERR_ARG, "kv_get_page_table: stream out of range");
  const auto& t = p->hp.tables[stream_idx];
  *n = (int)t.size();
  for (int i = 0; i < (int)t.size() && i < cap; ++i) indices[i] = t[i];
  *last_page_len = p->hp.last_page_len[stream_idx];
  return KV_OK;
}

int kv_get_kv_tiles(const kv_plan_t* p, int stream_idx, int* row, int* lo, int* hi, int* krow, int* step, int cap,
                    int* n) {
  if (!p || !n || cap < 0 || (cap > 0 && (!row || !lo || !hi))) return fail(KV_ERR_ARG, "kv_get_kv_tiles: bad argument");
  if (stream_idx < 0 || stream_idx >= (int)p->hp.reqs.size()) return fail(KV_ERR_ARG, "kv_get_kv_tiles: stream out of range");
  int t0 = 0;
  for (int r = 0; r < stream_idx; ++r) t0 += p->hp.reqs[r].n_tiles;
  const int nt = p->hp.reqs[stream_idx].n_tiles;
  *n = nt;
  for (int i = 0; i < nt && i < cap; ++i) {
    const pkv::KvTile& t = p->hp.tiles[t0 + i];
    row[i] = t.row;
    lo[i] = t.lo;
    hi[i] = t.hi;
    if (krow) krow[i] = t.krow;
    if (step) step[i] = t.step;
  }
  return KV_OK;
}

int kv_plan_get_stats(const kv_plan_t* p, kv_plan_stats* out) {
  if (!p || !out) return fail(KV_ERR_ARG, "kv_plan_get_stats: NULL argument");
  out->n_streams = (int)p->caches.size();
  out->n_ctas = (int)p->hp.units.size();
  out->n_split_units = p->hp.n_split_units;
  out->n_kv_tiles = (int)p->hp.tiles.size();
  out->tiles_per_cta = p->hp.max_tiles_per_cta;
  out->visible_tokens = p->hp.visible;
  out->fused_merge = p->hp.header.fused_merge;
  out->run_launches = (p->hp.header.n_units > 0 ? 1 : 0) +
                      (p->hp.header.n_merge > 0 && !p->hp.header.fused_merge ? 1 : 0);
  out->upload_launches = p->ws ? pkv::upload_launches(p->hp.image.size()) : 0;
  return KV_OK;
}

int kv_check_device(const kv_plan_t* p, void* stream) {
  if (!p || !p->ws) return fail(KV_ERR_ARG, "kv_check_device: plan without workspace");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kv_check_device: synchronize");
  uint32_t w = 0;
  e = cudaMemcpy(&w, p->ws, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "kv_check_device: read error word");
  if (w) return fail(KV_ERR_DEVICE_CHECK, "kernel error word " + std::to_string(w));
  return KV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// kv_run_static: kv_plan + kv_run for one block with the scratch (plan tables
// and split-KV partials) in a library-owned device array, for callers that
// cannot allocate device memory. Nothing here calls an allocator.

// Every device that loads this module holds this array until the process
// exits. In host code the name is only a stand-in for the device symbol: its
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_static_scratch[KV_STATIC_SCRATCH_BYTES];

namespace {

using pkv::kMaxDevices;
std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};   // device address of g_static_scratch, per device

// Device address of the array on the current device, looked up once per
// device with that device current.
int static_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "kv_run_static: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(KV_ERR_UNSUPPORTED, "kv_run_static: device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "kv_run_static: cudaGetSymbolAddress");
    g_static_addr[dev] = p;
  }
  *ptr = g_static_addr[dev];
  return KV_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" int kv_run_static(kv_cache_t* const* caches, int n_streams, int block, int tiles_per_split,
                             const void* q, void* out, int check, void* stream) {
  if (!q || !out) return fail(KV_ERR_ARG, "kv_run_static: NULL q/out");
  if (tiles_per_split < 0) return fail(KV_ERR_ARG, "kv_run_static: tiles_per_split < 0");
  std::vector<const pkv::PageState*> st;
  int rc = check_batch(caches, n_streams, &st);
  if (rc != KV_OK) return rc;
  const pkv::Config& g = st[0]->cfg;
  if (g.D != 64 && g.D != 128) return fail(KV_ERR_UNSUPPORTED, "kv_run_static: head_dim must be 64 or 128");
  if (!aligned16(q) || !aligned16(out)) return fail(KV_ERR_ARG, "kv_run_static: q/out not 16-byte aligned");
  if (block < 0 || block >= g.B) return fail(KV_ERR_ARG, "kv_run_static: block out of range");
  for (int i = 0; i < n_streams; ++i) {
    if (!caches[i]->st.is_appended(block)) return fail(KV_ERR_NOT_APPENDED, "kv_run_static: block not appended in this step");
    if (!caches[i]->dev->bound[block]) return fail(KV_ERR_ARG, "kv_run_static: no pool bound for this block");
  }

  kv_plan_t p;
  pkv::PlanInputs in;
  in.num_sms = device_sms();
  in.ctas_per_sm = pkv::attention_ctas_per_sm(g.D);
  in.tiles_per_split = tiles_per_split;
  in.max_tail_rows = pkv::attention_max_tail_rows(g.D);
  std::string why;
  rc = pkv::build_plan(st, in, &p.hp, &why);
  if (rc != KV_OK) return fail(rc, "kv_run_static: " + why);

  // Packed layout in the array: tables, then the partials of the slots the
  // schedule uses (not the worst case that kv_workspace_bytes provisions).
  size_t n_slots = 0;
  for (const pkv::KvMergeItem& m : p.hp.merges) n_slots = std::max(n_slots, (size_t)m.slot0 + (size_t)m.n);
  const size_t off_o = align256(p.hp.image.size());
  const size_t off_lse = align256(off_o + n_slots * pkv::kTile * (size_t)g.D * 4);
  const size_t need = align256(off_lse + n_slots * pkv::kTile * 4);
  if (need > KV_STATIC_SCRATCH_BYTES)
    return fail(KV_ERR_CAPACITY, "kv_run_static: this call needs " + std::to_string(need) +
                                     " bytes of scratch but the static array holds " +
                                     std::to_string((size_t)KV_STATIC_SCRATCH_BYTES) +
                                     "; use kv_plan/kv_run with a workspace or a larger tiles_per_split");
  pkv::KvPlanHeader& hd = p.hp.header;
  hd.off_part_o = (int64_t)off_o;
  hd.off_part_lse = (int64_t)off_lse;
  std::memcpy(p.hp.image.data(), &hd, sizeof(hd));

  void* scratch = nullptr;
  rc = static_scratch(&scratch);
  if (rc != KV_OK) return rc;
  // Everything but the error word (the header's first word) is uploaded, so
  // the word keeps the bits of earlier calls until a checking call clears it.
  static_assert(offsetof(pkv::KvPlanHeader, error) == 0, "error word first");
  constexpr size_t kW = sizeof(uint32_t);
  cudaError_t e = pkv::upload_plan(static_cast<uint8_t*>(scratch) + kW, p.hp.image.data() + kW,
                                   p.hp.image.size() - kW, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kv_run_static: upload");
  for (int i = 0; i < n_streams; ++i) {
    p.caches.push_back(caches[i]);
    p.epochs.push_back(caches[i]->st.epoch);
    p.total_T += g.page_size + g.NS;
  }
  p.H = g.H;
  p.D = g.D;
  p.dtype = g.dtype;
  p.ws = scratch;
  p.ws_bytes = KV_STATIC_SCRATCH_BYTES;
  rc = kv_run(&p, block, q, out, stream);
  if (rc != KV_OK || !check) return rc;
  e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kv_run_static: synchronize");
  uint32_t w = 0;
  e = cudaMemcpy(&w, scratch, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "kv_run_static: read error word");
  if (w) {
    const uint32_t zero = 0;
    e = cudaMemcpy(scratch, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "kv_run_static: clear error word");
    return fail(KV_ERR_DEVICE_CHECK, "kernel error word " + std::to_string(w));
  }
  return KV_OK;
}
