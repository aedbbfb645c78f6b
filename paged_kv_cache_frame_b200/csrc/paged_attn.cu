// Paged prefill attention for one frame, sm_100a.
//
// For every (request r, head h, query row) the launch computes
//   O = softmax(Q K^T / sqrt(D)) V
// over the K/V tiles of the request's visible page table ([P1] "FlashInfer
// Kernel Execution": the kernel attends only to the listed pages; [P3]
// "Visible Page Table Attention"). A CTA takes one or two consecutive 128-row
// query tiles of one head and a range of K/V tiles; when the range is a chunk
// of a split, it writes chunk-normalised outputs and log2-sum-exp values for
// the merge kernel. ([P1] is "How the Paged KV Cache Attention Mechanism
// Enables Long Sequence Inference in LingBot-Map", [P3] "FlashInfer Paged KV
// Cache Performance Benefits in LingBot-Map".)
//
// Roles. 12 warps (384 threads).
//   warps 0-3, 4-7   softmax warpgroups, one per 128-row query tile. Thread i
//                    owns query row i == TMEM lane i. Per K/V tile it reads its
//                    S row in two 64-column halves, keeps the running max/sum
//                    in the log2 domain, writes P (16-bit) to TMEM, and
//                    rescales its O row when the running max grows by more
//                    than 2^8 (lazy rescale: between rescales P may exceed 1,
//                    which the final division by the same sum cancels).
//   tail             warps 8 and 9: the unit's last query tile of at most 16
//                    rows (262 = 2 x 128 + 6 tokens per frame). An M = 128
//                    tensor-core tile would be almost all padding, so each of
//                    these warps computes the tail's scores and output for 64
//                    of every K/V tile's 128 rows with warp-level mma.sync
//                    m16n8k16, transposed so that the tail rows fill the N = 8
//                    side, reading K and V straight from the shared-memory
//                    ring, with its own running max/sum and O in registers.
//                    The two partial results are merged at the end.
//   producer         warp 10: TMA loads, the query tiles once, then K/V tiles
//                    of the page table into a STAGES-deep ring. A tile is 128
//                    pool rows of one head, one 3-D box load per 64 columns;
//                    the tile table gives each tile's row, so pages need not be
//                    contiguous.
//   MMA issuer       warp 11, also the TMEM allocator (tcgen05 kind::f16, fp32
//                    accumulators in TMEM): S = Q_t K^T (M=128, N=128, K=D) and
//                    O_t += P V (M=128, N=D, K=128, P read from TMEM). The
//                    whole warp runs the loop and one elected lane issues, so
//                    the descriptors stay warp-uniform.
//
// Schedule. Score tiles are numbered n = j * nq + t (K/V tile j, query tile t
// of nq). S_n goes to TMEM buffer n % NB and its P is written over it. NB is 3
// for head_dim 64 with two query tiles (3 x 128 columns and two 64-column O
// tiles fill the 512 columns), else 2. The issuer's order is fixed: S_0 ..
// S_{NB-1}, then PV_n followed by S_{n+NB}. A CTA's MMAs from one thread run
// in issue order, so S_{n+NB} cannot overwrite P_n before PV_n has read it,
// the scores of the next tiles are computed while the softmax works on the
// current one, and the softmax never waits for a PV before it stores P. The
// order gives the two facts the waits below rely on:
//   - once S_n has completed, every PV_m with m <= n - NB has completed; as
//     NB <= 2 nq, the O rescale at K/V tile j (after S_t(j) was read) waits
//     only for PV_t(j-1), because PV_t(j-2) is complete already;
//   - no barrier runs more than one phase ahead of a waiter (each waiter's
//     previous wait covered the phase before), so every parity wait is
//     unambiguous. Per-buffer s_full / p_full barriers carry the phases.
// The launch overlaps the previous kernel on the stream (programmatic
// dependent launch): everything before pdl_wait() is setup that touches no
// data an earlier kernel may still be writing.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include <type_traits>

#include "kernels.h"
#include "launch.cuh"
#include "merge.cuh"
#include "sm100.cuh"

namespace pkv {

constexpr int kMaxSmemTiles = 512;   // tile descriptors cached in shared memory
constexpr int kL2Ahead = 4;          // K/V tiles prefetched into L2 beyond the shared-memory ring
constexpr int kNextAhead = 8;        // first tiles of the unit prefetched for the next block's launch

template <int D>
struct AttnRoles {
  // warps 8 and 9 are the tail (with the softmax warpgroups, three warps on
  // each SM sub-partition), 10 the producer, 11 the MMA issuer and TMEM
  // allocator
  static constexpr int kTailWarps = 2, kTail0 = 8;
  static constexpr int kProducer = 10, kMma = 11;
  static constexpr int kWarps = 12;
  static constexpr int kThreads = 32 * kWarps;
};

template <int D, int STAGES>
struct AttnSmem {
  static constexpr int kTileBytes = kTile * D * 2;   // one 128-row Q, K or V tile
  static constexpr int kQ = 0;                       // two query tiles
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + STAGES * kTileBytes;
  // tail merge: per tail warp [16 rows][D] fp32 outputs, then maxima and sums
  static constexpr int kTW = AttnRoles<D>::kTailWarps;
  static constexpr int kTailO = kV + STAGES * kTileBytes;
  static constexpr int kTailML = kTailO + kTW * 16 * D * 4;
  static constexpr int kTiles = kTailML + 2 * kTW * 16 * 4;
  static constexpr int kBars = kTiles + kMaxSmemTiles * (int)sizeof(KvTile);
  static constexpr int kBytes = kBars + 256;
  static constexpr int kAlloc = kBytes + 1024;      // slack to align the base to 1 KB
};

// TMEM columns: the score buffers (128 columns each, P written over S) from
// column 0, then O_0, O_1. head_dim 64: three buffers, O_t at 384 + 64 t;
// head_dim 128: two, O_t at 256 + 128 t.
template <int D>
struct AttnTmem {
  static constexpr int kMaxBufs = D == 64 ? 3 : 2;
  __host__ __device__ static constexpr uint32_t S(int b) { return 128u * b; }
  __host__ __device__ static constexpr uint32_t O(int t) { return (D == 64 ? 384u : 256u) + (uint32_t)D * t; }
  static_assert((D == 64 ? 384 : 256) + 2 * D <= 512, "TMEM budget");
};

constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
// How long a CTA of a split group waits for the group's other CTAs before it
// leaves its share of the merge to the last one to arrive.
constexpr uint64_t kGroupWaitNs = 50000ull;

// Waits bounded by time only (used to drain in-flight async work on exit).
__device__ __forceinline__ void mbar_drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// Visible columns [base, base + 64) of a K/V tile as a bit mask (bit c for
// column base + c): [lo, hi), and with step > 1 only lo, lo + step, ...
__device__ __forceinline__ uint64_t visible_cols(const KvTile& t, int base) {
  const int lo = max(t.lo - base, 0), hi = min(t.hi - base, 64);
  if (hi <= lo) return 0;
  uint64_t m = (hi == 64 ? ~0ull : (1ull << hi) - 1) & ~((1ull << lo) - 1);
  if (t.step > 1) {
    int c = t.lo - base;
    if (c < 0) c += (-c + t.step - 1) / t.step * t.step;   // first visible column of this half
    uint64_t s = 0;
    for (; c < 64; c += t.step) s |= 1ull << c;
    m &= s;
  }
  return m;
}

template <bool kFP16>
__device__ __forceinline__ uint32_t pack16(float a, float b) {
  return kFP16 ? cvt_pack_f16(a, b) : cvt_pack_bf16(a, b);
}

template <bool kFP16>
__device__ __forceinline__ void unpack16(uint32_t v, float& a, float& b) {
  if (kFP16) {
    const __half2 h = *reinterpret_cast<const __half2*>(&v);
    a = __low2float(h);
    b = __high2float(h);
  } else {
    a = __uint_as_float(v << 16);
    b = __uint_as_float(v & 0xFFFF0000u);
  }
}

// kEmuMask: bit i set = pairs of score columns with (pair index % 8) == i take
// exp2 on the FMA pipe (exp2_poly2) instead of the MUFU unit.
template <int D, bool kFP16, int STAGES, uint32_t kEmuMask>
__global__ void __launch_bounds__(AttnRoles<D>::kThreads, 1)
    paged_prefill_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
  using R = AttnRoles<D>;
  using L = AttnSmem<D, STAGES>;
  using TM = AttnTmem<D>;
  constexpr int kThreads = R::kThreads;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(L::kAlloc <= 227 * 1024, "shared memory per CTA");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_q = bars;
  uint64_t* bar_kv_full = bars + 1;
  uint64_t* bar_kv_empty = bars + 1 + STAGES;
  uint64_t* bar_s_full = bars + 1 + 2 * STAGES;   // [3] S_n computed into buffer n % NB
  uint64_t* bar_p_full = bar_s_full + 3;          // [3] P_n written over it (and O_t rescaled)
  uint64_t* bar_pv_done = bar_s_full + 6;         // [2] PV_t(j) complete
  uint64_t* bar_o_final = bar_s_full + 8;
  uint64_t* bar_drain = bar_s_full + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s_full + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile uint32_t* merge_shares = tmem_slot + 2;   // shares of the split merge this CTA takes
  KvTile* tile_cache = reinterpret_cast<KvTile*>(smem + L::kTiles);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const KvUnit u = a.units[blockIdx.x];
  const KvReq rq = a.reqs[u.req];
  const int n_tiles = u.tile_end - u.tile_begin;
  const int nq = u.nq;
  const int tail_rows = u.tail_rows;
  const bool has_tail = tail_rows > 0;
  const KvTile* tiles_g = a.tiles + u.tile_begin;
  // rotating score buffers: three where two query tiles leave room for them
  const int nb = (TM::kMaxBufs == 3 && nq == 2) ? 3 : 2;
  if (n_tiles <= 0 || nq < 1 || nq > 2 || u.tail_rows < 0 || u.tail_rows > (D == 64 ? kMaxTailRows : 8)) {
    // the planner never emits such a unit
    if (threadIdx.x == 0) atomicOr(a.err, 2u);
    return;
  }

  // Tile descriptors into shared memory (off the softmax's critical path).
  for (int i = threadIdx.x; i < min(n_tiles, kMaxSmemTiles); i += kThreads) tile_cache[i] = tiles_g[i];
  auto tile_at = [&](int j) -> KvTile { return j < kMaxSmemTiles ? tile_cache[j] : tiles_g[j]; };

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      // released by the MMA issuer's commit and, with a tail, by each tail warp
      mbar_init(&bar_kv_empty[s], 1 + (has_tail ? R::kTailWarps : 0));
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&bar_s_full[b], 1);
      mbar_init(&bar_p_full[b], 128);
    }
    for (int t = 0; t < 2; ++t) mbar_init(&bar_pv_done[t], 1);
    mbar_init(bar_o_final, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == R::kMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // The producer's K/V loads, one K/V tile j into ring stage j % STAGES.
  const CUtensorMap* mkv = &maps.kv[u.req];
  auto load_kv = [&](int j) {
    const int s = j % STAGES;
    const KvTile t = tile_at(j);
    // the frame's own tiles from k, v when this launch appends it
    const bool own = a.fused_append && t.krow != kNotCurrent;
    const CUtensorMap* mk = own ? &maps.k : mkv;
    const CUtensorMap* mv = own ? &maps.v : mkv;
    const int rk = own ? rq.q_row0 + t.krow : t.row;
    const int rv = own ? rk : t.row + rq.page_size;
    mbar_arrive_expect_tx(&bar_kv_full[s], 2 * L::kTileBytes);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb) {
      tma_load_3d(smem + L::kK + s * L::kTileBytes + kb * 16384, mk, &bar_kv_full[s], kb * 64, u.head, rk);
      tma_load_3d(smem + L::kV + s * L::kTileBytes + kb * 16384, mv, &bar_kv_full[s], kb * 64, u.head, rv);
    }
  };
  // K/V rows of pool tiles that earlier frames wrote, prefetched into L2
  // kL2Ahead tiles ahead of the ring: a head's tile is 128 rows of 128
  // bytes, 2 KB apart in the pool, and its DRAM latency under load is
  // several ring periods.
  auto prefetch_l2 = [&](int j) {
    if (j >= n_tiles) return;
    const KvTile t = tile_at(j);
    if (t.krow != kNotCurrent) return;   // the frame's own rows: just written, or read from k, v
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb) {
      tma_prefetch_l2_3d(mkv, kb * 64, u.head, t.row);
      tma_prefetch_l2_3d(mkv, kb * 64, u.head, t.row + rq.page_size);
    }
  };
  int j_loaded = 0;   // K/V tiles whose loads the producer has issued (same in every lane)
  if (warp == R::kProducer) {
    if (lane == 0) {
      prefetch_tmap(&maps.q);
      prefetch_tmap(mkv);
      if (a.fused_append) {
        prefetch_tmap(&maps.k);
        prefetch_tmap(&maps.v);
      }
    }
    // Earlier frames' pool rows may be read before the previous kernel on
    // the stream has completed: that kernel is the previous block's launch,
    // its append or the plan upload, and none of them writes those rows (a
    // block's pool is written only by its own appends, stream-ordered long
    // before). The first ring stages are filled with them now; the frame's
    // own tiles, and q, wait.
    for (; j_loaded < min(n_tiles, STAGES) && tile_at(j_loaded).krow == kNotCurrent; ++j_loaded)
      if (lane == 0) load_kv(j_loaded);
    if (lane == 0)
      for (int jj = STAGES; jj < STAGES + kL2Ahead; ++jj) prefetch_l2(jj);
  }
  auto load_q = [&]() {
    mbar_arrive_expect_tx(bar_q, nq * L::kTileBytes);
    for (int t = 0; t < nq; ++t)
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_3d(smem + L::kQ + t * L::kTileBytes + kb * 16384, &maps.q, bar_q, kb * 64, u.head,
                    rq.q_row0 + (u.qtile + t) * kTile);
  };
  // no TMA write may still be in flight when the CTA exits
  auto drain_loads = [&](int j_end) {
    mbar_drain_wait(bar_q, 0);
    for (int jj = (j_end > STAGES ? j_end - STAGES : 0); jj < j_end; ++jj)
      mbar_drain_wait(&bar_kv_full[jj % STAGES], (jj / STAGES) & 1);
  };
  // The setup above overlaps the previous kernel (the frame's K/V append);
  // q, k, v and the frame's own rows are read only after it has completed.
  pdl_wait();

  if (a.fused_append && warp < 8) {
    // ------------------------------------------------- append (scatter)
    // This CTA's slice of every request's k, v rows, copied into the pool in
    // 16-byte vectors ([P1] "Appending New Frames": special tokens 0..NS-1 to
    // the special stream at the frame's offset, which may straddle two
    // pages; patch tokens to the frame's page). No CTA of this launch reads
    // those pool rows: the frame's own tiles come from k, v. The softmax
    // warps do it while the first scores are computed.
    const int T = rq.T, rv = a.row_vecs;
    const long long per_kv = (long long)T * rv, per_req = 2 * per_kv;
    const long long total = per_req * a.n_reqs;
    const long long i0 = total * blockIdx.x / gridDim.x, i1 = total * (blockIdx.x + 1) / gridDim.x;
    // vector i of the flattened [request][K/V][token][row vector] space: its
    // source in k/v and its destination in the pool
    auto locate = [&](long long i, const uint4** src, uint4** dst) {
      const int r = (int)(i / per_req);
      const long long rem = i - (long long)r * per_req;
      const int kv = rem >= per_kv;
      const long long rr = rem - kv * per_kv;
      const int tok = (int)(rr / rv);
      const int c = (int)(rr - (long long)tok * rv);
      const KvReq q = a.reqs[r];
      int page, slot;
      if (tok < q.NS) {
        const int jj = q.cur_sp0 + tok;
        page = q.sp_base + jj / q.page_size;
        slot = jj % q.page_size;
      } else {
        page = q.cur_page;
        slot = tok - q.NS;
      }
      *src = static_cast<const uint4*>(kv ? a.v : a.k) + (long long)(q.q_row0 + tok) * rv + c;
      *dst = static_cast<uint4*>(a.pools[r]) + (((long long)page * 2 + kv) * q.page_size + slot) * rv + c;
    };
    // a batch of loads in flight before their stores (the loop would
    // otherwise wait a full memory round trip per vector)
    constexpr int kBatch = 4;
    for (long long i = i0 + threadIdx.x; i < i1; i += kBatch * 256) {
      uint4 x[kBatch];
      uint4* dst[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const long long ib = i + (long long)b * 256;
        if (ib < i1) {
          const uint4* src;
          locate(ib, &src, &dst[b]);
          x[b] = __ldg(src);
        }
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
        if (i + (long long)b * 256 < i1) *dst[b] = x[b];
    }
  }

  if (warp == R::kProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      load_q();
      int j = j_loaded;
      for (; j < n_tiles; ++j) {
        const int s = j % STAGES;
        if (j >= STAGES && !mbar_wait(&bar_kv_empty[s], ((j / STAGES) - 1) & 1, abort_flag)) break;
        load_kv(j);
        if (j >= STAGES) prefetch_l2(j + kL2Ahead);
      }
      if (a.prefetch_next) {
        // The next block's launch of this plan runs the same units: the
        // first ring of this unit's tiles in its pools (rows of earlier
        // frames) into L2 now, while this CTA still computes.
        const CUtensorMap* mn = &maps.kv_next[u.req];
        for (int jj = 0; jj < min(n_tiles, kNextAhead); ++jj) {
          const KvTile t = tile_at(jj);
          if (t.krow != kNotCurrent) continue;
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb) {
            tma_prefetch_l2_3d(mn, kb * 64, u.head, t.row);
            tma_prefetch_l2_3d(mn, kb * 64, u.head, t.row + rq.page_size);
          }
        }
      }
      drain_loads(j);
    }
  } else if (warp == R::kMma) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issuer's loop (waits included); one elected
    // lane issues each MMA group and its commit.
    {
      // Descriptors are built once and stepped by constant offsets (the start
      // address field counts 16-byte units; shared-memory offsets stay far
      // below its 2^14 range, so the adds never carry out of it).
      constexpr uint32_t idS = umma_idesc_f16(128, 128, kFP16, false);
      constexpr uint32_t idO = umma_idesc_f16(128, D, kFP16, true);
      constexpr uint64_t kStage = L::kTileBytes >> 4;
      const uint64_t dQ = sdesc_sw128(smem_u32(smem + L::kQ), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(smem + L::kK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(smem + L::kV), 16384, 1024);
      // K-major k-step kk (16 elements): +32 bytes inside a 64-column box,
      // +16 KB to the next box
      auto kofs = [](int kk) -> uint64_t { return (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2); };
      auto issue_s = [&](int t, int j, int b) {   // S_n = Q_t K_j^T into buffer b
        const uint64_t k = dK + (j % STAGES) * kStage;
        const uint64_t q = dQ + t * kStage;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_f16_ss(tmem + TM::S(b), q + kofs(kk), k + kofs(kk), idS, kk > 0);
          umma_commit(&bar_s_full[b]);
        }
        __syncwarp();
      };
      auto issue_pv = [&](int t, int j, int b) {   // O_t += P_n V_j, P_n in buffer b
        const uint64_t v = dV + (j % STAGES) * kStage;
        if (elect_one()) {
          umma_f16_ts(tmem + TM::O(t), tmem + TM::S(b), v, idO, j > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < kTile / 16; ++kk)
            umma_f16_ts(tmem + TM::O(t), tmem + TM::S(b) + kk * 8, v + kk * 128, idO, 1u);
          umma_commit(&bar_pv_done[t]);
        }
        __syncwarp();
      };
      auto commit = [&](uint64_t* bar) {
        if (elect_one()) umma_commit(bar);
        __syncwarp();
      };
      // a wait whose outcome is the same in every lane
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
      };
      int kv_ready = -1;   // highest K/V tile whose load was waited for
      auto wait_kv = [&](int j) -> bool {
        if (j <= kv_ready) return true;
        if (!wait(&bar_kv_full[j % STAGES], (j / STAGES) & 1)) return false;
        kv_ready = j;
        return true;
      };
      // Score tile n = j * nq + t goes to buffer n % NB, P over S. The order
      // is fixed: S_0 .. S_{NB-1}, then PV_n followed by S_{n+NB}. S_{n+NB}
      // reuses the buffer PV_n reads, so it cannot go earlier (the tensor
      // pipe runs one thread's MMAs in issue order); PV_n needs P_n; and
      // neither waits for anything later. The issue of an MMA returns about
      // when the tensor pipe takes it and each barrier wait costs a shared-
      // memory round trip, so the issuer simply blocks on the next barrier
      // in that order (polling several candidates only adds latency).
      const int n_all = n_tiles * nq;
      int ns = 0, sj = 0, st = 0, sb = 0;   // next S: number, K/V tile, query tile, buffer
      auto next_s = [&]() -> bool {
        if (!wait_kv(sj)) return false;
        tc_fence_after();
        issue_s(st, sj, sb);
        ++ns;
        if (++st == nq) { st = 0; ++sj; }
        if (++sb == nb) sb = 0;
        return true;
      };
      bool ok = wait(bar_q, 0);
      while (ok && ns < min(nb, n_all)) ok = next_s();
      int pj = 0, pt = 0, pb = 0;   // next PV: K/V tile, query tile, buffer
      uint32_t ppar = 0;            // parity of its p_full phase
      for (int np = 0; ok && np < n_all; ++np) {
        if (!wait(&bar_p_full[pb], ppar)) { ok = false; break; }
        tc_fence_after();
        issue_pv(pt, pj, pb);
        if (++pt == nq) {   // every MMA of K/V tile pj issued
          commit(&bar_kv_empty[pj % STAGES]);
          pt = 0;
          ++pj;
        }
        if (++pb == nb) { pb = 0; ppar ^= 1u; }
        if (ns < n_all) ok = next_s();
      }
      commit(bar_o_final);
      pdl_trigger();   // the merge kernel may be scheduled (it waits for this grid)
      // every MMA of this warp must be complete before TMEM is released
      commit(bar_drain);
      mbar_drain_wait(bar_drain, 0);
    }
  } else if (warp < 8) {
    if ((warp >> 2) < nq) {
      // ---------------------------------------------------------- softmax
      const int t = warp >> 2;
      const int sub = warp & 3;
      const int row = threadIdx.x & 127;
      const int rows_valid = min(kTile, rq.T - (u.qtile + t) * kTile);
      const bool active = sub * 32 < rows_valid;   // warp-uniform
      const uint32_t lane_base = static_cast<uint32_t>(sub * 32) << 16;
      const uint32_t tO = tmem + TM::O(t) + lane_base;
      const float sl2 = a.scale_log2;
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      float m_run = -INFINITY;   // running max of s * log2(e)/sqrt(D), raised lazily
      float l_run = 0.f;         // running sum of 2^(s * sl2 - m_run)
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        // score tile n = j * nq + t in buffer n % NB, its P written over it
        const int n = j * nq + t;
        const int b = n % nb;
        const uint32_t tS = tmem + TM::S(b) + lane_base;
        // Every warp waits, rows or not: p_full counts 128 arrivals a phase.
        // The waits are warp-uniform: tcgen05.ld/st are .sync.aligned.
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_s_full[b], (n / nb) & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        const KvTile tl = tile_at(j);
        const bool masked = tl.lo > 0 || tl.hi < kTile || tl.step > 1;
        float alpha = 1.f;
        bool need = false;
        uint64_t acc[4] = {0, 0, 0, 0};
        uint32_t pa[32];   // P columns 0-63 of this row (16-bit pairs)
        uint32_t r[64];    // the scores of the half being worked on
        auto load_half = [&](int h) {
          tmem_ld_x64_wait(tS + 64 * h, r);
          if (masked) {
            const uint64_t vis = visible_cols(tl, 64 * h);
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (!((vis >> c) & 1)) r[c] = 0xFF800000u;   // -inf
          }
        };
        auto half_max = [&]() -> float {
          float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            mx0 = fmax3(mx0, __uint_as_float(r[c + 0]), __uint_as_float(r[c + 1]));
            mx1 = fmax3(mx1, __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
            mx2 = fmax3(mx2, __uint_as_float(r[c + 4]), __uint_as_float(r[c + 5]));
            mx3 = fmax3(mx3, __uint_as_float(r[c + 6]), __uint_as_float(r[c + 7]));
          }
          return fmax3(mx0, mx1, fmaxf(mx2, mx3)) * sl2;
        };
        // P = 2^(s * sl2 - m_run) in 16-bit pairs into pk, summed in fp32
        // into acc. A half can be fully masked (a short last tile of a
        // page), so the first half may leave m_run at -inf.
        auto exp_half = [&](uint32_t (&pk)[32]) {
          // m_run is -inf only while every column so far was masked: P is 0
          const float mu = m_run == -INFINITY ? 0.f : m_run;
          const uint64_t negm2 = f2_pack(-mu, -mu);
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const uint64_t x = f2_fma(f2_pack(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl2x2, negm2);
            uint64_t e;
            if ((kEmuMask >> ((c >> 1) & 7)) & 1u) {
              e = exp2_poly2(x);
            } else {
              float x0, x1;
              f2_unpack(x, x0, x1);
              e = f2_pack(ex2_approx(x0), ex2_approx(x1));
            }
            acc[(c >> 1) & 3] = f2_add(acc[(c >> 1) & 3], e);
            float e0, e1;
            f2_unpack(e, e0, e1);
            pk[c >> 1] = pack16<kFP16>(e0, e1);
          }
        };
        if (active) {
          load_half(0);
          const float m0 = half_max();
          if (m0 > m_run + kRescaleLog2) {
            alpha = ex2_approx(m_run - m0);   // 0 on the first tile (m_run = -inf)
            l_run *= alpha;
            m_run = m0;
            need = true;
          }
          exp_half(pa);
        }
        if (active) {
          tmem_st_x32(tS, pa);   // P columns 0-31 (16-bit pairs) over S columns 0-31, read
          load_half(1);
          const float m1 = half_max();
          const bool rare = m1 > m_run + kRescaleLog2;
          if (__any_sync(0xffffffffu, rare)) {
            // Rare: the second half raised the max past the threshold after
            // the first half's P was stored. Scale that half (and its sum)
            // down to the new max; the extra rounding stays at the 16-bit
            // level of P. The TMEM accesses are warp-collective, so the
            // whole warp takes this branch; other rows scale by 1 (exact).
            float a2 = 1.f;
            if (rare) {
              a2 = ex2_approx(m_run - m1);
              alpha *= a2;
              l_run *= a2;
              m_run = m1;
              need = true;
            }
            const uint64_t a22 = f2_pack(a2, a2);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = f2_mul(acc[i], a22);
            tmem_wait_st();
            tmem_ld_x32_wait(tS, pa);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float p0, p1;
              unpack16<kFP16>(pa[i], p0, p1);
              pa[i] = pack16<kFP16>(p0 * a2, p1 * a2);
            }
            tmem_st_x32(tS, pa);
          }
          uint32_t pb[32];
          exp_half(pb);
          tmem_st_x32(tS + 32, pb);   // P columns 32-63 over S columns 32-63
          float s0, s1;
          f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), s0, s1);
          l_run += s0 + s1;
          // Rescale O_t if the running max moved. O_t holds PV_t(0..j-1);
          // PV_t(j-2) completed before S_t(j) did (NB <= 2 nq), so the wait
          // for PV_t(j-1) cannot observe an earlier phase of pv_done.
          if (j > 0 && __any_sync(0xffffffffu, need)) {
            if (!__all_sync(0xffffffffu, mbar_wait(&bar_pv_done[t], (j - 1) & 1, abort_flag))) {
              ok = false;
            } else {
              tc_fence_after();
              const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
              for (int c = 0; c < D; c += 16) {
                uint32_t o[16];
                tmem_ld_x16_wait(tO + c, o);
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                  float x0, x1;
                  f2_unpack(f2_mul(f2_pack(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2), x0, x1);
                  o[i] = __float_as_uint(x0);
                  o[i + 1] = __float_as_uint(x1);
                }
                tmem_st_x16(tO + c, o);
              }
            }
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(&bar_p_full[b]);
        if (!ok) break;
      }
      ok = __all_sync(0xffffffffu, ok);
      if (ok && active && __all_sync(0xffffffffu, mbar_wait(bar_o_final, 0, abort_flag))) {
        tc_fence_after();
        const int grow = rq.q_row0 + (u.qtile + t) * kTile + row;
        const bool store = row < rows_valid;
        const float inv = 1.f / l_run;
        const int slot = u.slot[t];
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld_x32_wait(tO + c, o);
          if (!store) continue;
          if (slot < 0) {
            uint16_t* po = reinterpret_cast<uint16_t*>(a.out) + ((size_t)grow * a.H + u.head) * D + c;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 v;
              v.x = pack16<kFP16>(__uint_as_float(o[i + 0]) * inv, __uint_as_float(o[i + 1]) * inv);
              v.y = pack16<kFP16>(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
              v.z = pack16<kFP16>(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
              v.w = pack16<kFP16>(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
              *reinterpret_cast<uint4*>(po + i) = v;
            }
          } else {
            float* po = a.part_o + ((size_t)slot * kTile + row) * D + c;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(po + i) =
                  make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                              __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
          }
        }
        if (store && slot >= 0) a.part_lse[(size_t)slot * kTile + row] = m_run + log2f(l_run);
      }
    }
  } else if (has_tail && warp >= R::kTail0 && warp < R::kTail0 + R::kTailWarps) {
    // ------------------------------------------------------------ tail
    // Tail warp w takes K/V rows [64 w, 64 w + 64) of every tile and works
    // transposed, so the few tail rows sit in the narrow dimension:
    // S^T = K Q_tail^T as 4 m-tiles (16 K/V rows) x D/16 k-steps x NQ n-tiles
    // (8 query rows each) of m16n8k16, an online softmax per query column,
    // then O^T += V^T P^T (D/16 m-tiles of 16 output columns x 4 k-steps x NQ).
    // P^T goes from the accumulator layout to the operand layout with
    // movmatrix. Query rows past the tail are zero and never stored.
    auto tail_body = [&](auto nq_tag) {
      constexpr int NQ = decltype(nq_tag)::value;   // 8-row query groups (1 or 2)
      constexpr int kMT = 4;                         // S^T m-tiles per 64-row half
      constexpr int kDT = D / 16;                    // O^T m-tiles
      const int w = warp - R::kTail0;
      const int g = lane >> 2, q4 = lane & 3;
      const float sl2 = a.scale_log2;
      const int row0 = rq.q_row0 + (u.qtile + nq) * kTile;   // first tail row in q/out
      // B fragments of Q_tail^T: query row 8 n + g, columns 16 k + 2 q4 (+8)
      uint32_t qb[NQ][D / 16][2];
      {
        const uint32_t* qg = reinterpret_cast<const uint32_t*>(a.q);
#pragma unroll
        for (int n = 0; n < NQ; ++n) {
          const bool v = 8 * n + g < tail_rows;
          const size_t rr = ((size_t)(row0 + 8 * n + g) * a.H + u.head) * (D / 2);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            qb[n][k][0] = v ? qg[rr + 8 * k + q4] : 0u;
            qb[n][k][1] = v ? qg[rr + 8 * k + 4 + q4] : 0u;
          }
        }
      }
      float o[kDT][NQ][4];   // O^T: output columns 16 dm + g (+8), query rows 8 n + 2 q4 (+1)
#pragma unroll
      for (int dm = 0; dm < kDT; ++dm)
#pragma unroll
        for (int n = 0; n < NQ; ++n) o[dm][n][0] = o[dm][n][1] = o[dm][n][2] = o[dm][n][3] = 0.f;
      float m_q[NQ][2], l_q[NQ][2];   // per query row 8 n + 2 q4 + e: running max (log2), this lane's sum
#pragma unroll
      for (int n = 0; n < NQ; ++n) m_q[n][0] = m_q[n][1] = -INFINITY, l_q[n][0] = l_q[n][1] = 0.f;
      const uint32_t k_base = smem_u32(smem + L::kK);
      const uint32_t v_base = smem_u32(smem + L::kV);
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % STAGES;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_kv_full[s], (j / STAGES) & 1, abort_flag))) { ok = false; break; }
        const KvTile tl = tile_at(j);
        const uint32_t ks = k_base + s * L::kTileBytes;
        const uint32_t vs = v_base + s * L::kTileBytes;
        const uint64_t vis = visible_cols(tl, 64 * w);   // K/V rows 64 w .. 64 w + 63
        if (vis != 0) {                                    // else nothing visible in this half
          // S^T: m-tile i = K/V rows 64 w + 16 i .. + 15 (accumulator rows g, g + 8).
          // Every A fragment of a group of m-tiles is loaded before its MMAs,
          // so the shared-memory loads overlap one another.
          float sc[kMT][NQ][4];
          constexpr int kSG = D == 64 ? 4 : 2;   // m-tiles per load group
#pragma unroll
          for (int i0 = 0; i0 < kMT; i0 += kSG) {
            uint32_t af[kSG][D / 16][4];
#pragma unroll
            for (int ii = 0; ii < kSG; ++ii) {
              const int kr = 64 * w + 16 * (i0 + ii) + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
              for (int k = 0; k < D / 16; ++k) {
                const int ch = 2 * k + (lane >> 4);
                ldsm_x4(ks + (ch >> 3) * 16384 + kr * 128 + (((ch & 7) ^ (kr & 7)) << 4), af[ii][k]);
              }
            }
#pragma unroll
            for (int ii = 0; ii < kSG; ++ii) {
              const int i = i0 + ii;
#pragma unroll
              for (int n = 0; n < NQ; ++n) sc[i][n][0] = sc[i][n][1] = sc[i][n][2] = sc[i][n][3] = 0.f;
#pragma unroll
              for (int k = 0; k < D / 16; ++k)
#pragma unroll
                for (int n = 0; n < NQ; ++n) mma_16816<kFP16>(sc[i][n], af[ii][k], qb[n][k][0], qb[n][k][1]);
              // mask the K/V rows that are not visible
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                if (!((vis >> (16 * i + g + 8 * h)) & 1))
#pragma unroll
                  for (int n = 0; n < NQ; ++n) sc[i][n][2 * h] = sc[i][n][2 * h + 1] = -INFINITY;
              }
            }
          }
          // per query column: max over these K/V rows (lane values, then
          // the eight lanes with the same q4)
#pragma unroll
          for (int n = 0; n < NQ; ++n) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float mx = -INFINITY;
#pragma unroll
              for (int i = 0; i < kMT; ++i) mx = fmax3(mx, sc[i][n][e], sc[i][n][2 + e]);
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
              mx *= sl2;
              if (mx > m_q[n][e] + kRescaleLog2) {   // never true while every row was masked (-inf)
                const float al = ex2_approx(m_q[n][e] - mx);
                l_q[n][e] *= al;
#pragma unroll
                for (int dm = 0; dm < kDT; ++dm) { o[dm][n][e] *= al; o[dm][n][2 + e] *= al; }
                m_q[n][e] = mx;
              }
            }
          }
          // P^T as B fragments: k-step i = K/V rows 16 i .. + 15 of the half
          // (while every row so far was masked the max is -inf and P is 0)
          uint32_t pb[kMT][NQ][2];
#pragma unroll
          for (int n = 0; n < NQ; ++n) {
            const float m0 = m_q[n][0] == -INFINITY ? 0.f : m_q[n][0];
            const float m1 = m_q[n][1] == -INFINITY ? 0.f : m_q[n][1];
#pragma unroll
            for (int i = 0; i < kMT; ++i) {
              const float p0 = ex2_approx(fmaf(sc[i][n][0], sl2, -m0));
              const float p1 = ex2_approx(fmaf(sc[i][n][1], sl2, -m1));
              const float p2 = ex2_approx(fmaf(sc[i][n][2], sl2, -m0));
              const float p3 = ex2_approx(fmaf(sc[i][n][3], sl2, -m1));
              l_q[n][0] += p0 + p2;
              l_q[n][1] += p1 + p3;
              pb[i][n][0] = movmatrix_t(pack16<kFP16>(p0, p1));
              pb[i][n][1] = movmatrix_t(pack16<kFP16>(p2, p3));
            }
          }
          // O^T += V^T P^T: A fragments by transposed loads of V, a group of
          // output m-tiles loaded before its MMAs
          constexpr int kPG = D == 64 ? 4 : 2;   // output m-tiles per load group
#pragma unroll
          for (int d0 = 0; d0 < kDT; d0 += kPG) {
            uint32_t af[kPG][kMT][4];
#pragma unroll
            for (int dd = 0; dd < kPG; ++dd)
#pragma unroll
              for (int i = 0; i < kMT; ++i) {
                const int vr = 64 * w + 16 * i + (lane & 7) + 8 * (lane >> 4);
                const int ch = 2 * (d0 + dd) + ((lane >> 3) & 1);
                ldsm_x4_t(vs + (ch >> 3) * 16384 + vr * 128 + (((ch & 7) ^ (vr & 7)) << 4), af[dd][i]);
              }
#pragma unroll
            for (int dd = 0; dd < kPG; ++dd)
#pragma unroll
              for (int i = 0; i < kMT; ++i)
#pragma unroll
                for (int n = 0; n < NQ; ++n) mma_16816<kFP16>(o[d0 + dd][n], af[dd][i], pb[i][n][0], pb[i][n][1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_kv_empty[s]);
      }
      // this warp's sums per query row (over the eight lanes that hold it)
#pragma unroll
      for (int n = 0; n < NQ; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = l_q[n][e];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          l_q[n][e] = v;
        }
      constexpr int kTW = R::kTailWarps;
      float* xo = reinterpret_cast<float*>(smem + L::kTailO);    // [kTW][16 query rows][D]
      float* xm = reinterpret_cast<float*>(smem + L::kTailML);   // [kTW][16] maxima, then [kTW][16] sums
#pragma unroll
      for (int dm = 0; dm < kDT; ++dm)
#pragma unroll
        for (int n = 0; n < NQ; ++n)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int qr = 8 * n + 2 * q4 + e;
            xo[(w * 16 + qr) * D + 16 * dm + g] = o[dm][n][e];
            xo[(w * 16 + qr) * D + 16 * dm + g + 8] = o[dm][n][2 + e];
          }
      if (g == 0) {
#pragma unroll
        for (int n = 0; n < NQ; ++n)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            xm[w * 16 + 8 * n + 2 * q4 + e] = m_q[n][e];
            xm[kTW * 16 + w * 16 + 8 * n + 2 * q4 + e] = l_q[n][e];
          }
      }
      named_bar_sync(1, 32 * kTW);
      // (a failed wait in either warp also sets the abort flag, which marks
      // the launch's outputs invalid)
      ok = __all_sync(0xffffffffu, ok);
      // merge: thread i of the tail warps finishes row i / 4, columns (i % 4) D / 4 .. + D / 4 - 1
      constexpr int kCols = D / 4;
      const int i = w * 32 + lane;
      const int r = i >> 2, c0 = (i & 3) * kCols;
      if (ok && r < tail_rows) {
        float mw[kTW], M = -INFINITY;
#pragma unroll
        for (int q = 0; q < kTW; ++q) {
          mw[q] = xm[q * 16 + r];
          M = fmaxf(M, mw[q]);
        }
        float wq[kTW], Lsum = 0.f;
#pragma unroll
        for (int q = 0; q < kTW; ++q) {
          wq[q] = mw[q] == -INFINITY ? 0.f : ex2_approx(mw[q] - M);
          Lsum += wq[q] * xm[kTW * 16 + q * 16 + r];
        }
        const float inv = 1.f / Lsum;
        float res[kCols];
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
          float v = 0.f;
#pragma unroll
          for (int q = 0; q < kTW; ++q) v = fmaf(wq[q], xo[(q * 16 + r) * D + c0 + c], v);
          res[c] = v * inv;
        }
        const int slot = u.slot[nq];
        if (slot < 0) {
          uint16_t* po = reinterpret_cast<uint16_t*>(a.out) + ((size_t)(row0 + r) * a.H + u.head) * D + c0;
#pragma unroll
          for (int c = 0; c < kCols; c += 8) {
            uint4 v;
            v.x = pack16<kFP16>(res[c + 0], res[c + 1]);
            v.y = pack16<kFP16>(res[c + 2], res[c + 3]);
            v.z = pack16<kFP16>(res[c + 4], res[c + 5]);
            v.w = pack16<kFP16>(res[c + 6], res[c + 7]);
            *reinterpret_cast<uint4*>(po + c) = v;
          }
        } else {
          float* po = a.part_o + ((size_t)slot * kTile + r) * D + c0;
#pragma unroll
          for (int c = 0; c < kCols; c += 4)
            *reinterpret_cast<float4*>(po + c) = make_float4(res[c], res[c + 1], res[c + 2], res[c + 3]);
          if (c0 == 0) a.part_lse[(size_t)slot * kTile + r] = M + log2f(Lsum);
        }
      }
    };
    if (tail_rows <= 8)
      tail_body(std::integral_constant<int, 1>{});
    else if (D == 64)   // the planner gives head_dim 128 at most 8 tail rows
      tail_body(std::integral_constant<int, 2>{});
  }

  const bool fuse = a.fused_merge && u.n_chunks > 1;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == R::kMma) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (fuse) {
    // ---------------------------------------------------------- fused merge
    // The n CTAs of a split group (n <= 32) merge it in n shares of its R
    // query rows, CTA k taking rows [k R / n, (k + 1) R / n), once every
    // CTA's partials are written. One 64-bit word per group counts the
    // arrivals (high half) and marks abandoned shares (low half). A CTA that
    // is not the last to arrive waits a short, bounded time for the rest; if
    // the time runs out while the group is still incomplete it abandons its
    // share (a compare-and-swap that fails once the count is n) and leaves.
    // The last to arrive gets every abandoned share with its arrival and
    // merges them with its own. So no CTA depends on another being resident
    // (another kernel may hold SMs), and each share is merged exactly once.
    // The last CTA to leave resets the counters for the next launch.
    unsigned long long* word = reinterpret_cast<unsigned long long*>(a.groups + 4 * u.group);
    uint32_t* departed = a.groups + 4 * u.group + 2;
    const int n = u.n_chunks;
    constexpr unsigned long long kArrive = 1ull << 32;
    if (threadIdx.x == 0) {
      // release: every thread's partials (ordered before this thread by the
      // barrier above) before the arrival
      fence_acq_rel_gpu();
      const unsigned long long old = atomicAdd(word, kArrive);
      uint32_t mine = 1u << u.chunk;
      if ((old >> 32) == (unsigned long long)(n - 1)) {
        fence_acq_rel_gpu();     // acquire: the other CTAs' partials, released by their arrivals
        mine |= (uint32_t)old;   // the last to arrive: its share and every abandoned one
      } else {
        const uint64_t t0 = globaltimer_ns();
        for (;;) {
          const unsigned long long v = ld_acquire_gpu_u64(word);
          if ((v >> 32) >= (unsigned long long)n) break;   // complete: merge the own share
          if (globaltimer_ns() - t0 > kGroupWaitNs) {
            if (atomicCAS(word, v, v | mine) == v) { mine = 0; break; }   // abandoned
            continue;   // the word moved meanwhile: look again
          }
          __nanosleep(64);
        }
      }
      *merge_shares = mine;
    }
    __syncthreads();   // the acquire above, then this barrier, orders every thread's reads below
    uint32_t mine = *merge_shares;
    if (mine) {
      auto rows_of = [&](int t) { return t < nq ? min(kTile, rq.T - (u.qtile + t) * kTile) : tail_rows; };
      const int group_rows = rows_of(0) + (nq > 1 ? rows_of(1) : 0) + tail_rows;
      // A share's rows of every chunk's partials are staged in shared memory
      // (the Q and K/V stages, idle now) by bulk copies that complete on
      // bar_q, whose phase 0 was the Q load. A share of a group of R <= 272
      // rows in n <= 32 chunks has S <= ceil(R / n) rows: S n < R + n rows.
      float* stage = reinterpret_cast<float*>(smem);
      static_assert((2 * kTile + kMaxTailRows + 31) * D * 4 <= L::kTailO, "merge stage fits the Q and K/V stages");
      uint32_t phase = 1;
      for (; mine; mine &= mine - 1) {
        const int k = __ffs(mine) - 1;
        const int r0 = (int)((long long)k * group_rows / n);
        const int r1 = (int)((long long)(k + 1) * group_rows / n);
        const int S = r1 - r0;
        if (threadIdx.x == 0) {
          fence_proxy_async_global();   // the partials acquired above, before the copies read them
          fence_async_smem();           // the stage's earlier reads (before the barrier), before the copies write it
          mbar_arrive_expect_tx(bar_q, (uint32_t)(S * n * D * 4));
          // [r0, r1) by query tile (index nq: the tail), one copy per chunk
          for (int t = 0, gr = 0; t <= nq; gr += rows_of(t), ++t) {
            const int a0 = max(r0, gr), a1 = min(r1, gr + rows_of(t));
            if (a1 <= a0) continue;
            const float* src = a.part_o + ((size_t)(u.slot[t] - u.chunk) * kTile + (a0 - gr)) * D;
            for (int c = 0; c < n; ++c)
              bulk_g2s(stage + ((size_t)c * S + (a0 - r0)) * D, src + (size_t)c * kTile * D,
                       (uint32_t)((a1 - a0) * D * 4), bar_q);
          }
        }
        const bool got = merge_rows_staged<D, kFP16>(
            stage, S, a.part_lse, n, threadIdx.x >> 3, kThreads / 8, threadIdx.x & 7,
            [&]() { return mbar_wait(bar_q, phase & 1u, abort_flag); },
            [&](int i, int* slot0, int* row, uint16_t** out_row) {
              int t = 0, r = r0 + i;
              while (t < nq && r >= rows_of(t)) r -= rows_of(t++);
              const int orow = rq.q_row0 + (u.qtile + t) * kTile + r;
              *slot0 = u.slot[t] - u.chunk;
              *row = r;
              *out_row = reinterpret_cast<uint16_t*>(a.out) + ((size_t)orow * a.H + u.head) * D;
            });
        if (!got) mbar_drain_wait(bar_q, phase & 1u);   // no copy may land after the stage is reused
        __syncthreads();   // the stage is free for the next share's copies
        phase ^= 1u;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && atomicAdd(departed, 1u) == (uint32_t)(n - 1)) {
      atomicExch(word, 0ull);
      atomicExch(departed, 0u);
    }
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(a.err, 1u);
}

// Exponentials on the FMA pipe: pair position 7 of every 8 (12.5 %). The
// softmax is bound by instruction issue more than by the MUFU unit here, and
// the polynomial costs six instructions a pair against two MUFU ones.
constexpr uint32_t kEmu = 0x80u;

template <int D, bool kFP16, int STAGES>
static cudaError_t launch_attn_t(const AttnMaps& maps, const AttnArgs& a, int n_units, cudaStream_t stream) {
  using L = AttnSmem<D, STAGES>;
  auto kern = paged_prefill_attn_kernel<D, kFP16, STAGES, kEmu>;
  static std::atomic<uint8_t> configured[kMaxDevices];   // per device: smem attribute set
  const cudaError_t e = ensure_dynamic_smem(kern, L::kAlloc, configured);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(n_units), dim3(AttnRoles<D>::kThreads), L::kAlloc, stream, maps, a);
}

cudaError_t launch_attention(const AttnMaps& maps, const AttnArgs& a, int D, bool fp16, int n_units,
                             cudaStream_t stream) {
  if (n_units <= 0) return cudaSuccess;
  if (D == 64) return fp16 ? launch_attn_t<64, true, 4>(maps, a, n_units, stream)
                           : launch_attn_t<64, false, 4>(maps, a, n_units, stream);
  if (D == 128) return fp16 ? launch_attn_t<128, true, 2>(maps, a, n_units, stream)
                            : launch_attn_t<128, false, 2>(maps, a, n_units, stream);
  return cudaErrorInvalidValue;
}

int attention_ctas_per_sm(int) { return 1; }

// head_dim 128 keeps tails to one 8-row n-tile: its 16-row form would hold
// 64 fp32 output accumulators per lane and spill at the 168-register cap.
int attention_max_tail_rows(int D) { return D == 64 ? kMaxTailRows : 8; }

}  // namespace pkv
