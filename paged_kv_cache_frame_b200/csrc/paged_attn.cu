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
// Roles. head_dim 64: 12 warps (384 threads); head_dim 128: 10 warps (320).
//   warps 0-3, 4-7   softmax warpgroups, one per 128-row query tile. Thread i
//                    owns query row i == TMEM lane i. Per K/V tile it reads its
//                    S row in two 64-column halves, keeps the running max/sum
//                    in the log2 domain, writes P (16-bit) to TMEM -- the first
//                    half as soon as the previous PV has read P, so its store
//                    overlaps the second half -- and rescales its O row when
//                    the running max grows by more than 2^8 (lazy rescale:
//                    between rescales P may exceed 1, which the final division
//                    by the same sum cancels).
//   producer         warp 9 (head_dim 64) / 8 (head_dim 128): TMA loads, the
//                    query tiles once, then K/V tiles of the page table into a
//                    STAGES-deep ring. A tile is 128 pool rows of one head, one
//                    3-D box load per 64 columns; the tile table gives each
//                    tile's row, so pages need not be contiguous.
//   MMA issuer       warp 11 / 9, also the TMEM allocator (tcgen05 kind::f16,
//                    fp32 accumulators in TMEM): S_t = Q_t K^T (M=128, N=128,
//                    K=D) and O_t += P_t V (M=128, N=D, K=128, P read from
//                    TMEM). Each query tile advances on its own, scores first.
//   tail             warps 8 and 10 (head_dim 64): the unit's last query tile
//                    of at most 16 rows (262 = 2 x 128 + 6 tokens per frame).
//                    An M = 128 tensor-core tile would be almost all padding,
//                    so each of these warps computes the tail's scores and
//                    output for 64 of every K/V tile's 128 rows with warp-level
//                    mma.sync m16n8k16, transposed so that the tail rows fill
//                    the N = 8 side, reading K and V straight from the
//                    shared-memory ring, with its own running max/sum and O in
//                    registers. The two partial results are merged at the end.
// TMEM. head_dim 64: S_t at [128 t, +128), P_t at [256 + 64 t, +64), O_t at
// [384 + 64 t, +64). P has its own columns, so the tensor core computes
// S_t(j+1) as soon as the softmax has read S_t(j), while the exponentials of
// tile j run. head_dim 128: O_t takes [256 + 128 t, +128), so P_t is written
// over the S_t columns it came from and S_t(j+1) follows PV_t(j).
// The launch overlaps the previous kernel on the stream (programmatic
// dependent launch): everything before pdl_wait() is setup that touches no
// data an earlier kernel may still be writing.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include <type_traits>

#include "kernels.h"
#include "launch.cuh"
#include "sm100.cuh"

namespace pkv {

constexpr int kMaxSmemTiles = 512;   // tile descriptors cached in shared memory

#ifdef PKV_TRACE
// Instrumented builds only: per-tile clock64() stamps of each role of CTA 0,
// read back with kv_debug_trace(). Layout [role 0..5][tile < 64][event < 8].
__device__ unsigned long long g_pkv_trace[6][64][8];
// per CTA: globaltimer at entry, after the prologue, at exit; and its SM
__device__ unsigned long long g_pkv_cta[1024][6];
#define PKV_TRACE_AT(role, j, ev) \
  do { if (blockIdx.x == 0 && (j) < 64) g_pkv_trace[role][j][ev] = clock64(); } while (0)
#define PKV_CTA_AT(ev) \
  do { if (threadIdx.x == 0 && blockIdx.x < 1024) { \
         g_pkv_cta[blockIdx.x][ev] = globaltimer_ns(); \
         if ((ev) != 1) g_pkv_cta[blockIdx.x][4 + (ev) / 2] = clock64(); } } while (0)
#else
#define PKV_TRACE_AT(role, j, ev) do { } while (0)
#define PKV_CTA_AT(ev) do { } while (0)
#endif

template <int D>
struct AttnRoles {
  static constexpr bool kTail = D == 64;
  // head_dim 64: warps 8 and 10 are the tail (with the softmax warpgroups,
  // three warps per SM sub-partition), 9 the producer, 11 the MMA issuer
  static constexpr int kTailWarps = 2;   // each takes 64 of a K/V tile's 128 columns
  static constexpr int kProducer = kTail ? 9 : 8, kMma = kTail ? 11 : 9;
  static constexpr int kWarps = kTail ? 12 : 10;
  static constexpr int kThreads = 32 * kWarps;
};

template <int D, int STAGES>
struct AttnSmem {
  static constexpr bool kTail = AttnRoles<D>::kTail;
  static constexpr int kTileBytes = kTile * D * 2;   // one 128-row Q, K or V tile
  static constexpr int kQ = 0;                       // two query tiles
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + STAGES * kTileBytes;
  // tail merge: per tail warp [16 rows][D] fp32 outputs, then maxima and sums
  static constexpr int kTW = AttnRoles<D>::kTailWarps;
  static constexpr int kTailO = kV + STAGES * kTileBytes;
  static constexpr int kTailML = kTailO + (kTail ? kTW * 16 * D * 4 : 0);
  static constexpr int kTiles = kTailML + (kTail ? 2 * kTW * 16 * 4 : 0);
  static constexpr int kBars = kTiles + kMaxSmemTiles * 8;
  static constexpr int kBytes = kBars + 256;
  static constexpr int kAlloc = kBytes + 1024;      // slack to align the base to 1 KB
};

template <int D>
struct AttnTmem {
  static constexpr bool kSepP = D == 64;             // P in its own columns
  __host__ __device__ static constexpr uint32_t S(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t P(int t) { return kSepP ? 256u + 64u * t : 128u * t; }
  __host__ __device__ static constexpr uint32_t O(int t) { return (kSepP ? 384u : 256u) + (uint32_t)D * t; }
  static_assert((kSepP ? 384 : 256) + 2 * D <= 512, "TMEM budget");
};

constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

// Waits bounded by time only (used to drain in-flight async work on exit).
__device__ __forceinline__ void mbar_drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
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
  constexpr bool kSepP = TM::kSepP;
  constexpr bool kTail = R::kTail;
  constexpr int kThreads = R::kThreads;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_q = bars;
  uint64_t* bar_kv_full = bars + 1;
  uint64_t* bar_kv_empty = bars + 1 + STAGES;
  uint64_t* bar_s_full = bars + 1 + 2 * STAGES;   // [2] S_t(j) computed
  uint64_t* bar_s_free = bar_s_full + 2;          // [2] S_t(j) read by its softmax
  uint64_t* bar_p_full = bar_s_full + 4;          // [2] P_t(j) written (and O_t rescaled)
  uint64_t* bar_pv_done = bar_s_full + 6;         // [2] PV_t(j) complete
  uint64_t* bar_o_final = bar_s_full + 8;
  uint64_t* bar_drain = bar_s_full + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s_full + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  KvTile* tile_cache = reinterpret_cast<KvTile*>(smem + L::kTiles);

  PKV_CTA_AT(0);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const KvUnit u = a.units[blockIdx.x];
  const KvReq rq = a.reqs[u.req];
  const int n_tiles = u.tile_end - u.tile_begin;
  const int nq = u.nq;
  const int tail_rows = kTail ? u.tail_rows : 0;
  const bool has_tail = tail_rows > 0;
  const KvTile* tiles_g = a.tiles + u.tile_begin;
  if (n_tiles <= 0 || nq < 1 || nq > 2 || u.tail_rows < 0 || u.tail_rows > kMaxTailRows ||
      (!kTail && u.tail_rows != 0)) {   // the planner never emits such a unit
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
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar_s_full[t], 1);
      mbar_init(&bar_s_free[t], 128);
      mbar_init(&bar_p_full[t], 128);
      mbar_init(&bar_pv_done[t], 1);
    }
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
  // The setup above overlaps the previous kernel (the frame's K/V append);
  // the pool and q are read only after it has completed.
  pdl_wait();
  PKV_CTA_AT(1);

  if (warp == R::kProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const CUtensorMap* mkv = &maps.kv[u.req];
      prefetch_tmap(&maps.q);
      prefetch_tmap(mkv);
      mbar_arrive_expect_tx(bar_q, nq * L::kTileBytes);
      for (int t = 0; t < nq; ++t)
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_3d(smem + L::kQ + t * L::kTileBytes + kb * 16384, &maps.q, bar_q, kb * 64, u.head,
                      rq.q_row0 + (u.qtile + t) * kTile);
      int j = 0;
      for (; j < n_tiles; ++j) {
        const int s = j % STAGES;
        if (j >= STAGES && !mbar_wait(&bar_kv_empty[s], ((j / STAGES) - 1) & 1, abort_flag)) break;
        PKV_TRACE_AT(5, j, 0);
        const KvTile t = tile_at(j);
        mbar_arrive_expect_tx(&bar_kv_full[s], 2 * L::kTileBytes);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          tma_load_3d(smem + L::kK + s * L::kTileBytes + kb * 16384, mkv, &bar_kv_full[s], kb * 64, u.head,
                      t.row);
          tma_load_3d(smem + L::kV + s * L::kTileBytes + kb * 16384, mkv, &bar_kv_full[s], kb * 64, u.head,
                      t.row + rq.page_size);
        }
      }
      // no TMA write may still be in flight when the CTA exits
      mbar_drain_wait(bar_q, 0);
      for (int jj = (j > STAGES ? j - STAGES : 0); jj < j; ++jj)
        mbar_drain_wait(&bar_kv_full[jj % STAGES], (jj / STAGES) & 1);
    }
  } else if (warp == R::kMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Descriptors are built once and stepped by constant offsets (the start
      // address field counts 16-byte units; shared-memory offsets stay far
      // below its 2^14 range, so the adds never carry out of it).
      constexpr uint32_t idS = umma_idesc_f16(128, 128, kFP16, false);
      constexpr uint32_t idO = umma_idesc_f16(128, D, kFP16, true);
      constexpr uint64_t kStage = L::kTileBytes >> 4;
      const uint64_t dQ = sdesc_sw128(smem_u32(smem + L::kQ), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(smem + L::kK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(smem + L::kV), 16384, 1024);
      int kv_ready = -1;   // highest K/V tile whose load was waited for
      auto wait_kv = [&](int j) -> bool {
        if (j <= kv_ready) return true;
        if (!mbar_wait(&bar_kv_full[j % STAGES], (j / STAGES) & 1, abort_flag)) return false;
        tc_fence_after();
        kv_ready = j;
        return true;
      };
      // K-major k-step kk (16 elements): +32 bytes inside a 64-column box,
      // +16 KB to the next box
      auto kofs = [](int kk) -> uint64_t { return (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2); };
      auto issue_s = [&](int t, int j) {   // S_t = Q_t K_j^T
        const uint64_t k = dK + (j % STAGES) * kStage;
        const uint64_t q = dQ + t * kStage;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16_ss(tmem + TM::S(t), q + kofs(kk), k + kofs(kk), idS, kk > 0);
        umma_commit(&bar_s_full[t]);
      };
      auto issue_pv = [&](int t, int j) {   // O_t += P_t V_j, P_t from TMEM
        const uint64_t v = dV + (j % STAGES) * kStage;
        umma_f16_ts(tmem + TM::O(t), tmem + TM::P(t), v, idO, j > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < kTile / 16; ++kk)
          umma_f16_ts(tmem + TM::O(t), tmem + TM::P(t) + kk * 8, v + kk * 128, idO, 1u);
        if (kSepP) umma_commit(&bar_pv_done[t]);
      };
      bool ok = mbar_wait(bar_q, 0, abort_flag) && wait_kv(0);
      if (ok)
        for (int t = 0; t < nq; ++t) issue_s(t, 0);
      if (kSepP) {
        // Each query tile advances on its own: S_t(j) once softmax t has read
        // S_t(j-1) and K(j) has landed, PV_t(j) once P_t(j) is written. The
        // scores come first (the softmax waits on them); a K/V stage is
        // released once every MMA that reads it has been issued. Non-blocking
        // polls under one bounded wait.
        int ns[2] = {1, 1};   // next S_t to issue
        int np[2] = {0, 0};   // next PV_t to issue
        if (nq < 2) ns[1] = np[1] = n_tiles;
        int ne = 0;           // next K/V stage release
        uint64_t t0 = globaltimer_ns();
        for (uint32_t spin = 1; ok && ne < n_tiles; ++spin) {
          bool progress = false;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int j = ns[t];
            if (j < n_tiles && mbar_test_wait(&bar_s_free[t], (j - 1) & 1)) {
              if (j > kv_ready) {
                if (!mbar_test_wait(&bar_kv_full[j % STAGES], (j / STAGES) & 1)) continue;
                kv_ready = j;
              }
              PKV_TRACE_AT(4, j - 1, 1 + t);
              tc_fence_after();
              issue_s(t, j);
              ns[t] = j + 1;
              progress = true;
            }
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int j = np[t];
            if (j < n_tiles && mbar_test_wait(&bar_p_full[t], j & 1)) {
              PKV_TRACE_AT(4, j, 4 + t);
              tc_fence_after();
              issue_pv(t, j);
              np[t] = j + 1;
              progress = true;
            }
          }
          while (ne < min(np[0], np[1])) {   // PV_t(ne) issued for every t (and so S_t(ne))
            umma_commit(&bar_kv_empty[ne % STAGES]);
            PKV_TRACE_AT(4, ne, 7);
            ++ne;
            progress = true;
          }
          if (progress) {
            t0 = globaltimer_ns();
          } else {
            // back off: this warp shares its SM sub-partition with two
            // softmax warps, whose issue slots a tight poll would take
            __nanosleep(32);
            if ((spin & 15u) == 0 && (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs)) {
              *abort_flag = 1;
              ok = false;
            }
          }
        }
      } else {
        for (int j = 0; ok && j < n_tiles; ++j) {
          const bool more = j + 1 < n_tiles;
          PKV_TRACE_AT(4, j, 0);
          // P_t(j) sits in the S_t columns: S_t(j+1) follows PV_t(j)
          for (int t = 0; t < nq; ++t) {
            if (!mbar_wait(&bar_p_full[t], j & 1, abort_flag)) { ok = false; break; }
            PKV_TRACE_AT(4, j, 4 + t);
            tc_fence_after();
            issue_pv(t, j);
            if (more) {
              if (!wait_kv(j + 1)) { ok = false; break; }
              issue_s(t, j + 1);
            }
          }
          if (!ok) break;
          umma_commit(&bar_kv_empty[j % STAGES]);
          PKV_TRACE_AT(4, j, 7);
        }
      }
      umma_commit(bar_o_final);
      pdl_trigger();   // the merge kernel may be scheduled (it waits for this grid)
      // every MMA of this CTA must be complete before TMEM is released
      umma_commit(bar_drain);
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
      const uint32_t tS = tmem + TM::S(t) + lane_base;
      const uint32_t tP = tmem + TM::P(t) + lane_base;
      const uint32_t tO = tmem + TM::O(t) + lane_base;
      const float sl2 = a.scale_log2;
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      float m_run = -INFINITY;   // running max of s * log2(e)/sqrt(D), raised lazily
      float l_run = 0.f;         // running sum of 2^(s * sl2 - m_run)
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        // every wait is made warp-uniform: tcgen05.ld/st are .sync.aligned
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_s_full[t], j & 1, abort_flag))) { ok = false; break; }
        if (row == 0) PKV_TRACE_AT(t, j, 0);
        tc_fence_after();
        const KvTile tl = tile_at(j);
        const bool masked = tl.lo > 0 || tl.hi < kTile;
        float alpha = 1.f;
        bool need = false;
        uint32_t pa[32], pb[32];   // this row of P_t(j): columns 0-63, 64-127 as 16-bit pairs
        uint64_t acc[4] = {0, 0, 0, 0};
        auto load_half = [&](int h, uint32_t (&r)[64]) {
          tmem_ld_x64_wait(tS + 64 * h, r);
          if (masked) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (64 * h + c < tl.lo || 64 * h + c >= tl.hi) r[c] = 0xFF800000u;   // -inf
          }
        };
        auto half_max = [&](const uint32_t (&r)[64]) -> float {
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
        // P = 2^(s * sl2 - m_run) in 16-bit pairs into pk, summed
        // in fp32 into acc. A half can be fully masked (a short last tile of a
        // page), so the first half may leave m_run at -inf.
        auto exp_half = [&](const uint32_t (&sv)[64], uint32_t (&pk)[32]) {
          // m_run is -inf only while every column so far was masked: P is 0
          const float mu = m_run == -INFINITY ? 0.f : m_run;
          const uint64_t negm2 = f2_pack(-mu, -mu);
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2, negm2);
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
          uint32_t r[64];
          load_half(0, r);
          if (row == 0) PKV_TRACE_AT(t, j, 3);
          const float m0 = half_max(r);
          if (m0 > m_run + kRescaleLog2) {
            alpha = ex2_approx(m_run - m0);   // 0 on the first tile (m_run = -inf)
            l_run *= alpha;
            m_run = m0;
            need = true;
          }
          exp_half(r, pa);
        }
        if (row == 0) PKV_TRACE_AT(t, j, 1);
        // P_t's columns and O_t are free once PV_t(j-1) is complete; the
        // first half of P goes out now, so its store overlaps the second half
        if (kSepP && j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(&bar_pv_done[t], (j - 1) & 1, abort_flag))) { ok = false; break; }
          tc_fence_after();
        }
        if (row == 0) PKV_TRACE_AT(t, j, 4);
        if (active) {
          if (kSepP) tmem_st_x32(tP, pa);
          uint32_t r[64];
          load_half(1, r);
          if (row == 0) PKV_TRACE_AT(t, j, 5);
          const float m1 = half_max(r);
          const bool rare = m1 > m_run + kRescaleLog2;
          if (__any_sync(0xffffffffu, rare)) {
            // Rare: the second half raised the max past the threshold after
            // the first half's P was formed. Scale that half (and its sum)
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
            if (kSepP) {
              tmem_wait_st();
              tmem_ld_x32_wait(tP, pa);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              float p0, p1;
              unpack16<kFP16>(pa[i], p0, p1);
              pa[i] = pack16<kFP16>(p0 * a2, p1 * a2);
            }
            if (kSepP) tmem_st_x32(tP, pa);
          }
          if (kSepP) {   // S_t(j) fully read: the next tile's scores may overwrite it
            tc_fence_before();
            mbar_arrive(&bar_s_free[t]);
          }
          exp_half(r, pb);
          float s0, s1;
          f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), s0, s1);
          l_run += s0 + s1;
          if (!kSepP) tmem_st_x32(tP, pa);   // over S_t, now read
          tmem_st_x32(tP + 32, pb);
          // rescale O_t if the running max moved
          if (j > 0 && __any_sync(0xffffffffu, need)) {
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
          if (row == 0) PKV_TRACE_AT(t, j, 6);
          tmem_wait_st();
        } else if (kSepP) {
          mbar_arrive(&bar_s_free[t]);
        }
        tc_fence_before();
        if (row == 0) PKV_TRACE_AT(t, j, 2);
        if ((row & 31) == 0) PKV_TRACE_AT(3, j, 4 * t + (row >> 5));   // each warp's arrival
        mbar_arrive(&bar_p_full[t]);
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
          uint32_t r[32];
          tmem_ld_x32_wait(tO + c, r);
          if (!store) continue;
          if (slot < 0) {
            uint16_t* o = reinterpret_cast<uint16_t*>(a.out) + ((size_t)grow * a.H + u.head) * D + c;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 v;
              v.x = pack16<kFP16>(__uint_as_float(r[i + 0]) * inv, __uint_as_float(r[i + 1]) * inv);
              v.y = pack16<kFP16>(__uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
              v.z = pack16<kFP16>(__uint_as_float(r[i + 4]) * inv, __uint_as_float(r[i + 5]) * inv);
              v.w = pack16<kFP16>(__uint_as_float(r[i + 6]) * inv, __uint_as_float(r[i + 7]) * inv);
              *reinterpret_cast<uint4*>(o + i) = v;
            }
          } else {
            float* po = a.part_o + ((size_t)slot * kTile + row) * D + c;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(po + i) =
                  make_float4(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv,
                              __uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
          }
        }
        if (store && slot >= 0) a.part_lse[(size_t)slot * kTile + row] = m_run + log2f(l_run);
      }
    }
  } else if (kTail && has_tail && (warp == 8 || warp == 10)) {
    // ------------------------------------------------------------ tail
    // Tail warp w takes K/V rows [64 w, 64 w + 64) of every tile and works
    // transposed, so the few tail rows sit in the narrow dimension:
    // S^T = K Q_tail^T as 4 m-tiles (16 K/V rows) x 4 k-steps x NQ n-tiles
    // (8 query rows each) of m16n8k16, softmax per query column, then
    // O^T += V^T P^T (4 m-tiles of 16 output columns x 4 k-steps x NQ). P^T
    // goes from the accumulator layout to the operand layout with movmatrix.
    // Query rows past the tail are zero and never stored.
    auto tail_body = [&](auto nq_tag) {
      constexpr int NQ = decltype(nq_tag)::value;   // 8-row query groups (1 or 2)
      constexpr int kCW = kTile / R::kTailWarps;     // K/V rows per tail warp (64)
      constexpr int kMT = kCW / 16;                  // S^T m-tiles
      constexpr int kDT = D / 16;                    // O^T m-tiles
      const int w = (warp - 8) >> 1;
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
        PKV_TRACE_AT(2, j, 0);
        const KvTile tl = tile_at(j);
        const uint32_t ks = k_base + s * L::kTileBytes;
        const uint32_t vs = v_base + s * L::kTileBytes;
        // S^T: m-tile i = K/V rows kCW w + 16 i .. + 15 (accumulator rows g, g + 8)
        float sc[kMT][NQ][4];
#pragma unroll
        for (int i = 0; i < kMT; ++i) {
#pragma unroll
          for (int n = 0; n < NQ; ++n) sc[i][n][0] = sc[i][n][1] = sc[i][n][2] = sc[i][n][3] = 0.f;
          const int kr = kCW * w + 16 * i + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const int ch = 2 * k + (lane >> 4);
            uint32_t af[4];
            ldsm_x4(ks + (ch >> 3) * 16384 + kr * 128 + (((ch & 7) ^ (kr & 7)) << 4), af);
#pragma unroll
            for (int n = 0; n < NQ; ++n) mma_16816<kFP16>(sc[i][n], af, qb[n][k][0], qb[n][k][1]);
          }
          // mask K/V rows outside [lo, hi)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int kvr = kCW * w + 16 * i + g + 8 * h;
            if (kvr < tl.lo || kvr >= tl.hi)
#pragma unroll
              for (int n = 0; n < NQ; ++n) sc[i][n][2 * h] = sc[i][n][2 * h + 1] = -INFINITY;
          }
        }
        // per query column: max over this warp's K/V rows (lane values, then
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
        // P^T as B fragments: k-step i = K/V rows 16 i .. + 15 of this warp's
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
        // O^T += V^T P^T: A fragments by transposed loads of V
#pragma unroll
        for (int dm = 0; dm < kDT; ++dm) {
#pragma unroll
          for (int i = 0; i < kMT; ++i) {
            const int vr = kCW * w + 16 * i + (lane & 7) + 8 * (lane >> 4);
            const int ch = 2 * dm + ((lane >> 3) & 1);
            uint32_t af[4];
            ldsm_x4_t(vs + (ch >> 3) * 16384 + vr * 128 + (((ch & 7) ^ (vr & 7)) << 4), af);
#pragma unroll
            for (int n = 0; n < NQ; ++n) mma_16816<kFP16>(o[dm][n], af, pb[i][n][0], pb[i][n][1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_kv_empty[s]);
        PKV_TRACE_AT(2, j, 1);
      }
      // this warp's sums per query row
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
      ok = __all_sync(0xffffffffu, ok);
      // merge: thread i of the tail warps finishes row i / 4, columns 16 (i % 4) .. + 15
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
    else
      tail_body(std::integral_constant<int, 2>{});
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == R::kMma) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(a.err, 1u);
#ifdef PKV_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 1024) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    g_pkv_cta[blockIdx.x][3] = smid;
  }
#endif
  PKV_CTA_AT(2);
}

// Exponentials on the FMA pipe: pair positions {6, 7} of every 8 (25 %).
constexpr uint32_t kEmu = 0xC0u;

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

bool attention_tail_ok(int D) { return D == 64; }

#ifdef PKV_TRACE
extern "C" int kv_debug_trace(void* host, size_t bytes) {
  if (bytes < sizeof(g_pkv_trace)) return -1;
  return cudaMemcpyFromSymbol(host, g_pkv_trace, sizeof(g_pkv_trace)) == cudaSuccess ? 0 : -7;
}
extern "C" int kv_debug_cta(void* host, size_t bytes) {
  if (bytes < sizeof(g_pkv_cta)) return -1;
  return cudaMemcpyFromSymbol(host, g_pkv_cta, sizeof(g_pkv_cta)) == cudaSuccess ? 0 : -7;
}
#endif

}  // namespace pkv
