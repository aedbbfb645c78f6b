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
// Roles (320 threads):
//   warps 0-3, 4-7  softmax warpgroups, one per 128-row query tile. Thread i
//                   owns query row i == TMEM lane i: it loads its 128-column S
//                   row once, keeps the running max/sum in the log2 domain,
//                   writes P (16-bit) to TMEM, rescales its O row when the
//                   running max grows by more than 2^8 (lazy rescale: between
//                   rescales P may exceed 1, which the final division by the
//                   same sum cancels), and runs the epilogue.
//                   With head_dim 64 a query tile of at most 16 rows can ride
//                   along as a tail. Its scores are computed transposed,
//                   S^T = K Q_tail^T (M = 128 K/V rows, N = 16 query rows), and
//                   warpgroup 0 runs its softmax after its own tile's: thread i
//                   then owns K/V row i, the column reductions go through warp
//                   shuffles and shared memory, P^T goes to shared memory and
//                   O^T += V^T P^T is an M = 64, N = 16 MMA.
//   warp 8          TMA producer: the query tiles once, then K/V tiles of the
//                   page table into a STAGES-deep ring. A tile is 128 pool rows
//                   of one head, one 3-D box load per 64 columns; the page table
//                   gives each tile's row, so pages need not be contiguous.
//   warp 9          TMEM allocator and MMA issuer (tcgen05 kind::f16, fp32
//                   accumulators in TMEM): S_t = Q_t K^T (M=128, N=128, K=D),
//                   O_t += P_t V (M=128, N=D, K=128, P read from TMEM) and the
//                   tail's two MMAs.
// TMEM. head_dim 64: S_t at [128 t, +128), one P buffer at [256, 320) that the
// two tiles take in turn, O_t at [320 + 64 t, +64), tail S^T at [448, 464) and
// O^T at [464, 480) (M = 64 layout: row d in lane d % 16 + 32 (d / 16)). P
// has its own columns, so S_t(j+1) is computed as soon as the softmax has
// read S_t(j): the tensor core works on the next tile while the
// exponentials of this one run. head_dim 128: O_t takes [256 + 128 t, +128),
// so P_t is written over the S_t columns it came from, S_t(j+1) waits for
// PV_t(j), and there is no tail.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace pkv {

constexpr int kMaxSmemTiles = 512;   // tile descriptors cached in shared memory

#ifdef PKV_TRACE
// Instrumented builds only: per-tile clock64() stamps of each role of CTA 0,
// read back with kv_debug_trace(). Layout [role 0..5][tile < 64][event < 8].
__device__ unsigned long long g_pkv_trace[6][64][8];
#define PKV_TRACE_AT(role, j, ev) \
  do { if (blockIdx.x == 0 && (j) < 64) g_pkv_trace[role][j][ev] = clock64(); } while (0)
#else
#define PKV_TRACE_AT(role, j, ev) do { } while (0)
#endif

template <int D, int STAGES>
struct AttnSmem {
  static constexpr bool kTail = D == 64;
  static constexpr int kTileBytes = kTile * D * 2;   // one 128-row Q, K or V tile
  static constexpr int kQ = 0;                       // two query tiles
  static constexpr int kQt = 2 * kTileBytes;         // tail query tile (first 16 rows used)
  static constexpr int kK = kQt + (kTail ? kTileBytes : 0);
  static constexpr int kV = kK + STAGES * kTileBytes;
  static constexpr int kPt = kV + STAGES * kTileBytes;   // tail P: [16 rows][128] 16-bit, swizzled
  static constexpr int kTailL = kPt + (kTail ? 4096 : 0); // tail partial sums [128 threads][16]
  static constexpr int kRed = kTailL + (kTail ? 8192 : 0); // tail reductions [3][4 warps][16] + maxima [16]
  static constexpr int kTiles = kRed + (kTail ? 1024 : 0);
  static constexpr int kBars = kTiles + kMaxSmemTiles * 8;
  static constexpr int kBytes = kBars + 256;
  static constexpr int kAlloc = kBytes + 1024;      // slack to align the base to 1 KB
};

template <int D>
struct AttnTmem {
  static constexpr bool kSepP = D == 64;             // P in its own (shared) columns
  __host__ __device__ static constexpr uint32_t S(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t P(int t) { return kSepP ? 256u : 128u * t; }
  __host__ __device__ static constexpr uint32_t O(int t) { return (kSepP ? 320u : 256u) + (uint32_t)D * t; }
  static constexpr uint32_t kSt = 448, kOt = 464;    // tail (head_dim 64 only)
  static_assert((kSepP ? 320 : 256) + 2 * D <= (kSepP ? 448 : 512), "TMEM budget");
};

constexpr int kThreads = 512;
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

// One round of a multi-column warp max: lanes whose `off` bit is set keep the
// upper HALF of their columns and send the lower half to lane ^ off (and the
// other way round), so HALF values remain, each reduced over twice the lanes.
template <int HALF>
__device__ __forceinline__ void halving_max_round(float (&w)[16], int lane, int off) {
  const bool up = (lane & off) != 0;
#pragma unroll
  for (int k = 0; k < HALF; ++k) {
    const float send = up ? w[k] : w[k + HALF];
    const float keep = up ? w[k + HALF] : w[k];
    w[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
  }
}

// kEmuMask: bit i set = pairs of score columns with (pair index % 8) == i take
// exp2 on the FMA pipe (exp2_poly2) instead of the MUFU unit.
template <int D, bool kFP16, int STAGES, uint32_t kEmuMask>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
  using L = AttnSmem<D, STAGES>;
  using TM = AttnTmem<D>;
  constexpr bool kSepP = TM::kSepP;
  constexpr bool kTail = L::kTail;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(kTail == kSepP, "the tail uses the TMEM the shared P buffer frees");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_q = bars;
  uint64_t* bar_kv_full = bars + 1;
  uint64_t* bar_kv_empty = bars + 1 + STAGES;
  uint64_t* bar_s_full = bars + 1 + 2 * STAGES;   // [3] S_t(j) computed (t = 2: tail S^T)
  uint64_t* bar_s_free = bar_s_full + 3;          // [3] S_t(j) read by its softmax
  uint64_t* bar_p_full = bar_s_full + 6;          // [3] P_t(j) written (and O_t rescaled)
  uint64_t* bar_pv_done = bar_s_full + 9;         // [3] PV_t(j) complete
  uint64_t* bar_o_final = bar_s_full + 12;
  uint64_t* bar_drain = bar_s_full + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s_full + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  KvTile* tile_cache = reinterpret_cast<KvTile*>(smem + L::kTiles);

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

  // Tile descriptors into shared memory (off the softmax's critical path);
  // the tail's P buffer starts at zero (its rows past the tail stay zero).
  for (int i = threadIdx.x; i < min(n_tiles, kMaxSmemTiles); i += kThreads) tile_cache[i] = tiles_g[i];
  if (kTail && has_tail)
    for (int i = threadIdx.x; i < 4096 / 16; i += kThreads)
      reinterpret_cast<uint4*>(smem + L::kPt)[i] = make_uint4(0, 0, 0, 0);
  auto tile_at = [&](int j) -> KvTile { return j < kMaxSmemTiles ? tile_cache[j] : tiles_g[j]; };

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
    }
    for (int t = 0; t < 3; ++t) {
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
  if (warp == 13) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  fence_async_smem();   // the zeroed tail P buffer is read by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 12) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const CUtensorMap* mkv = &maps.kv[u.req];
      prefetch_tmap(&maps.q);
      prefetch_tmap(mkv);
      const int nq_load = nq + (has_tail ? 1 : 0);
      mbar_arrive_expect_tx(bar_q, nq_load * L::kTileBytes);
      for (int t = 0; t < nq_load; ++t)
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_3d(smem + (t < nq ? L::kQ + t * L::kTileBytes : L::kQt) + kb * 16384, &maps.q, bar_q, kb * 64,
                      u.head, rq.q_row0 + (u.qtile + t) * kTile);
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
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Descriptors are built once and stepped by constant offsets (the start
      // address field counts 16-byte units; shared-memory offsets stay far
      // below its 2^14 range, so the adds never carry out of it).
      constexpr uint32_t idS = umma_idesc_f16(128, 128, kFP16, false);
      constexpr uint32_t idO = umma_idesc_f16(128, D, kFP16, true);
      constexpr uint32_t idSt = umma_idesc_f16(128, 16, kFP16, false);
      constexpr uint32_t idOt = umma_idesc_f16(64, 16, kFP16, false, true);
      constexpr uint64_t kStage = L::kTileBytes >> 4;
      const uint64_t dQ = sdesc_sw128(smem_u32(smem + L::kQ), 16, 1024);
      const uint64_t dQt = sdesc_sw128(smem_u32(smem + L::kQt), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(smem + L::kK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(smem + L::kV), 16384, 1024);
      const uint64_t dPt = sdesc_sw128(smem_u32(smem + L::kPt), 16, 1024);
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
      auto issue_s = [&](int t, int j) {
        const uint64_t k = dK + (j % STAGES) * kStage;
        if (t < 2) {   // S_t = Q_t K_j^T
          const uint64_t q = dQ + t * kStage;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_f16_ss(tmem + TM::S(t), q + kofs(kk), k + kofs(kk), idS, kk > 0);
        } else {       // S^T = K_j Q_tail^T
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_f16_ss(tmem + TM::kSt, k + kofs(kk), dQt + kofs(kk), idSt, kk > 0);
        }
        umma_commit(&bar_s_full[t]);
      };
      auto issue_pv = [&](int t, int j) {
        const uint64_t v = dV + (j % STAGES) * kStage;
        if (t < 2) {   // O_t += P_t V_j, P_t from TMEM
          umma_f16_ts(tmem + TM::O(t), tmem + TM::P(t), v, idO, j > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < kTile / 16; ++kk)
            umma_f16_ts(tmem + TM::O(t), tmem + TM::P(t) + kk * 8, v + kk * 128, idO, 1u);
        } else {       // O^T += V_j^T P^T (A = V^T: MN-major view of the V tile)
          umma_f16_ss(tmem + TM::kOt, v, dPt, idOt, j > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < kTile / 16; ++kk)
            umma_f16_ss(tmem + TM::kOt, v + kk * 128, dPt + (uint64_t)((kk >> 2) * 128 + (kk & 3) * 2), idOt, 1u);
        }
        if (kSepP) umma_commit(&bar_pv_done[t]);
      };
      const int n_jobs = nq + (has_tail ? 1 : 0);   // query tiles 0, 1 then the tail (slot 2)
      auto job = [&](int k) { return k < nq ? k : 2; };
      bool ok = mbar_wait(bar_q, 0, abort_flag) && wait_kv(0);
      if (ok)
        for (int k = 0; k < n_jobs; ++k) issue_s(job(k), 0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const bool more = j + 1 < n_tiles;
        PKV_TRACE_AT(4, j, 0);
        if (kSepP) {
          // Per query tile (then the tail): the next tile's scores as soon as
          // the softmax has read this tile's, then this tile's PV. Job by
          // job, so PV_0(j) -- which warpgroup 1 waits for before it takes
          // the shared P buffer -- never waits on warpgroup 1.
          for (int k = 0; k < n_jobs; ++k) {
            const int t = job(k);
            if (more) {
              if (!mbar_wait(&bar_s_free[t], j & 1, abort_flag) || !wait_kv(j + 1)) { ok = false; break; }
              PKV_TRACE_AT(4, j, 1 + k);
              tc_fence_after();
              issue_s(t, j + 1);
            }
            if (!mbar_wait(&bar_p_full[t], j & 1, abort_flag)) { ok = false; break; }
            PKV_TRACE_AT(4, j, 4 + k);
            tc_fence_after();
            issue_pv(t, j);
          }
          if (!ok) break;
        } else {
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
        }
        umma_commit(&bar_kv_empty[j % STAGES]);
        PKV_TRACE_AT(4, j, 7);
      }
      umma_commit(bar_o_final);
      // every MMA of this CTA must be complete before TMEM is released
      umma_commit(bar_drain);
      mbar_drain_wait(bar_drain, 0);
    }
  } else if ((warp >> 2) < nq) {
    // ------------------------------------------------------------ softmax
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
    // The shared P buffer is taken in the order P_0(0), P_1(0), P_0(1), ...:
    // before writing P_t(j) wait for the PV that read it last.
    const bool other = nq == 2;
    auto p_buffer_free = [&](int j) -> bool {   // also covers this tile's own PV_t(j-1)
      if (!kSepP) return true;
      uint64_t* bar;
      uint32_t parity;
      if (t == 0) {
        if (j == 0) return true;
        bar = &bar_pv_done[other ? 1 : 0];
        parity = (j - 1) & 1;
      } else {
        bar = &bar_pv_done[0];
        parity = j & 1;
      }
      const bool w = __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
      tc_fence_after();
      return w;
    };
    float m_run = -INFINITY;   // running max of s * log2(e)/sqrt(D), raised lazily
    float l_run = 0.f;         // running sum of 2^(s * sl2 - m_run)
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      // every wait is made warp-uniform: tcgen05.ld/st are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(&bar_s_full[t], j & 1, abort_flag))) { ok = false; break; }
      if (row == 0) PKV_TRACE_AT(t, j, 0);
      tc_fence_after();
      // Pass 1 reads S in two 64-column halves for the row max; pass 2 reads
      // them again for the exponentials and releases S after the second
      // half, so S_t(j+1) overlaps the rest of this tile's work and at most
      // 64 scores are ever live in registers.
      const KvTile tl = tile_at(j);
      const bool masked = tl.lo > 0 || tl.hi < kTile;
      auto load_half = [&](int h, uint32_t (&r)[64]) {
        tmem_ld_x64_wait(tS + 64 * h, r);
        if (masked) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (64 * h + c < tl.lo || 64 * h + c >= tl.hi) r[c] = 0xFF800000u;   // -inf
        }
      };
      float alpha = 1.f;
      bool need = false;
      uint32_t r[64];
      if (active) {
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          load_half(h, r);
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            mx0 = fmax3(mx0, __uint_as_float(r[c + 0]), __uint_as_float(r[c + 1]));
            mx1 = fmax3(mx1, __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
            mx2 = fmax3(mx2, __uint_as_float(r[c + 4]), __uint_as_float(r[c + 5]));
            mx3 = fmax3(mx3, __uint_as_float(r[c + 6]), __uint_as_float(r[c + 7]));
          }
        }
        const float m_cand = fmax3(mx0, mx1, fmaxf(mx2, mx3)) * sl2;
        need = m_cand > m_run + kRescaleLog2;
        if (need) {
          alpha = ex2_approx(m_run - m_cand);   // 0 on the first tile (m_run = -inf)
          l_run *= alpha;
          m_run = m_cand;
        }
      }
      // P = 2^(s * sl2 - m_run) in 16-bit pairs, summed in fp32, per half;
      // the first half is computed before the (shared) P buffer is claimed
      const uint64_t negm2 = f2_pack(-m_run, -m_run);
      uint64_t acc[4] = {0, 0, 0, 0};
      auto exp_half = [&](const uint32_t (&sv)[64], uint32_t (&pk)[32]) {
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
      uint32_t pk[32];
      if (active) {
        load_half(0, r);
        exp_half(r, pk);
      }
      if (row == 0) PKV_TRACE_AT(t, j, 1);
      if (!p_buffer_free(j)) { ok = false; break; }
      if (active) {
        tmem_st_x32(tP, pk);
        load_half(1, r);
      }
      if (kSepP) {   // S_t(j) fully read: the next tile's scores may overwrite it
        tc_fence_before();
        mbar_arrive(&bar_s_free[t]);
      }
      if (active) {
        exp_half(r, pk);
        tmem_st_x32(tP + 32, pk);
        float s0, s1;
        f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), s0, s1);
        l_run += s0 + s1;
        // O_t is idle (PV_t(j-1) done, PV_t(j) waits for p_full): rescale it
        // if the running max moved
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
        tmem_wait_st();
      }
      tc_fence_before();
      if (row == 0) PKV_TRACE_AT(t, j, 2);
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
  } else if ((warp >> 2) == 2) {
    if (kTail && has_tail) {
      // ------------------------------------------------------------ tail softmax
      const int sub = warp & 3;
      const int i = threadIdx.x & 127;   // K/V row of the tile == TMEM lane of S^T
      const int nqt = tail_rows;
      const uint32_t lane_base = static_cast<uint32_t>(sub * 32) << 16;
      const uint32_t tSt = tmem + TM::kSt + lane_base;
      const uint32_t tOt = tmem + TM::kOt + lane_base;
      const float sl2 = a.scale_log2;
      float* red = reinterpret_cast<float*>(smem + L::kRed);   // [2][4][16] maxima, [4][16] sums
      uint8_t* pt = smem + L::kPt + (i >> 6) * 2048 + ((i & 7) << 1);   // P^T[c][i] at pt + c * 128 ^ ...
      const uint32_t chunk = (i & 63) >> 3;
      float m_c[kMaxTailRows], l_c[kMaxTailRows];
#pragma unroll
      for (int c = 0; c < kMaxTailRows; ++c) {
        m_c[c] = -INFINITY;
        l_c[c] = 0.f;
      }
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_s_full[2], j & 1, abort_flag))) { ok = false; break; }
        PKV_TRACE_AT(2, j, 0);
        tc_fence_after();
        uint32_t r[16];
        tmem_ld_x16_wait(tSt, r);
        tc_fence_before();
        mbar_arrive(&bar_s_free[2]);
        const KvTile tl = tile_at(j);
        const bool valid = i >= tl.lo && i < tl.hi;
        float v[kMaxTailRows];
#pragma unroll
        for (int c = 0; c < kMaxTailRows; ++c) v[c] = valid ? __uint_as_float(r[c]) : -INFINITY;
        float* rb = red + (j & 1) * 64;
        {
          // Column maxima over the warp by halving exchanges: after rounds
          // with lane offsets 16, 8, 4, 2 each lane holds one column
          // (c = lane bits 4..1) reduced over 16 lanes; offset 1 finishes it.
          float w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) w[c] = v[c];
          halving_max_round<8>(w, lane, 16);
          halving_max_round<4>(w, lane, 8);
          halving_max_round<2>(w, lane, 4);
          halving_max_round<1>(w, lane, 2);
          w[0] = fmaxf(w[0], __shfl_xor_sync(0xffffffffu, w[0], 1));
          if ((lane & 1) == 0) rb[sub * 16 + (lane >> 1)] = w[0];
        }
        named_bar_sync(1, 128);
        float alpha[kMaxTailRows];
        bool any_need = false;
#pragma unroll
        for (int c = 0; c < kMaxTailRows; ++c) {
          alpha[c] = 1.f;
          if (c < nqt) {
            const float mc = fmaxf(fmaxf(rb[c], rb[16 + c]), fmaxf(rb[32 + c], rb[48 + c])) * sl2;
            if (mc > m_c[c] + kRescaleLog2) {
              alpha[c] = ex2_approx(m_c[c] - mc);
              l_c[c] *= alpha[c];
              m_c[c] = mc;
              any_need = true;
            }
          }
        }
        // O^T(j-1) must be complete before P^T is rewritten and O^T rescaled
        if (j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(&bar_pv_done[2], (j - 1) & 1, abort_flag))) { ok = false; break; }
          tc_fence_after();
        }
        // every thread computed the same maxima, so any_need is uniform
        if (j > 0 && any_need) {
          uint32_t o[16];
          tmem_ld_x16_wait(tOt, o);
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha[c]);
          tmem_st_x16(tOt, o);
          tmem_wait_st();
        }
#pragma unroll
        for (int c = 0; c < kMaxTailRows; ++c) {
          if (c < nqt) {
            const float p = valid ? ex2_approx(fmaf(v[c], sl2, -m_c[c])) : 0.f;
            l_c[c] += p;
            *reinterpret_cast<uint16_t*>(pt + c * 128 + ((chunk ^ (c & 7)) << 4)) =
                static_cast<uint16_t>(pack16<kFP16>(p, 0.f) & 0xFFFFu);
          }
        }
        fence_async_smem();
        tc_fence_before();
        PKV_TRACE_AT(2, j, 1);
        mbar_arrive(&bar_p_full[2]);
      }
      // the row sums: across threads, once
      named_bar_sync(1, 128);
      float* rl = red + 128;
#pragma unroll
      for (int c = 0; c < kMaxTailRows; ++c) {
        if (c < nqt) {
          float w = l_c[c];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
          if (lane == 0) rl[sub * 16 + c] = w;
        }
      }
      named_bar_sync(1, 128);
      ok = __all_sync(0xffffffffu, ok);
      if (ok && __all_sync(0xffffffffu, mbar_wait(bar_o_final, 0, abort_flag))) {
        tc_fence_after();
        uint32_t o[16];
        tmem_ld_x16_wait(tOt, o);
        const int slot = u.slot[nq];
        const int d = sub * 16 + lane;   // O^T row held by this lane (M = 64 layout)
        const int row0 = (u.qtile + nq) * kTile;
        if (lane < 16) {
#pragma unroll
          for (int c = 0; c < kMaxTailRows; ++c) {
            if (c < nqt) {
              const float l = rl[c] + rl[16 + c] + rl[32 + c] + rl[48 + c];
              const float x = __uint_as_float(o[c]) / l;
              if (slot < 0) {
                reinterpret_cast<uint16_t*>(a.out)[((size_t)(rq.q_row0 + row0 + c) * a.H + u.head) * D + d] =
                    static_cast<uint16_t>(pack16<kFP16>(x, 0.f) & 0xFFFFu);
              } else {
                a.part_o[((size_t)slot * kTile + c) * D + d] = x;
                if (d == 0) a.part_lse[(size_t)slot * kTile + c] = m_c[c] + log2f(l);
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 13) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(a.err, 1u);
}

// Exponentials on the FMA pipe: pair positions {5, 6, 7} of every 8 (37.5 %).
constexpr uint32_t kEmu = 0xE0u;

template <int D, bool kFP16, int STAGES>
static cudaError_t launch_attn_t(const AttnMaps& maps, const AttnArgs& a, int n_units, cudaStream_t stream) {
  using L = AttnSmem<D, STAGES>;
  auto kern = paged_prefill_attn_kernel<D, kFP16, STAGES, kEmu>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  kern<<<n_units, kThreads, L::kAlloc, stream>>>(maps, a);
  return cudaGetLastError();
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
#endif

}  // namespace pkv
