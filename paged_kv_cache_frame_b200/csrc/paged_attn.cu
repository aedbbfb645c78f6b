// Paged prefill attention for one frame, sm_100a.
//
// For every (request r, head h, 128-row query tile) the CTA computes
//   O = softmax(Q K^T / sqrt(D)) V
// over the K/V tiles of the request's visible page table ([P1] "FlashInfer
// Kernel Execution": the kernel attends only to the listed pages; [P3]
// "Visible Page Table Attention"). A CTA may own only a chunk of the tiles
// (split-KV); it then writes its chunk-normalised output and log2-sum-exp for
// the merge kernel. ([P1] is "How the Paged KV Cache Attention Mechanism
// Enables Long Sequence Inference in LingBot-Map", [P3] "FlashInfer Paged KV
// Cache Performance Benefits in LingBot-Map".)
//
// Roles (192 threads):
//   warps 0-3  softmax: thread i owns query row i == TMEM lane i. Loads S from
//              TMEM, online max/sum in the log2 domain, writes P (16-bit) to
//              shared memory, rescales O in TMEM when the running max moves,
//              and runs the epilogue.
//   warp 4     TMA producer: Q once, then K/V tiles of the page table into a
//              STAGES-deep ring. A tile is 128 pool rows of one head, gathered
//              by one 3-D box load per 64 columns; the page table gives the
//              row of each tile, so pages need not be contiguous.
//   warp 5     TMEM allocator and MMA issuer: S = Q K^T (M=128, N=128, K=D) and
//              O += P V (M=128, N=D, K=128) as tcgen05 kind::f16 with fp32
//              accumulators in TMEM. S(j+1) is issued as soon as the softmax
//              has read S(j), so the tensor core overlaps the exponentials.
// TMEM: S in columns [0, 128), O in [128, 128 + D).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace pkv {

template <int D, int STAGES>
struct AttnSmem {
  static constexpr int kTileBytes = kTile * D * 2;   // one 128-row K, V or Q tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + STAGES * kTileBytes;
  static constexpr int kP = kV + STAGES * kTileBytes;
  static constexpr int kBars = kP + kTile * kTile * 2;
  static constexpr int kBytes = kBars + 256;
  static constexpr int kAlloc = kBytes + 1024;      // slack to align the base to 1 KB
};

constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;

__device__ __forceinline__ uint32_t pack2(float a, float b, bool fp16) {
  if (fp16) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Waits bounded by time only (used to drain in-flight async work on exit).
__device__ __forceinline__ void mbar_drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

template <int D, bool kFP16, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
  using L = AttnSmem<D, STAGES>;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_q = bars;
  uint64_t* bar_kv_full = bars + 1;
  uint64_t* bar_kv_empty = bars + 1 + STAGES;
  uint64_t* bar_s_full = bars + 1 + 2 * STAGES;
  uint64_t* bar_s_free = bar_s_full + 1;
  uint64_t* bar_p_full = bar_s_full + 2;
  uint64_t* bar_o_done = bar_s_full + 3;
  uint64_t* bar_drain = bar_s_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s_full + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const KvUnit u = a.units[blockIdx.x];
  const KvReq rq = a.reqs[u.req];
  const int n_tiles = u.tile_end - u.tile_begin;
  const KvTile* tiles = a.tiles + u.tile_begin;
  if (n_tiles <= 0) {   // the planner never emits an empty unit
    if (threadIdx.x == 0) atomicOr(a.err, 2u);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_s_free, 128);
    mbar_init(bar_p_full, 128);
    mbar_init(bar_o_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;
  const uint32_t tO = tmem + 128;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const CUtensorMap* mkv = &maps.kv[u.req];
      prefetch_tmap(&maps.q);
      prefetch_tmap(mkv);
      mbar_arrive_expect_tx(bar_q, L::kTileBytes);
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_3d(smem + L::kQ + kb * 16384, &maps.q, bar_q, kb * 64, u.head,
                    rq.q_row0 + u.qtile * kTile);
      int j = 0;
      for (; j < n_tiles; ++j) {
        const int s = j % STAGES;
        if (j >= STAGES && !mbar_wait(&bar_kv_empty[s], ((j / STAGES) - 1) & 1, abort_flag)) break;
        const KvTile t = tiles[j];
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
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = umma_idesc_f16(128, 128, kFP16, false);
      constexpr uint32_t idO = umma_idesc_f16(128, D, kFP16, true);
      const uint32_t sQ = smem_u32(smem + L::kQ);
      const uint32_t sK = smem_u32(smem + L::kK);
      const uint32_t sV = smem_u32(smem + L::kV);
      const uint32_t sP = smem_u32(smem + L::kP);
      auto issue_s = [&](int j) -> bool {
        const int s = j % STAGES;
        if (!mbar_wait(&bar_kv_full[s], (j / STAGES) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kb = sK + s * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_f16_ss(tS, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), idS, kk > 0);
        }
        umma_commit(bar_s_full);
        return true;
      };
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles) {
          if (!mbar_wait(bar_s_free, j & 1, abort_flag)) break;
          if (!issue_s(j + 1)) break;
        }
        if (!mbar_wait(bar_p_full, j & 1, abort_flag)) break;
        tc_fence_after();
        const int s = j % STAGES;
        const uint32_t vb = sV + s * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint32_t poff = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_f16_ss(tO, sdesc_sw128(sP + poff, 16, 1024), sdesc_sw128(vb + kk * 2048, 16384, 1024), idO,
                      (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bar_kv_empty[s]);
        umma_commit(bar_o_done);
      }
      // every MMA of this CTA must be complete before TMEM is released
      umma_commit(bar_drain);
      mbar_drain_wait(bar_drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x;
    const int rows_valid = min(kTile, rq.T - u.qtile * kTile);
    const bool active = warp * 32 < rows_valid;   // warp-uniform
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      // every wait is made warp-uniform: tcgen05.ld/st are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full, j & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      float p[kTile];
      if (active) {
#pragma unroll
        for (int c = 0; c < kTile / 32; ++c) {
          uint32_t r[32];
          tmem_ld32_wait(tS + lane_base + c * 32, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) p[c * 32 + i] = __uint_as_float(r[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_s_free);
      float alpha = 1.f;
      if (active) {
        const KvTile t = tiles[j];
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < kTile; ++c) {
          p[c] = (c < t.lo || c >= t.hi) ? -INFINITY : p[c];
          mx = fmaxf(mx, p[c]);
        }
        const float m_new = fmaxf(m_run, mx * sl2);
        alpha = ex2_approx(m_run - m_new);   // 0 on the first tile (m_run = -inf)
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < kTile; ++c) {
          p[c] = ex2_approx(fmaf(p[c], sl2, -m_new));
          sum += p[c];
        }
        l_run = l_run * alpha + sum;
        m_run = m_new;
      }
      if (j > 0) {
        // PV(j-1) must be done before O is rescaled and P is overwritten
        if (!__all_sync(0xffffffffu, mbar_wait(bar_o_done, (j - 1) & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        if (active && __any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32_wait(tO + lane_base + c * 32, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tO + lane_base + c * 32, r);
          }
          tmem_wait_st();
        }
      }
      if (active) {
        uint8_t* prow = smem + L::kP + row * 128;
#pragma unroll
        for (int ch = 0; ch < kTile / 8; ++ch) {
          uint4 v;
          v.x = pack2(p[ch * 8 + 0], p[ch * 8 + 1], kFP16);
          v.y = pack2(p[ch * 8 + 2], p[ch * 8 + 3], kFP16);
          v.z = pack2(p[ch * 8 + 4], p[ch * 8 + 5], kFP16);
          v.w = pack2(p[ch * 8 + 6], p[ch * 8 + 7], kFP16);
          const int kb = ch >> 3, cc = ch & 7;
          *reinterpret_cast<uint4*>(prow + kb * 16384 + ((cc ^ (row & 7)) << 4)) = v;
        }
        fence_async_smem();
      }
      tc_fence_before();
      mbar_arrive(bar_p_full);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && active && n_tiles > 0) {
      if (__all_sync(0xffffffffu, mbar_wait(bar_o_done, (n_tiles - 1) & 1, abort_flag))) {
        tc_fence_after();
        const int grow = rq.q_row0 + u.qtile * kTile + row;
        const bool store = row < rows_valid;
        const float inv = 1.f / l_run;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32_wait(tO + lane_base + c * 32, r);
          if (!store) continue;
          if (u.slot < 0) {
            uint16_t* o = reinterpret_cast<uint16_t*>(a.out) + ((size_t)grow * a.H + u.head) * D + c * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 v;
              v.x = pack2(__uint_as_float(r[i + 0]) * inv, __uint_as_float(r[i + 1]) * inv, kFP16);
              v.y = pack2(__uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv, kFP16);
              v.z = pack2(__uint_as_float(r[i + 4]) * inv, __uint_as_float(r[i + 5]) * inv, kFP16);
              v.w = pack2(__uint_as_float(r[i + 6]) * inv, __uint_as_float(r[i + 7]) * inv, kFP16);
              *reinterpret_cast<uint4*>(o + i) = v;
            }
          } else {
            float* po = a.part_o + ((size_t)u.slot * kTile + row) * D + c * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float4 v = make_float4(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv,
                                     __uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
              *reinterpret_cast<float4*>(po + i) = v;
            }
          }
        }
        if (store && u.slot >= 0) a.part_lse[(size_t)u.slot * kTile + row] = m_run + log2f(l_run);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(a.err, 1u);
}

template <int D, bool kFP16, int STAGES>
static cudaError_t launch_attn_t(const AttnMaps& maps, const AttnArgs& a, int n_units, cudaStream_t stream) {
  using L = AttnSmem<D, STAGES>;
  auto kern = paged_prefill_attn_kernel<D, kFP16, STAGES>;
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
  if (D == 64) return fp16 ? launch_attn_t<64, true, 2>(maps, a, n_units, stream)
                           : launch_attn_t<64, false, 2>(maps, a, n_units, stream);
  if (D == 128) return fp16 ? launch_attn_t<128, true, 2>(maps, a, n_units, stream)
                            : launch_attn_t<128, false, 2>(maps, a, n_units, stream);
  return cudaErrorInvalidValue;
}

int attention_ctas_per_sm(int D) { return 1; }

}  // namespace pkv
