// Split-KV merge of one query row, by one warp. With per-chunk normalised
// outputs O_c and log2-sum-exp values L_c of the row,
//   O = sum_c 2^(L_c - L*) O_c / sum_c 2^(L_c - L*),   L* = max_c L_c,
// which equals the softmax over the union of the chunks. Lane c holds chunk
// c's weight (32 chunks per pass) and the lanes split the head dimension,
// reading every chunk's row with independent vector loads. The partials are
// read through L2 only (ld.global.cg): they were written by other CTAs, and
// in the fused form by CTAs of the same launch.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "kv_layout.h"
#include "sm100.cuh"

namespace pkv {

template <int V>
struct VecF;
template <>
struct VecF<2> {
  using T = float2;
};
template <>
struct VecF<4> {
  using T = float4;
};

__device__ __forceinline__ float2 ldcg_vec(const float2* p) { return __ldcg(p); }
__device__ __forceinline__ float4 ldcg_vec(const float4* p) { return __ldcg(p); }

__device__ __forceinline__ void fma_vec(float (&acc)[2], const float2& v, float w) {
  acc[0] = fmaf(w, v.x, acc[0]);
  acc[1] = fmaf(w, v.y, acc[1]);
}
__device__ __forceinline__ void fma_vec(float (&acc)[4], const float4& v, float w) {
  acc[0] = fmaf(w, v.x, acc[0]);
  acc[1] = fmaf(w, v.y, acc[1]);
  acc[2] = fmaf(w, v.z, acc[2]);
  acc[3] = fmaf(w, v.w, acc[3]);
}

// Row `row` of slots slot0 .. slot0 + n - 1 (partials [slot][128][D] and
// [slot][128]) into out_row[0 .. D) in the 16-bit output type.
template <int D, bool kFP16>
__device__ __forceinline__ void merge_row_warp(const float* part_o, const float* part_lse, int slot0, int n,
                                               int row, uint16_t* out_row, int lane) {
  constexpr int V = D / 32;     // columns per lane: 2 (D = 64) or 4 (D = 128)
  constexpr int kPre = 16;      // chunks whose rows are requested with the lse values
  constexpr size_t kStride = (size_t)kTile * D / V;   // one slot, in vectors
  using Vec = typename VecF<V>::T;
  const float* lse = part_lse + (size_t)slot0 * kTile + row;   // chunk c at lse[c * kTile]
  const Vec* po = reinterpret_cast<const Vec*>(part_o + ((size_t)slot0 * kTile + row) * D) + lane;
  // Neither the first chunks' rows nor their lse values depend on the
  // other, so both go out before the first result comes back.
  const float l0 = lane < n ? __ldcg(lse + (size_t)lane * kTile) : -INFINITY;
  Vec x[kPre];
#pragma unroll
  for (int k = 0; k < kPre; ++k)
    if (k < n) x[k] = ldcg_vec(po + k * kStride);
  // global max of the log2-sum-exps
  float top = l0;
  for (int c0 = 32; c0 < n; c0 += 32)
    top = fmaxf(top, c0 + lane < n ? __ldcg(lse + (size_t)(c0 + lane) * kTile) : -INFINITY);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int c0 = 0; c0 < n; c0 += 32) {
    const int nc = min(32, n - c0);
    const float l = c0 == 0 ? l0 : (lane < nc ? __ldcg(lse + (size_t)(c0 + lane) * kTile) : -INFINITY);
    const float w = lane < nc ? ex2_approx(l - top) : 0.f;
    wsum += w;
    int c = 0;
    if (c0 == 0) {
#pragma unroll
      for (int k = 0; k < kPre; ++k)
        if (k < nc) fma_vec(acc, x[k], __shfl_sync(0xffffffffu, w, k));
      c = min(kPre, nc);
    }
    const Vec* pc = po + (size_t)c0 * kStride;
    for (; c + 4 <= nc; c += 4) {   // four independent loads in flight
      Vec y[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) y[k] = ldcg_vec(pc + (c + k) * kStride);
#pragma unroll
      for (int k = 0; k < 4; ++k) fma_vec(acc, y[k], __shfl_sync(0xffffffffu, w, c + k));
    }
    for (; c < nc; ++c) fma_vec(acc, ldcg_vec(pc + c * kStride), __shfl_sync(0xffffffffu, w, c));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  const float inv = 1.f / wsum;
  uint32_t packed[V / 2];
#pragma unroll
  for (int i = 0; i < V; i += 2)
    packed[i / 2] = kFP16 ? cvt_pack_f16(acc[i] * inv, acc[i + 1] * inv) : cvt_pack_bf16(acc[i] * inv, acc[i + 1] * inv);
  uint16_t* o = out_row + lane * V;
  if (V == 2)
    *reinterpret_cast<uint32_t*>(o) = packed[0];
  else
    *reinterpret_cast<uint2*>(o) = make_uint2(packed[0], packed[V / 2 - 1]);
}

}  // namespace pkv

namespace pkv {

// The same merge for the S rows of one share, their chunks' partial rows
// already requested into shared memory (`stage`, [n][S][D] fp32): 8 lanes
// per row, lane l holding output columns 4 (l + 8 v) .. 4 (l + 8 v) + 3 (v <
// D/32, so a row's 8 lanes read 128 contiguous bytes at a time) and the
// log2-sum-exps of chunks l, l + 8, l + 16, l + 24 (n <= 32). Each row's lse
// values are loaded before `wait()` (the stage's completion) is called.
// row_of(i) gives share row i's (slot0, row, output row pointer); rows i =
// first, first + stride, ... < S go to the calling group. Returns false if
// wait() failed (nothing was read from the stage then).
template <int D, bool kFP16, typename Wait, typename RowOf>
__device__ __forceinline__ bool merge_rows_staged(const float* stage, int S, const float* part_lse, int n, int first,
                                                  int stride, int l8, Wait wait, RowOf row_of) {
  constexpr int kV4 = D / 32;                  // float4 per lane per chunk
  const int g0 = threadIdx.x & 24;             // first lane of this row's group
  const unsigned gmask = 0xFFu << g0;
  const size_t chunk4 = (size_t)S * D / 4;     // one chunk's rows in the stage, in float4
  bool waited = false;
  for (int i = first; i < S; i += stride) {
    int slot0, row;
    uint16_t* out_row;
    row_of(i, &slot0, &row, &out_row);
    const float* lse = part_lse + (size_t)slot0 * kTile + row;
    float lv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) lv[q] = l8 + 8 * q < n ? __ldcg(lse + (size_t)(l8 + 8 * q) * kTile) : -INFINITY;
    if (!waited) {
      if (!wait()) return false;
      waited = true;
    }
    float top = fmaxf(fmaxf(lv[0], lv[1]), fmaxf(lv[2], lv[3]));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) top = fmaxf(top, __shfl_xor_sync(gmask, top, o));
    float wl[4];
    float wsum = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      wl[q] = l8 + 8 * q < n ? ex2_approx(lv[q] - top) : 0.f;
      wsum += wl[q];
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) wsum += __shfl_xor_sync(gmask, wsum, o);
    float acc[kV4][4];
#pragma unroll
    for (int v = 0; v < kV4; ++v) acc[v][0] = acc[v][1] = acc[v][2] = acc[v][3] = 0.f;
    const float4* xs = reinterpret_cast<const float4*>(stage + (size_t)i * D) + l8;
    for (int c = 0; c < n; ++c) {
      // chunk c's weight is wl[c / 8] of lane c % 8 (c is uniform over the group)
      const int q = c >> 3;
      const float sel = q == 0 ? wl[0] : q == 1 ? wl[1] : q == 2 ? wl[2] : wl[3];
      const float w = __shfl_sync(gmask, sel, g0 + (c & 7));
#pragma unroll
      for (int v = 0; v < kV4; ++v) {
        const float4 y = xs[(size_t)c * chunk4 + 8 * v];
        acc[v][0] = fmaf(w, y.x, acc[v][0]);
        acc[v][1] = fmaf(w, y.y, acc[v][1]);
        acc[v][2] = fmaf(w, y.z, acc[v][2]);
        acc[v][3] = fmaf(w, y.w, acc[v][3]);
      }
    }
    const float inv = 1.f / wsum;
#pragma unroll
    for (int v = 0; v < kV4; ++v) {
      const uint32_t p0 = kFP16 ? cvt_pack_f16(acc[v][0] * inv, acc[v][1] * inv)
                                : cvt_pack_bf16(acc[v][0] * inv, acc[v][1] * inv);
      const uint32_t p1 = kFP16 ? cvt_pack_f16(acc[v][2] * inv, acc[v][3] * inv)
                                : cvt_pack_bf16(acc[v][2] * inv, acc[v][3] * inv);
      *reinterpret_cast<uint2*>(out_row + 4 * (l8 + 8 * v)) = make_uint2(p0, p1);
    }
  }
  return true;
}

}  // namespace pkv
