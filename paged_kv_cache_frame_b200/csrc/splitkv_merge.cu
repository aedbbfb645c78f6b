// Split-KV merge: combine the chunk partials of one (request, head, q-tile).
// With per-chunk normalised outputs O_c and log2-sum-exp values L_c,
//   O = sum_c 2^(L_c - L*) O_c / sum_c 2^(L_c - L*),   L* = max_c L_c,
// which equals the softmax over the union of the chunks. One warp per query
// row: lane c holds chunk c's weight (32 chunks per pass), and the lanes
// split the head dimension, reading every chunk's row with independent
// vector loads.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "kernels.h"
#include "launch.cuh"
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

template <int D, bool kFP16>
__global__ void __launch_bounds__(256) splitkv_merge_kernel(const MergeArgs m) {
  constexpr int V = D / 32;     // columns per lane: 2 (D = 64) or 4 (D = 128)
  constexpr int kPre = 16;      // chunks whose rows are requested with the lse values
  constexpr size_t kStride = (size_t)kTile * D / V;   // one slot, in vectors
  using Vec = typename VecF<V>::T;
  pdl_wait();      // the partials come from the attention kernel
  pdl_trigger();
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int item = gwarp / kTile;
  const int row = gwarp % kTile;
  if (item >= m.n_items) return;
  const KvMergeItem it = m.items[item];
  if (row >= it.rows) return;
  const int n = it.n;
  const float* lse = m.part_lse + (size_t)it.slot0 * kTile + row;   // chunk c at lse[c * kTile]
  const Vec* po = reinterpret_cast<const Vec*>(m.part_o + ((size_t)it.slot0 * kTile + row) * D) + lane;
  // Neither the first chunks' rows nor their lse values depend on the
  // other, so both go out before the first result comes back.
  const float l0 = lane < n ? lse[(size_t)lane * kTile] : -INFINITY;
  Vec x[kPre];
#pragma unroll
  for (int k = 0; k < kPre; ++k)
    if (k < n) x[k] = po[k * kStride];
  // global max of the log2-sum-exps
  float top = l0;
  for (int c0 = 32; c0 < n; c0 += 32)
    top = fmaxf(top, c0 + lane < n ? lse[(size_t)(c0 + lane) * kTile] : -INFINITY);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int c0 = 0; c0 < n; c0 += 32) {
    const int nc = min(32, n - c0);
    const float l = c0 == 0 ? l0 : (lane < nc ? lse[(size_t)(c0 + lane) * kTile] : -INFINITY);
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
      for (int k = 0; k < 4; ++k) y[k] = pc[(c + k) * kStride];
#pragma unroll
      for (int k = 0; k < 4; ++k) fma_vec(acc, y[k], __shfl_sync(0xffffffffu, w, c + k));
    }
    for (; c < nc; ++c) fma_vec(acc, pc[c * kStride], __shfl_sync(0xffffffffu, w, c));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  const float inv = 1.f / wsum;
  const size_t orow = ((size_t)(it.row0 + row) * m.H + it.head) * D + lane * V;
  uint32_t packed[V / 2];
#pragma unroll
  for (int i = 0; i < V; i += 2)
    packed[i / 2] = kFP16 ? cvt_pack_f16(acc[i] * inv, acc[i + 1] * inv) : cvt_pack_bf16(acc[i] * inv, acc[i + 1] * inv);
  if (V == 2)
    reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(m.out) + orow)[0] = packed[0];
  else
    *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(m.out) + orow) = make_uint2(packed[0], packed[V / 2 - 1]);
}

cudaError_t launch_merge(const MergeArgs& m, int D, bool fp16, cudaStream_t stream) {
  if (m.n_items <= 0) return cudaSuccess;
  const long long warps = (long long)m.n_items * kTile;
  const int blocks = (int)((warps * 32 + 255) / 256);
  if (D == 64)
    return fp16 ? launch_pdl(splitkv_merge_kernel<64, true>, dim3(blocks), dim3(256), 0, stream, m)
                : launch_pdl(splitkv_merge_kernel<64, false>, dim3(blocks), dim3(256), 0, stream, m);
  if (D == 128)
    return fp16 ? launch_pdl(splitkv_merge_kernel<128, true>, dim3(blocks), dim3(256), 0, stream, m)
                : launch_pdl(splitkv_merge_kernel<128, false>, dim3(blocks), dim3(256), 0, stream, m);
  return cudaErrorInvalidValue;
}

}  // namespace pkv
