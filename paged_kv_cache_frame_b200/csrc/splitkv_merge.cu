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

template <int D, bool kFP16>
__global__ void __launch_bounds__(256) splitkv_merge_kernel(const MergeArgs m) {
  constexpr int V = D / 32;   // columns per lane: 2 (D = 64) or 4 (D = 128)
  using Vec = typename VecF<V>::T;
  pdl_wait();      // the partials come from the attention kernel
  pdl_trigger();
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int item = gwarp / kTile;
  const int row = gwarp % kTile;
  if (item >= m.n_items) return;
  const KvMergeItem it = m.items[item];
  const KvReq rq = m.reqs[it.req];
  if (it.qtile * kTile + row >= rq.T) return;
  // global max of the log2-sum-exps
  float top = -INFINITY;
  for (int c0 = 0; c0 < it.n; c0 += 32) {
    const float l = c0 + lane < it.n ? m.part_lse[(size_t)(it.slot0 + c0 + lane) * kTile + row] : -INFINITY;
    top = fmaxf(top, l);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int c0 = 0; c0 < it.n; c0 += 32) {
    const int nc = min(32, it.n - c0);
    const float w = lane < nc ? ex2_approx(m.part_lse[(size_t)(it.slot0 + c0 + lane) * kTile + row] - top) : 0.f;
    wsum += w;
    const Vec* po = reinterpret_cast<const Vec*>(m.part_o + ((size_t)(it.slot0 + c0) * kTile + row) * D) + lane;
    constexpr size_t kStride = (size_t)kTile * D / V;   // one slot, in vectors
    int c = 0;
    for (; c + 4 <= nc; c += 4) {   // four independent loads in flight
      Vec x[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = po[(c + k) * kStride];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float wk = __shfl_sync(0xffffffffu, w, c + k);
        const float* xf = reinterpret_cast<const float*>(&x[k]);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = fmaf(wk, xf[i], acc[i]);
      }
    }
    for (; c < nc; ++c) {
      const Vec x = po[c * kStride];
      const float wk = __shfl_sync(0xffffffffu, w, c);
      const float* xf = reinterpret_cast<const float*>(&x);
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = fmaf(wk, xf[i], acc[i]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  const float inv = 1.f / wsum;
  const size_t orow = ((size_t)(rq.q_row0 + it.qtile * kTile + row) * m.H + it.head) * D + lane * V;
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
