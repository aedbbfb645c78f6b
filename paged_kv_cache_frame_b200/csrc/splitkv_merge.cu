// Split-KV merge: combine the chunk partials of one (request, head, q-tile).
// With per-chunk normalised outputs O_c and log2-sum-exp values L_c,
//   O = sum_c 2^(L_c - L*) O_c / sum_c 2^(L_c - L*),   L* = max_c L_c,
// which equals the softmax over the union of the chunks. One warp per query
// row; lanes stride over the head dimension.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace pkv {

template <int D, bool kFP16>
__global__ void __launch_bounds__(256) splitkv_merge_kernel(const MergeArgs m) {
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int item = gwarp / kTile;
  const int row = gwarp % kTile;
  if (item >= m.n_items) return;
  const KvMergeItem it = m.items[item];
  const KvReq rq = m.reqs[it.req];
  if (it.qtile * kTile + row >= rq.T) return;
  float top = -INFINITY;
  for (int c = 0; c < it.n; ++c) top = fmaxf(top, m.part_lse[(size_t)(it.slot0 + c) * kTile + row]);
  constexpr int V = D / 32;
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int c = 0; c < it.n; ++c) {
    const size_t base = (size_t)(it.slot0 + c) * kTile + row;
    const float w = ex2_approx(m.part_lse[base] - top);
    wsum += w;
    const float* po = m.part_o + base * D;
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = fmaf(w, po[lane + 32 * i], acc[i]);
  }
  const float inv = 1.f / wsum;
  const size_t orow = ((size_t)(rq.q_row0 + it.qtile * kTile + row) * m.H + it.head) * D;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const float x = acc[i] * inv;
    if (kFP16)
      reinterpret_cast<__half*>(m.out)[orow + lane + 32 * i] = __float2half_rn(x);
    else
      reinterpret_cast<__nv_bfloat16*>(m.out)[orow + lane + 32 * i] = __float2bfloat16_rn(x);
  }
}

cudaError_t launch_merge(const MergeArgs& m, int D, bool fp16, cudaStream_t stream) {
  if (m.n_items <= 0) return cudaSuccess;
  const long long warps = (long long)m.n_items * kTile;
  const int blocks = (int)((warps * 32 + 255) / 256);
  if (D == 64) {
    if (fp16) splitkv_merge_kernel<64, true><<<blocks, 256, 0, stream>>>(m);
    else splitkv_merge_kernel<64, false><<<blocks, 256, 0, stream>>>(m);
  } else if (D == 128) {
    if (fp16) splitkv_merge_kernel<128, true><<<blocks, 256, 0, stream>>>(m);
    else splitkv_merge_kernel<128, false><<<blocks, 256, 0, stream>>>(m);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pkv
