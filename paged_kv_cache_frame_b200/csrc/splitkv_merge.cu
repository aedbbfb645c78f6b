// Split-KV merge as its own launch, for schedules whose CTAs cannot all be
// resident at once (otherwise the attention kernel merges in its epilogue):
// one warp per query row of every (request, head, q-tile) that was split.
#include "kernels.h"
#include "launch.cuh"
#include "merge.cuh"

namespace pkv {

template <int D, bool kFP16>
__global__ void __launch_bounds__(256) splitkv_merge_kernel(const MergeArgs m) {
  pdl_wait();      // the partials come from the attention kernel
  pdl_trigger();
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int item = gwarp / kTile;
  const int row = gwarp % kTile;
  if (item >= m.n_items) return;
  const KvMergeItem it = m.items[item];
  if (row >= it.rows) return;
  uint16_t* out_row = reinterpret_cast<uint16_t*>(m.out) + ((size_t)(it.row0 + row) * m.H + it.head) * D;
  merge_row_warp<D, kFP16>(m.part_o, m.part_lse, it.slot0, it.n, row, out_row, lane);
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
