// append_frame scatter ([P1] "Appending New Frames": the frame's K/V are split
// into special and patch parts; special tokens go to the continuous special
// pages, patch tokens to the frame's newly allocated or recycled patch page.
// [P1] is "How the Paged KV Cache Attention Mechanism Enables Long Sequence
// Inference in LingBot-Map").
//
// k, v: [T, H, D]; token t < NS is special token sp0 + t of the stream,
// stored at page sp_base + (sp0 + t) / page_size, slot (sp0 + t) % page_size
// (sp_base: the stream's first special page);
// token t >= NS is patch row t - NS of page `patch_page`. Pool
// [max_pages, 2, page_size, H, D] with dimension 1 = K/V. One thread moves one
// 16-byte vector; consecutive threads move consecutive vectors of a token row,
// so loads and stores are fully coalesced.
#include "kernels.h"
#include "launch.cuh"

namespace pkv {

__global__ void __launch_bounds__(256) append_scatter_kernel(const AppendArgs a) {
  pdl_wait();      // k/v may come from the previous kernel; the pool from the one before
  pdl_trigger();   // the attention kernel may set up meanwhile (it waits for this one)
  const long long per_kv = (long long)a.T * a.row_vecs;
  const long long total = 2 * per_kv;
  const uint4* k = reinterpret_cast<const uint4*>(a.k);
  const uint4* v = reinterpret_cast<const uint4*>(a.v);
  uint4* pool = reinterpret_cast<uint4*>(a.pool);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int kv = i >= per_kv;
    const long long rem = i - kv * per_kv;
    const int t = (int)(rem / a.row_vecs);
    const int c = (int)(rem - (long long)t * a.row_vecs);
    int page, slot;
    if (t < a.NS) {
      const int j = a.sp0 + t;
      page = a.sp_base + j / a.page_size;
      slot = j % a.page_size;
    } else {
      page = a.patch_page;
      slot = t - a.NS;
    }
    const uint4 x = kv ? v[rem] : k[rem];
    pool[(((long long)page * 2 + kv) * a.page_size + slot) * a.row_vecs + c] = x;
  }
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  const long long total = 2LL * a.T * a.row_vecs;
  if (total == 0) return cudaSuccess;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  return launch_pdl(append_scatter_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, a);
}

}  // namespace pkv
