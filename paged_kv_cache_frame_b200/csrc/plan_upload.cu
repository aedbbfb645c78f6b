// Plan upload without host staging memory: the serialised plan travels in the
// launch parameters of a one-block copy kernel (up to kChunkWords words per
// launch), so the upload is asynchronous on the caller's stream, needs no
// pinned buffer and never waits for earlier work.
#include "kernels.h"
#include "launch.cuh"

namespace pkv {

template <int kWords>
struct UploadChunk {
  uint32_t* dst;
  int n_words;
  uint32_t words[kWords];
};

template <int kWords>
__global__ void __launch_bounds__(256) plan_upload_kernel(const __grid_constant__ UploadChunk<kWords> c) {
  pdl_wait();   // earlier kernels may still read the tables this overwrites
  for (int i = threadIdx.x; i < c.n_words; i += blockDim.x) c.dst[i] = c.words[i];
}

template <int kWords>
static cudaError_t launch_chunk(uint32_t* dst, const uint32_t* src, int n, cudaStream_t stream) {
  UploadChunk<kWords> c;
  c.dst = dst;
  c.n_words = n;
  for (int i = 0; i < n; ++i) c.words[i] = src[i];
  return launch_pdl(plan_upload_kernel<kWords>, dim3(1), dim3(256), 0, stream, c);
}

constexpr int kMax = 7680;   // 30 KB of payload per launch (kernel parameters allow 32 KB)

int upload_launches(size_t bytes) { return (int)(((bytes + 3) / 4 + kMax - 1) / kMax); }

cudaError_t upload_plan(void* dst, const void* src, size_t bytes, cudaStream_t stream) {
  const uint32_t* s = static_cast<const uint32_t*>(src);
  uint32_t* d = static_cast<uint32_t*>(dst);
  size_t words = (bytes + 3) / 4;
  while (words > 0) {
    const int n = (int)(words < (size_t)kMax ? words : (size_t)kMax);
    cudaError_t e;
    if (n <= 1024) e = launch_chunk<1024>(d, s, n, stream);
    else if (n <= 3072) e = launch_chunk<3072>(d, s, n, stream);
    else e = launch_chunk<kMax>(d, s, n, stream);
    if (e != cudaSuccess) return e;
    s += n;
    d += n;
    words -= n;
  }
  return cudaSuccess;
}

}  // namespace pkv
