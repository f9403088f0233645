// copy.cu -- the copy-on-write kernel (sm_100a): every (src, dst) pair of the mapping, whole
// blocks across heads. The copy itself and its sources are in copy_impl.cuh.
#include "copy_impl.cuh"

namespace pkv {

namespace {

constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(const CopyParams p) {
  copy_detail::copy_all(p, (int64_t)blockIdx.x * kCopyThreads + threadIdx.x, (int64_t)gridDim.x * kCopyThreads);
}

}  // namespace

cudaError_t launch_copy(const CopyParams& p, cudaStream_t stream) {
  if (p.n_pairs == 0) return cudaSuccess;
  // about four 16-byte vectors per thread
  const int64_t vecs = (int64_t)p.n_pairs * ((p.k_block_bytes + p.v_block_bytes) / 16);
  int64_t ctas = (vecs + 4 * kCopyThreads - 1) / (4 * kCopyThreads);
  ctas = ctas < 1 ? 1 : (ctas > 1024 ? 1024 : ctas);
  copy_blocks_kernel<<<(unsigned)ctas, kCopyThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
