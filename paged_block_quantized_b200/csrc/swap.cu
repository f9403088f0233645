// swap.cu -- block swap between the device pool and a pool in pinned host memory (sm_100a).
//
// deepinsea.top "PagedAttention 内存管理深度解析", section "Swap 机制": when device memory runs
// short, KV-cache blocks are moved out to CPU memory and brought back later; the page warns that
// the transfer is slow and should be a last resort. Here a swap moves whole blocks (every head's K
// codes, V codes, scales and zero points) between two pools of the same geometry: the device pool
// and a host pool in page-locked memory that the GPU addresses directly (unified addressing).
//
// One launch moves any number of scattered blocks: each thread copies 16-byte vectors of the
// pairs' code ranges taken one after another, four independent loads in flight before their
// stores (reads of host memory cross the bus with microseconds of latency, so many must be
// outstanding at once), then the per-head scale and zero-point entries.
#include "common.cuh"
#include "internal.h"

namespace pkv {

namespace {

constexpr int kSwapThreads = 256;
constexpr int kSwapUnroll = 4;

__global__ void __launch_bounds__(kSwapThreads) swap_blocks_kernel(const SwapParams p) {
  const int64_t k_vec = p.k_block_bytes / 16, v_vec = p.v_block_bytes / 16, per = k_vec + v_vec;
  const int64_t total = (int64_t)p.n_pairs * per;
  const int64_t tid = (int64_t)blockIdx.x * kSwapThreads + threadIdx.x;
  const int64_t nth = (int64_t)gridDim.x * kSwapThreads;
  for (int64_t base = tid; base < total; base += kSwapUnroll * nth) {
    uint4 val[kSwapUnroll];
    uint4* dst[kSwapUnroll];
#pragma unroll
    for (int u = 0; u < kSwapUnroll; ++u) {
      dst[u] = nullptr;
      const int64_t i = base + u * nth;
      if (i >= total) continue;
      const int64_t pair = i / per, e = i - pair * per;
      const int32_t s = p.block_mapping[2 * pair], d = p.block_mapping[2 * pair + 1];
      if (s < 0 || s >= p.src_blocks || d < 0 || d >= p.dst_blocks) {
        if (e == 0) record_error(p.dev_error, PKV_DEVERR_BLOCK_ID);
        continue;
      }
      if (e < k_vec) {
        val[u] = reinterpret_cast<const uint4*>(p.src_k + (size_t)s * p.k_block_bytes)[e];
        dst[u] = reinterpret_cast<uint4*>(p.dst_k + (size_t)d * p.k_block_bytes) + e;
      } else {
        val[u] = reinterpret_cast<const uint4*>(p.src_v + (size_t)s * p.v_block_bytes)[e - k_vec];
        dst[u] = reinterpret_cast<uint4*>(p.dst_v + (size_t)d * p.v_block_bytes) + (e - k_vec);
      }
    }
#pragma unroll
    for (int u = 0; u < kSwapUnroll; ++u)
      if (dst[u] != nullptr) *dst[u] = val[u];
  }
  const int H = p.num_kv_heads;
  for (int64_t i = tid; i < (int64_t)p.n_pairs * H; i += nth) {
    const int64_t pair = i / H, h = i - pair * H;
    const int32_t s = p.block_mapping[2 * pair], d = p.block_mapping[2 * pair + 1];
    if (s < 0 || s >= p.src_blocks || d < 0 || d >= p.dst_blocks) continue;
    if (p.src_ks) p.dst_ks[(size_t)d * H + h] = p.src_ks[(size_t)s * H + h];
    if (p.src_vs) p.dst_vs[(size_t)d * H + h] = p.src_vs[(size_t)s * H + h];
    if (p.src_zp) p.dst_zp[(size_t)d * H + h] = p.src_zp[(size_t)s * H + h];
  }
}

}  // namespace

cudaError_t launch_swap(const SwapParams& p, cudaStream_t stream) {
  if (p.n_pairs == 0) return cudaSuccess;
  const int64_t vecs = (int64_t)p.n_pairs * ((p.k_block_bytes + p.v_block_bytes) / 16);
  int64_t ctas = (vecs + kSwapUnroll * kSwapThreads - 1) / (kSwapUnroll * kSwapThreads);
  ctas = ctas < 1 ? 1 : (ctas > 2048 ? 2048 : ctas);
  swap_blocks_kernel<<<(unsigned)ctas, kSwapThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
