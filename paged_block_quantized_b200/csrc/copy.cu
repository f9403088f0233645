// copy.cu -- copy-on-write block copies (sm_100a).
//
// deepinsea.top "PagedAttention 内存管理深度解析", section "Copy-on-Write 机制": sequences forked for
// beam search share physical blocks, and a block is copied only when one of them is about to write
// into it; yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section
// "PagedAttention分页注意力机制与vLLM实现": a fork writes its new tokens into new blocks without
// touching the shared prefix. A block of the pool is contiguous across heads ([nb][H][bs][row]),
// so one (src, dst) pair is two contiguous byte ranges (K codes, V codes) plus H scales (and zero
// points), copied here with 16-byte vector loads and stores.
#include "common.cuh"
#include "internal.h"

namespace pkv {

namespace {

constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(const CopyParams p) {
  const int pair = blockIdx.x;
  const int src = p.block_mapping[2 * pair];
  const int dst = p.block_mapping[2 * pair + 1];
  if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
    if (blockIdx.y == 0 && threadIdx.x == 0) record_error(p.dev_error, PKV_DEVERR_BLOCK_ID);
    return;
  }
  if (src == dst) return;
  const int64_t k_vec = p.k_block_bytes / 16, v_vec = p.v_block_bytes / 16;
  const uint4* ks = reinterpret_cast<const uint4*>(p.k_codes + (size_t)src * p.k_block_bytes);
  uint4* kd = reinterpret_cast<uint4*>(p.k_codes + (size_t)dst * p.k_block_bytes);
  const uint4* vs = reinterpret_cast<const uint4*>(p.v_codes + (size_t)src * p.v_block_bytes);
  uint4* vd = reinterpret_cast<uint4*>(p.v_codes + (size_t)dst * p.v_block_bytes);
  const int64_t stride = (int64_t)gridDim.y * kCopyThreads;
  for (int64_t i = (int64_t)blockIdx.y * kCopyThreads + threadIdx.x; i < k_vec + v_vec; i += stride) {
    if (i < k_vec) {
      kd[i] = ks[i];
    } else {
      vd[i - k_vec] = vs[i - k_vec];
    }
  }
  if (blockIdx.y == 0) {
    const int H = p.num_kv_heads;
    for (int h = threadIdx.x; h < H; h += kCopyThreads) {
      if (p.k_scale) p.k_scale[(size_t)dst * H + h] = p.k_scale[(size_t)src * H + h];
      if (p.v_scale) p.v_scale[(size_t)dst * H + h] = p.v_scale[(size_t)src * H + h];
      if (p.v_zp) p.v_zp[(size_t)dst * H + h] = p.v_zp[(size_t)src * H + h];
    }
  }
}

}  // namespace

cudaError_t launch_copy(const CopyParams& p, cudaStream_t stream) {
  if (p.n_pairs == 0) return cudaSuccess;
  const int64_t vecs = (p.k_block_bytes + p.v_block_bytes) / 16;
  int slices = (int)((vecs + 4 * kCopyThreads - 1) / (4 * kCopyThreads));  // ~4 vectors per thread
  slices = slices < 1 ? 1 : (slices > 64 ? 64 : slices);
  dim3 grid(p.n_pairs, slices);
  copy_blocks_kernel<<<grid, kCopyThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
