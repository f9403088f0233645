// copy_impl.cuh -- copy-on-write block copies, device code shared by the copy kernel (copy.cu)
// and the fused decode step (decode_kernel.cuh).
//
// deepinsea.top "PagedAttention 内存管理深度解析", section "Copy-on-Write 机制": sequences forked for
// beam search share physical blocks, and a block is copied only when one of them is about to write
// into it; yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section
// "PagedAttention分页注意力机制与vLLM实现": a fork writes its new tokens into new blocks without
// touching the shared prefix. A block of the pool is contiguous across heads ([nb][H][bs][row]),
// so one (src, dst) pair is two contiguous byte ranges (K codes, V codes) plus H scales (and zero
// points), copied with 16-byte vector loads and stores.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace pkv {
namespace copy_detail {

// Thread `tid` of `nthreads` copies vectors tid, tid + nthreads, ... of the pairs' code ranges
// taken one after another, then scale entries the same way. A pair with an out-of-range id is
// skipped and reported (once, by the thread that meets its first vector); a pair with
// src == dst is a no-op.
__device__ __forceinline__ void copy_all(const CopyParams& p, int64_t tid, int64_t nthreads) {
  const int64_t k_vec = p.k_block_bytes / 16, v_vec = p.v_block_bytes / 16, per = k_vec + v_vec;
  const int64_t total = (int64_t)p.n_pairs * per;
  const bool narrow = total < (1ll << 32);  // 32-bit division suffices
  for (int64_t i = tid; i < total; i += nthreads) {
    const int64_t pair = narrow ? (int64_t)((uint32_t)i / (uint32_t)per) : i / per;
    const int64_t e = i - pair * per;
    const int src = p.block_mapping[2 * pair];
    const int dst = p.block_mapping[2 * pair + 1];
    if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
      if (e == 0) record_error(p.dev_error, PKV_DEVERR_BLOCK_ID);
      continue;
    }
    if (src == dst) continue;
    if (e < k_vec) {
      reinterpret_cast<uint4*>(p.k_codes + (size_t)dst * p.k_block_bytes)[e] =
          reinterpret_cast<const uint4*>(p.k_codes + (size_t)src * p.k_block_bytes)[e];
    } else {
      reinterpret_cast<uint4*>(p.v_codes + (size_t)dst * p.v_block_bytes)[e - k_vec] =
          reinterpret_cast<const uint4*>(p.v_codes + (size_t)src * p.v_block_bytes)[e - k_vec];
    }
  }
  const int H = p.num_kv_heads;
  for (int64_t i = tid; i < (int64_t)p.n_pairs * H; i += nthreads) {
    const int64_t pair = i / H, h = i - pair * H;
    const int src = p.block_mapping[2 * pair];
    const int dst = p.block_mapping[2 * pair + 1];
    if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks || src == dst) continue;
    if (p.k_scale) p.k_scale[(size_t)dst * H + h] = p.k_scale[(size_t)src * H + h];
    if (p.v_scale) p.v_scale[(size_t)dst * H + h] = p.v_scale[(size_t)src * H + h];
    if (p.v_zp) p.v_zp[(size_t)dst * H + h] = p.v_zp[(size_t)src * H + h];
  }
}

}  // namespace copy_detail
}  // namespace pkv
