// prefill.cu -- launch of the chunked-prefill kernel (prefill_kernel.cuh): one CTA per 128 query
// columns of one (sequence, KV head), INT8 K with INT8 or INT4 V, head_dim 128, block size 16 or 32.
#include <cstring>

#include "prefill_kernel.cuh"
#include "prefill_tc.cuh"

// 1: the fifth-generation tensor-core kernel (prefill_tc.cuh); 0: the warp-level mma kernel
// (prefill_kernel.cuh)
#ifndef PKV_PREFILL_TC
#define PKV_PREFILL_TC 1
#endif

namespace pkv {

bool prefill_supported(int32_t k_dtype, int32_t v_dtype, int32_t block_size, int32_t head_dim) {
  return k_dtype == PKV_INT8_SYM && (v_dtype == PKV_INT8_SYM || v_dtype == PKV_INT4_ASYM) &&
         (block_size == 16 || block_size == 32) && head_dim == 128;
}

namespace {

template <int VT, int BS, bool PREFIX>
cudaError_t launch_prefill_t(const PrefillParams& p, int32_t n_groups, cudaStream_t stream) {
#if PKV_PREFILL_TC
  using C = prefill_tc::Cfg<VT, BS>;
  auto kern = prefill_tc::paged_prefill_tc_kernel<VT, BS, PREFIX>;
  constexpr int kThreads = prefill_tc::kThreads;
#else
  using C = prefill_detail::Cfg<VT, BS>;
  auto kern = prefill_detail::paged_prefill_kernel<VT, BS, PREFIX>;
  constexpr int kThreads = prefill_detail::kThreads;
#endif
  static unsigned long long configured = 0;  // one bit per device; benign race
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!(configured & (1ull << (dev & 63)))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured |= 1ull << (dev & 63);
  }
  TileMaps tm;
  memset(&tm, 0, sizeof(tm));
  const uint64_t rows = (uint64_t)p.num_blocks * p.num_kv_heads * BS;
  if (!encode_tile_map(&tm.k, p.k_codes, rows, C::K_ROW, BS)) return cudaErrorInvalidValue;
  if constexpr (C::V_SWZ) {
    if (!encode_tile_map(&tm.v, p.v_codes, rows, C::V_ROW, BS)) return cudaErrorInvalidValue;
  }
  const int col_rows = PREFIX ? p.max_group_size : p.max_q_len;
  const int chunks = (col_rows * p.group + prefill_detail::kCols - 1) / prefill_detail::kCols;
  dim3 grid(chunks, p.num_kv_heads, PREFIX ? n_groups * p.splits : p.num_seqs);
  kern<<<grid, kThreads, C::SMEM, stream>>>(p, tm);
  return cudaGetLastError();
}

}  // namespace

template <bool PREFIX>
cudaError_t launch_mode(const PrefillParams& p, int32_t n_groups, cudaStream_t stream) {
  if (p.v_dtype == PKV_INT8_SYM) {
    if (p.block_size == 16) return launch_prefill_t<PKV_INT8_SYM, 16, PREFIX>(p, n_groups, stream);
    if (p.block_size == 32) return launch_prefill_t<PKV_INT8_SYM, 32, PREFIX>(p, n_groups, stream);
  } else if (p.v_dtype == PKV_INT4_ASYM) {
    if (p.block_size == 16) return launch_prefill_t<PKV_INT4_ASYM, 16, PREFIX>(p, n_groups, stream);
    if (p.block_size == 32) return launch_prefill_t<PKV_INT4_ASYM, 32, PREFIX>(p, n_groups, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_prefill(const PrefillParams& p, cudaStream_t stream) { return launch_mode<false>(p, 0, stream); }

cudaError_t launch_prefix(const PrefillParams& p, int32_t n_groups, cudaStream_t stream) {
  return launch_mode<true>(p, n_groups, stream);
}

}  // namespace pkv
