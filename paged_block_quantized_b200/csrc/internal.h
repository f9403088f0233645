// internal.h -- kernel launch interfaces behind the C ABI (not part of the public header).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pkv.h"

namespace pkv {

// ---------------------------------------------------------------- decode
struct DecodeParams {
  const void* k_codes;
  const void* v_codes;
  const float* k_scale;
  const float* v_scale;
  const uint8_t* v_zp;
  const __half* q;
  __half* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* seq_order;  // [S] walk order of the sequences, or NULL (index order)
  // shared-prefix decode: the first shared_blocks[s] blocks of sequence s were attended by the
  // prefix pass, whose prefix_splits partials per (sequence, head group) the merge folds in
  const int32_t* shared_blocks;  // [S] or NULL
  const float* ws_pml;           // [(S*HG) * prefix_splits][GT][2]
  const float* ws_pacc;          // [(S*HG) * prefix_splits][GT][D]
  int32_t prefix_splits;
  int32_t max_shared_blocks;     // host bound: counts above it are clamped (and reported)
  uint32_t* ws_count;  // [S * HG] tickets of split units (zero between calls)
  float* ws_ml;        // [(S*HG + W) * GT][2] partial running max (log2 domain) and sum
  float* ws_acc;       // [(S*HG + W) * GT][D] partial un-normalised accumulators
  int32_t* dev_error;
  int32_t num_seqs;
  int32_t num_blocks;
  int32_t num_kv_heads;
  int32_t num_q_heads;
  int32_t group;  // num_q_heads / num_kv_heads
  int32_t max_blocks_per_seq;
  int32_t max_context_len;
  float scale_log2;  // softmax_scale * log2(e)
};

struct DecodeShape {
  int32_t k_dtype, v_dtype, block_size, head_dim;
  int32_t heads_per_warp;  // query heads of one KV group handled together (divides group)
  int32_t grid_ctas;       // persistent grid size
};

struct DecodeKernelInfo {
  int32_t warps_per_cta;
  int32_t ctas_per_sm;  // resident CTAs per SM the kernel is built for
  int32_t smem_bytes;
  int32_t stages;       // copy-ring depth per warp
};

// Query heads handled together by one warp: 8 (tensor cores, when the dtypes allow) or the
// largest of 4, 2, 1 that divides the group.
int32_t decode_heads_per_warp(int32_t group, int32_t k_dtype, int32_t v_dtype, int32_t head_dim);
bool decode_supported(int32_t k_dtype, int32_t v_dtype, int32_t block_size, int32_t head_dim);
// Static launch facts of the kernel instantiation for `sh` (no device needed); false if none.
bool decode_kernel_info(const DecodeShape& sh, DecodeKernelInfo* info);

cudaError_t launch_decode(const DecodeParams& p, const DecodeShape& sh, cudaStream_t stream);
// Grouped-query decode on tcgen05 (gqa_tc.cuh): INT8 K, INT8 / INT4 V, D 128, 8 heads per unit. The
// (non-fused) decode takes it for these shapes; `workers` bounds its partial slots as the
// workspace was sized (units + workers).
bool gqa_tc_eligible(const DecodeShape& sh, int32_t num_seqs, int32_t num_q_heads);
cudaError_t launch_gqa_tc(const DecodeParams& p, const DecodeShape& sh, int64_t workers, cudaStream_t stream);

// Tensor maps of the K and V code pools for the tensor-core engine's tiled copies: the pool as
// rows of `row_bytes` (a multiple of 128; 2-D, or 3-D in 128-byte units), boxes of `box_rows`
// rows, 128-byte swizzle. False if the driver cannot encode it.
struct TileMaps {
  CUtensorMap k;
  CUtensorMap v;
};
bool encode_tile_map(CUtensorMap* map, const void* base, uint64_t rows, int row_bytes, int box_rows);

// ---------------------------------------------------------------- store
struct StoreParams {
  void* k_codes;
  void* v_codes;
  float* k_scale;
  float* v_scale;
  uint8_t* v_zp;
  const __half* k_new;
  const __half* v_new;
  const int64_t* slot_mapping;
  int32_t* dev_error;
  int32_t T;
  int32_t num_blocks;
  int32_t num_kv_heads;
  int32_t block_size;
  int32_t head_dim;
  int32_t k_dtype;
  int32_t v_dtype;
};
cudaError_t launch_store(const StoreParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- copy
struct CopyParams {
  uint8_t* k_codes;
  uint8_t* v_codes;
  float* k_scale;
  float* v_scale;
  uint8_t* v_zp;
  const int32_t* block_mapping;
  int32_t* dev_error;
  int32_t n_pairs;
  int32_t num_blocks;
  int32_t num_kv_heads;
  int64_t k_block_bytes;  // bytes of one block of K codes (all heads)
  int64_t v_block_bytes;
};
cudaError_t launch_copy(const CopyParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- swap
// Whole blocks from one pool to another of the same geometry (device <-> pinned host memory);
// every pointer is an address the device can dereference.
struct SwapParams {
  const uint8_t* src_k;
  const uint8_t* src_v;
  const float* src_ks;   // NULL when the side is FP16 (then dst_ks unused too)
  const float* src_vs;
  const uint8_t* src_zp; // NULL unless V is INT4
  uint8_t* dst_k;
  uint8_t* dst_v;
  float* dst_ks;
  float* dst_vs;
  uint8_t* dst_zp;
  const int32_t* block_mapping;  // [n_pairs][2] = {src block, dst block}
  int32_t* dev_error;
  int32_t n_pairs;
  int32_t src_blocks;
  int32_t dst_blocks;
  int32_t num_kv_heads;
  int64_t k_block_bytes;
  int64_t v_block_bytes;
};
cudaError_t launch_swap(const SwapParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- chunked prefill
struct PrefillParams {
  const void* k_codes;
  const void* v_codes;
  const float* k_scale;
  const float* v_scale;
  const uint8_t* v_zp;
  const __half* q;
  __half* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* cu_q_lens;  // [S+1] rows of each sequence's chunk in q / out
  int32_t* dev_error;
  int32_t num_seqs;
  int32_t num_blocks;
  int32_t num_kv_heads;
  int32_t num_q_heads;
  int32_t group;
  int32_t max_blocks_per_seq;
  int32_t max_context_len;
  int32_t max_q_len;
  int32_t total_q;
  int32_t block_size;
  int32_t v_dtype;
  float scale_log2;
  // shared-prefix pass of the decode (the same kernel in its prefix mode)
  const int32_t* group_start;    // [groups + 1] offsets into members
  const int32_t* members;        // sequence ids of the groups, one after another
  const int32_t* shared_blocks;  // [S] leading blocks shared with the group
  float* pml;                    // partials out: [(S * Hq/gt) * splits][gt][2] (max in log2 units, sum)
  float* pacc;                   // [(S * Hq/gt) * splits][gt][D]
  int32_t n_members;
  int32_t max_group_size;
  int32_t splits;                // shared blocks cut into this many parts (one CTA each)
  int32_t per_split;
  int32_t gt;                    // query heads per head group of the decode
  int32_t max_shared_blocks;     // host bound, clamped as the decode clamps it
};
bool prefill_supported(int32_t k_dtype, int32_t v_dtype, int32_t block_size, int32_t head_dim);
cudaError_t launch_prefill(const PrefillParams& p, cudaStream_t stream);
// the prefix mode: grid (column chunks of the largest group, KV heads, groups x splits)
cudaError_t launch_prefix(const PrefillParams& p, int32_t n_groups, cudaStream_t stream);

// ---------------------------------------------------------------- fused step
// Copy-on-write copies, then the store, then the decode, in one cooperative launch of the decode
// kernel: every warp takes part in the copies and the stores, with a grid-wide barrier after each
// phase, before any decode read of the pool.
struct StepParams {
  int32_t fused;  // 0: decode only (the other fields are unused)
  CopyParams copy;
  StoreParams store;
  uint32_t* bar;  // [2] in the workspace: barrier arrivals, warps done (zero between calls)
};
cudaError_t launch_decode_step(const DecodeParams& p, const StepParams& sp, const DecodeShape& sh,
                               cudaStream_t stream);
// per dtype pair (decode_i8i8.cu, decode_i8i4.cu, decode_f16.cu, decode_fp8.cu)
cudaError_t launch_decode_i8i8(const DecodeParams&, const StepParams&, const DecodeShape&, cudaStream_t);
cudaError_t launch_decode_i8i4(const DecodeParams&, const StepParams&, const DecodeShape&, cudaStream_t);
cudaError_t launch_decode_f16(const DecodeParams&, const StepParams&, const DecodeShape&, cudaStream_t);
cudaError_t launch_decode_fp8(const DecodeParams&, const StepParams&, const DecodeShape&, cudaStream_t);
bool decode_info_i8i8(const DecodeShape&, DecodeKernelInfo*);
bool decode_info_i8i4(const DecodeShape&, DecodeKernelInfo*);
bool decode_info_f16(const DecodeShape&, DecodeKernelInfo*);
bool decode_info_fp8(const DecodeShape&, DecodeKernelInfo*);

}  // namespace pkv
