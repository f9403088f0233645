// api.cu -- the C ABI of include/pkv.h: host-side validation, launch geometry, dispatch.
//
// Every entry point checks its arguments on the host before anything is enqueued and returns
// PKV_ERR_INVALID_ARG / PKV_ERR_UNSUPPORTED without touching device memory; a launch failure is
// reported as PKV_ERR_CUDA. Nothing here allocates device memory or keeps per-call state.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/pkv.h"
#include "internal.h"

namespace {

using namespace pkv;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool dtype_known_k(int32_t d) { return d == PKV_FP16 || d == PKV_INT8_SYM || d == PKV_FP8_E4M3; }
bool dtype_known_v(int32_t d) { return d == PKV_FP16 || d == PKV_INT8_SYM || d == PKV_INT4_ASYM || d == PKV_FP8_E4M3; }

int64_t row_bytes(int32_t dtype, int32_t head_dim) {
  if (dtype == PKV_FP16) return 2 * (int64_t)head_dim;
  if (dtype == PKV_INT4_ASYM) return head_dim / 2;
  return head_dim;  // INT8, E4M3
}

// Checks shared by every call that reads or writes the pool.
pkv_status check_desc(const pkv_cache_desc* d) {
  if (d == nullptr) return PKV_ERR_INVALID_ARG;
  if (d->num_blocks <= 0 || d->num_kv_heads <= 0 || d->head_dim <= 0 || d->block_size <= 0)
    return PKV_ERR_INVALID_ARG;
  if (d->head_dim % 16 != 0) return PKV_ERR_INVALID_ARG;
  if (!dtype_known_k(d->k_dtype) || !dtype_known_v(d->v_dtype)) return PKV_ERR_INVALID_ARG;
  if (d->block_size != 16 && d->block_size != 32) return PKV_ERR_UNSUPPORTED;
  if ((d->k_dtype == PKV_FP8_E4M3) != (d->v_dtype == PKV_FP8_E4M3)) return PKV_ERR_UNSUPPORTED;  // both or neither
  if (d->head_dim != 64 && d->head_dim != 128 && d->head_dim != 256) return PKV_ERR_UNSUPPORTED;
  if (d->k_codes == nullptr || d->v_codes == nullptr) return PKV_ERR_INVALID_ARG;
  if (!aligned(d->k_codes, 16) || !aligned(d->v_codes, 16)) return PKV_ERR_INVALID_ARG;
  if (d->k_dtype != PKV_FP16 && (d->k_scale == nullptr || !aligned(d->k_scale, 4))) return PKV_ERR_INVALID_ARG;
  if (d->v_dtype != PKV_FP16 && (d->v_scale == nullptr || !aligned(d->v_scale, 4))) return PKV_ERR_INVALID_ARG;
  if (d->v_dtype == PKV_INT4_ASYM && d->v_zp == nullptr) return PKV_ERR_INVALID_ARG;
  return PKV_OK;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int& c = cached[dev & 63];
  if (c == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    c = n;
  }
  return c;
}

// Fewest blocks a worker warp gets on average by default: smaller batches use fewer warps
// rather than cutting every (sequence, head group) into pieces that each need a merge.
constexpr int64_t kMinBlocksPerWorker = 4;

struct DecodeGeometry {
  DecodeShape shape;
  int32_t workers;          // worker warps of the persistent grid
  size_t counter_bytes;     // split-unit tickets, then the fused step's 2 barrier counters (256-byte padded)
  size_t ml_bytes;          // partial (max, sum) pairs (256-byte padded)
  size_t workspace_bytes;   // counters + (max, sum) + partial accumulators
};

// Worker warps: every resident warp of the GPU by default; with partition_tokens > 0, about one
// warp per partition_tokens tokens of the largest possible work (fewer warps, fewer splits).
pkv_status decode_geometry(const pkv_cache_desc* d, int32_t num_seqs, int32_t num_q_heads,
                           int32_t max_context_len, int32_t partition_tokens, DecodeGeometry* g) {
  if (num_seqs < 0 || num_q_heads <= 0 || max_context_len < 0 || partition_tokens < 0) return PKV_ERR_INVALID_ARG;
  if (num_q_heads % d->num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
  if (partition_tokens % d->block_size != 0) return PKV_ERR_INVALID_ARG;
  // the decode's tiled copies address a cache side's token rows with a signed 32-bit coordinate
  if ((int64_t)d->num_blocks * d->num_kv_heads * d->block_size > INT32_MAX) return PKV_ERR_UNSUPPORTED;
  const int32_t group = num_q_heads / d->num_kv_heads;
  DecodeShape& sh = g->shape;
  sh.k_dtype = d->k_dtype;
  sh.v_dtype = d->v_dtype;
  sh.block_size = d->block_size;
  sh.head_dim = d->head_dim;
  sh.heads_per_warp = decode_heads_per_warp(group, d->k_dtype, d->v_dtype, d->head_dim);
  DecodeKernelInfo info;
  if (!decode_kernel_info(sh, &info)) return PKV_ERR_UNSUPPORTED;
  const int64_t max_workers = (int64_t)sm_count() * info.ctas_per_sm * info.warps_per_cta;
  // blocks of the largest possible batch: the real total is only known on the device
  const int64_t hg = num_q_heads / sh.heads_per_warp;
  const int64_t blocks = (int64_t)num_seqs * hg * ((max_context_len + d->block_size - 1) / d->block_size);
  // blocks per worker: the requested partition, or a few blocks (one ring's worth) at least
  const int64_t per = partition_tokens > 0 ? partition_tokens / d->block_size : kMinBlocksPerWorker;
  int64_t workers = (blocks + per - 1) / per;
  workers = (workers + info.warps_per_cta - 1) / info.warps_per_cta * info.warps_per_cta;
  if (workers < info.warps_per_cta) workers = info.warps_per_cta;
  if (workers > max_workers) workers = max_workers;
  sh.grid_ctas = (int32_t)(workers / info.warps_per_cta);
  g->workers = (int32_t)workers;
  const size_t units = (size_t)num_seqs * (num_q_heads / sh.heads_per_warp);
  const size_t slots = units + (size_t)workers;
  g->counter_bytes = ((units + 2) * sizeof(uint32_t) + 255) / 256 * 256;
  g->ml_bytes = (slots * sh.heads_per_warp * 2 * sizeof(float) + 255) / 256 * 256;
  g->workspace_bytes =
      num_seqs > 0 ? g->counter_bytes + g->ml_bytes + slots * sh.heads_per_warp * d->head_dim * sizeof(float) : 0;
  return PKV_OK;
}

// Store arguments: checks and kernel parameters (T > 0).
pkv_status make_store_params(const pkv_cache_desc* desc, const void* k_new, const void* v_new,
                             const int64_t* slot_mapping, int32_t T, int32_t* dev_error, StoreParams* p) {
  if (k_new == nullptr || v_new == nullptr || slot_mapping == nullptr) return PKV_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(slot_mapping, 8)) return PKV_ERR_INVALID_ARG;
  if (dev_error != nullptr && !aligned(dev_error, 4)) return PKV_ERR_INVALID_ARG;
  p->k_codes = desc->k_codes;
  p->v_codes = desc->v_codes;
  p->k_scale = desc->k_scale;
  p->v_scale = desc->v_scale;
  p->v_zp = desc->v_zp;
  p->k_new = static_cast<const __half*>(k_new);
  p->v_new = static_cast<const __half*>(v_new);
  p->slot_mapping = slot_mapping;
  p->dev_error = dev_error;
  p->T = T;
  p->num_blocks = desc->num_blocks;
  p->num_kv_heads = desc->num_kv_heads;
  p->block_size = desc->block_size;
  p->head_dim = desc->head_dim;
  p->k_dtype = desc->k_dtype;
  p->v_dtype = desc->v_dtype;
  return PKV_OK;
}

// Copy arguments: checks and kernel parameters (n_pairs > 0).
pkv_status make_copy_params(const pkv_cache_desc* desc, const int32_t* block_mapping, int32_t n_pairs,
                            int32_t* dev_error, CopyParams* p) {
  if (block_mapping == nullptr || !aligned(block_mapping, 4)) return PKV_ERR_INVALID_ARG;
  if (dev_error != nullptr && !aligned(dev_error, 4)) return PKV_ERR_INVALID_ARG;
  p->k_codes = static_cast<uint8_t*>(desc->k_codes);
  p->v_codes = static_cast<uint8_t*>(desc->v_codes);
  p->k_scale = desc->k_dtype != PKV_FP16 ? desc->k_scale : nullptr;
  p->v_scale = desc->v_dtype != PKV_FP16 ? desc->v_scale : nullptr;
  p->v_zp = desc->v_dtype == PKV_INT4_ASYM ? desc->v_zp : nullptr;
  p->block_mapping = block_mapping;
  p->dev_error = dev_error;
  p->n_pairs = n_pairs;
  p->num_blocks = desc->num_blocks;
  p->num_kv_heads = desc->num_kv_heads;
  p->k_block_bytes = (int64_t)desc->num_kv_heads * desc->block_size * row_bytes(desc->k_dtype, desc->head_dim);
  p->v_block_bytes = (int64_t)desc->num_kv_heads * desc->block_size * row_bytes(desc->v_dtype, desc->head_dim);
  return PKV_OK;
}

// Decode arguments: checks and kernel parameters (num_seqs > 0, geometry already computed).
pkv_status make_decode_params(const pkv_cache_desc* desc, const DecodeGeometry& g, void* out, const void* q,
                              int32_t num_seqs, int32_t num_q_heads, const int32_t* block_tables,
                              int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t max_context_len,
                              float softmax_scale, void* workspace, size_t workspace_bytes, int32_t* dev_error,
                              DecodeParams* pp) {
  if (out == nullptr || q == nullptr || block_tables == nullptr || context_lens == nullptr) return PKV_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PKV_ERR_INVALID_ARG;
  if (max_blocks_per_seq <= 0) return PKV_ERR_INVALID_ARG;
  if (dev_error != nullptr && !aligned(dev_error, 4)) return PKV_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < g.workspace_bytes || !aligned(workspace, 16)) return PKV_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return PKV_ERR_INVALID_ARG;  // NaN
  DecodeParams& p = *pp;
  p.k_codes = desc->k_codes;
  p.v_codes = desc->v_codes;
  p.k_scale = desc->k_scale;
  p.v_scale = desc->v_scale;
  p.v_zp = desc->v_zp;
  p.q = static_cast<const __half*>(q);
  p.out = static_cast<__half*>(out);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.seq_order = nullptr;
  p.shared_blocks = nullptr;
  p.ws_pml = nullptr;
  p.ws_pacc = nullptr;
  p.prefix_splits = 0;
  p.max_shared_blocks = 0;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.ws_count = reinterpret_cast<uint32_t*>(ws);
  p.ws_ml = reinterpret_cast<float*>(ws + g.counter_bytes);
  p.ws_acc = reinterpret_cast<float*>(ws + g.counter_bytes + g.ml_bytes);
  p.dev_error = dev_error;
  p.num_seqs = num_seqs;
  p.num_blocks = desc->num_blocks;
  p.num_kv_heads = desc->num_kv_heads;
  p.num_q_heads = num_q_heads;
  p.group = num_q_heads / desc->num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_context_len = max_context_len;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;  // log2(e)
  return PKV_OK;
}


// Bytes of one pool array (which: 0 K codes, 1 V codes, 2 K scales, 3 V scales, 4 zero points).
size_t pool_array_bytes(const pkv_cache_desc* d, int which) {
  const size_t tiles = (size_t)d->num_blocks * d->num_kv_heads;
  switch (which) {
    case 0: return tiles * d->block_size * row_bytes(d->k_dtype, d->head_dim);
    case 1: return tiles * d->block_size * row_bytes(d->v_dtype, d->head_dim);
    case 2: return d->k_dtype != PKV_FP16 ? tiles * sizeof(float) : 0;
    case 3: return d->v_dtype != PKV_FP16 ? tiles * sizeof(float) : 0;
    default: return d->v_dtype == PKV_INT4_ASYM ? tiles : 0;
  }
}

// The address through which the current device reaches [p, p + bytes), or nullptr when the range
// is not entirely of the wanted kind: memory of the current device (host == false), or page-locked
// host memory mapped into the device's address space (host == true). Both ends are checked.
const void* device_view(const void* p, size_t bytes, bool host) {
  if (p == nullptr || bytes == 0) return nullptr;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  cudaPointerAttributes a, b;
  const char* last = static_cast<const char*>(p) + (bytes - 1);
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess || cudaPointerGetAttributes(&b, last) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (host) {
    if (a.type != cudaMemoryTypeHost || b.type != cudaMemoryTypeHost) return nullptr;
    if (a.devicePointer == nullptr || b.devicePointer == nullptr) return nullptr;
    if (static_cast<const char*>(b.devicePointer) - static_cast<const char*>(a.devicePointer) != (ptrdiff_t)(bytes - 1))
      return nullptr;
    return a.devicePointer;
  }
  const bool ok_a = a.type == cudaMemoryTypeManaged || (a.type == cudaMemoryTypeDevice && a.device == dev);
  const bool ok_b = b.type == cudaMemoryTypeManaged || (b.type == cudaMemoryTypeDevice && b.device == dev);
  return ok_a && ok_b ? p : nullptr;
}

// The shared-prefix pass of pkv_paged_attention_decode_ex: how the shared blocks are cut among CTAs
// and where its partials go in the workspace (after the decode's own regions).
struct PrefixPlan {
  bool on = false;
  int32_t splits = 0, per_split = 0;
  size_t pml_off = 0, pacc_off = 0, total = 0;
};

pkv_status prefix_plan(const pkv_cache_desc* d, const DecodeGeometry& g, int32_t num_seqs, int32_t num_q_heads,
                       const pkv_decode_options* o, PrefixPlan* pl) {
  pl->total = g.workspace_bytes;
  if (o == nullptr || o->num_prefix_groups == 0 || num_seqs == 0) return PKV_OK;
  if (o->num_prefix_groups < 0 || o->num_prefix_groups > 65535) return PKV_ERR_INVALID_ARG;
  if (!prefill_supported(d->k_dtype, d->v_dtype, d->block_size, d->head_dim)) return PKV_ERR_UNSUPPORTED;
  if (o->max_group_size <= 0 || o->max_shared_blocks < 0 || o->num_prefix_members <= 0) return PKV_ERR_INVALID_ARG;
  if (o->prefix_group_start == nullptr || o->prefix_members == nullptr || o->shared_blocks == nullptr)
    return PKV_ERR_INVALID_ARG;
  if (!aligned(o->prefix_group_start, 4) || !aligned(o->prefix_members, 4) || !aligned(o->shared_blocks, 4))
    return PKV_ERR_INVALID_ARG;
  const int32_t group = num_q_heads / d->num_kv_heads;
  const int64_t chunks = ((int64_t)o->max_group_size * group + 127) / 128;
  const int64_t ctas = (int64_t)o->num_prefix_groups * d->num_kv_heads * chunks;
  if (chunks > INT32_MAX || d->num_kv_heads > 65535) return PKV_ERR_UNSUPPORTED;
  // about one CTA per SM in all (the pass runs one CTA per SM), at most 16 parts, each a whole
  // number of the pass's 64-token steps: every part adds a partial state per member and head,
  // written once and read once by the decode
  const int64_t step = 64 / d->block_size;
  int64_t splits = ((int64_t)sm_count() + ctas - 1) / ctas;
  splits = splits < 1 ? 1 : (splits > 16 ? 16 : splits);
  int64_t per = o->max_shared_blocks > 0 ? (o->max_shared_blocks + splits - 1) / splits : 1;
  per = (per + step - 1) / step * step;
  splits = o->max_shared_blocks > 0 ? (o->max_shared_blocks + per - 1) / per : 1;
  if ((int64_t)o->num_prefix_groups * splits > 65535) return PKV_ERR_UNSUPPORTED;  // grid z
  pl->on = true;
  pl->splits = (int32_t)splits;
  pl->per_split = (int32_t)per;
  const size_t gt = (size_t)g.shape.heads_per_warp;
  const size_t slots = (size_t)num_seqs * (num_q_heads / gt) * (size_t)splits;
  pl->pml_off = (g.workspace_bytes + 255) / 256 * 256;
  pl->pacc_off = pl->pml_off + (slots * gt * 2 * sizeof(float) + 255) / 256 * 256;
  pl->total = pl->pacc_off + slots * gt * d->head_dim * sizeof(float);
  return PKV_OK;
}

// Any memory the device can dereference (its own, or mapped host memory): the address to use.
const void* device_view_any(const void* p, size_t bytes) {
  const void* v = device_view(p, bytes, false);
  return v != nullptr ? v : device_view(p, bytes, true);
}

}  // namespace

extern "C" {

const char* pkv_status_string(pkv_status status) {
  switch (status) {
    case PKV_OK: return "PKV_OK";
    case PKV_ERR_INVALID_ARG: return "PKV_ERR_INVALID_ARG";
    case PKV_ERR_UNSUPPORTED: return "PKV_ERR_UNSUPPORTED";
    case PKV_ERR_OUT_OF_BLOCKS: return "PKV_ERR_OUT_OF_BLOCKS";
    case PKV_ERR_CUDA: return "PKV_ERR_CUDA";
    case PKV_ERR_DEVICE_TIMEOUT: return "PKV_ERR_DEVICE_TIMEOUT";
  }
  return "PKV_ERR_UNKNOWN";
}

size_t pkv_tile_bytes(const pkv_cache_desc* desc, int32_t which_v) {
  if (desc == nullptr || desc->head_dim <= 0 || desc->block_size <= 0) return 0;
  const int32_t dt = which_v ? desc->v_dtype : desc->k_dtype;
  if (which_v ? !dtype_known_v(dt) : !dtype_known_k(dt)) return 0;
  return (size_t)desc->block_size * (size_t)row_bytes(dt, desc->head_dim);
}

pkv_status pkv_store_quantized(const pkv_cache_desc* desc, const void* k_new, const void* v_new,
                               const int64_t* slot_mapping, int32_t T, int32_t* dev_error, pkv_stream_t stream) {
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  if (T < 0) return PKV_ERR_INVALID_ARG;
  if (T == 0) return PKV_OK;
  StoreParams p;
  st = make_store_params(desc, k_new, v_new, slot_mapping, T, dev_error, &p);
  if (st != PKV_OK) return st;
  return launch_store(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_decode_workspace_size(const pkv_cache_desc* desc, int32_t num_seqs, int32_t num_q_heads,
                                     int32_t max_context_len, int32_t partition_tokens, size_t* bytes) {
  if (bytes == nullptr) return PKV_ERR_INVALID_ARG;
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  DecodeGeometry g;
  st = decode_geometry(desc, num_seqs, num_q_heads, max_context_len, partition_tokens, &g);
  if (st != PKV_OK) return st;
  *bytes = g.workspace_bytes;
  return PKV_OK;
}

pkv_status pkv_decode_partitioning(const pkv_cache_desc* desc, int32_t num_seqs, int32_t num_q_heads,
                                   int32_t max_context_len, int32_t partition_tokens, int32_t* num_workers_out,
                                   int32_t* num_ctas_out) {
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  DecodeGeometry g;
  st = decode_geometry(desc, num_seqs, num_q_heads, max_context_len, partition_tokens, &g);
  if (st != PKV_OK) return st;
  if (num_workers_out) *num_workers_out = g.workers;
  if (num_ctas_out) *num_ctas_out = g.shape.grid_ctas;
  return PKV_OK;
}

pkv_status pkv_paged_attention_decode(const pkv_cache_desc* desc, void* out, const void* q, int32_t num_seqs,
                                      int32_t num_q_heads, const int32_t* block_tables, int32_t max_blocks_per_seq,
                                      const int32_t* context_lens, int32_t max_context_len, float softmax_scale,
                                      int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                                      int32_t* dev_error, pkv_stream_t stream) {
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  if (!decode_supported(desc->k_dtype, desc->v_dtype, desc->block_size, desc->head_dim)) return PKV_ERR_UNSUPPORTED;
  DecodeGeometry g;
  st = decode_geometry(desc, num_seqs, num_q_heads, max_context_len, partition_tokens, &g);
  if (st != PKV_OK) return st;
  if (num_seqs == 0) return PKV_OK;
  DecodeParams p;
  st = make_decode_params(desc, g, out, q, num_seqs, num_q_heads, block_tables, max_blocks_per_seq, context_lens,
                          max_context_len, softmax_scale, workspace, workspace_bytes, dev_error, &p);
  if (st != PKV_OK) return st;
  return launch_decode(p, g.shape, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_decode_ex_workspace_size(const pkv_cache_desc* desc, int32_t num_seqs, int32_t num_q_heads,
                                        int32_t max_context_len, int32_t partition_tokens,
                                        const pkv_decode_options* options, size_t* bytes) {
  if (bytes == nullptr) return PKV_ERR_INVALID_ARG;
  if (options != nullptr && options->struct_bytes != sizeof(pkv_decode_options))
    return options->struct_bytes < sizeof(size_t) ? PKV_ERR_INVALID_ARG : PKV_ERR_UNSUPPORTED;
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  DecodeGeometry g;
  st = decode_geometry(desc, num_seqs, num_q_heads, max_context_len, partition_tokens, &g);
  if (st != PKV_OK) return st;
  PrefixPlan pl;
  st = prefix_plan(desc, g, num_seqs, num_q_heads, options, &pl);
  if (st != PKV_OK) return st;
  *bytes = pl.total;
  return PKV_OK;
}

pkv_status pkv_paged_attention_decode_ex(const pkv_cache_desc* desc, void* out, const void* q, int32_t num_seqs,
                                         int32_t num_q_heads, const int32_t* block_tables,
                                         int32_t max_blocks_per_seq, const int32_t* context_lens,
                                         int32_t max_context_len, float softmax_scale, int32_t partition_tokens,
                                         const pkv_decode_options* options, void* workspace, size_t workspace_bytes,
                                         int32_t* dev_error, pkv_stream_t stream) {
  if (options != nullptr && options->struct_bytes != sizeof(pkv_decode_options))
    return options->struct_bytes < sizeof(size_t) ? PKV_ERR_INVALID_ARG : PKV_ERR_UNSUPPORTED;
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  if (!decode_supported(desc->k_dtype, desc->v_dtype, desc->block_size, desc->head_dim)) return PKV_ERR_UNSUPPORTED;
  DecodeGeometry g;
  st = decode_geometry(desc, num_seqs, num_q_heads, max_context_len, partition_tokens, &g);
  if (st != PKV_OK) return st;
  PrefixPlan pl;
  st = prefix_plan(desc, g, num_seqs, num_q_heads, options, &pl);
  if (st != PKV_OK) return st;
  if (num_seqs == 0) return PKV_OK;
  if (workspace_bytes < pl.total) return PKV_ERR_INVALID_ARG;
  DecodeParams p;
  st = make_decode_params(desc, g, out, q, num_seqs, num_q_heads, block_tables, max_blocks_per_seq, context_lens,
                          max_context_len, softmax_scale, workspace, workspace_bytes, dev_error, &p);
  if (st != PKV_OK) return st;
  if (options != nullptr && options->seq_order != nullptr) {
    if (!aligned(options->seq_order, 4)) return PKV_ERR_INVALID_ARG;
    p.seq_order = options->seq_order;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (pl.on) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    PrefillParams pp = {};
    pp.k_codes = desc->k_codes;
    pp.v_codes = desc->v_codes;
    pp.k_scale = desc->k_scale;
    pp.v_scale = desc->v_scale;
    pp.v_zp = desc->v_zp;
    pp.q = static_cast<const __half*>(q);
    pp.block_tables = block_tables;
    pp.context_lens = context_lens;
    pp.dev_error = dev_error;
    pp.num_seqs = num_seqs;
    pp.num_blocks = desc->num_blocks;
    pp.num_kv_heads = desc->num_kv_heads;
    pp.num_q_heads = num_q_heads;
    pp.group = num_q_heads / desc->num_kv_heads;
    pp.max_blocks_per_seq = max_blocks_per_seq;
    pp.max_context_len = max_context_len;
    pp.block_size = desc->block_size;
    pp.v_dtype = desc->v_dtype;
    pp.scale_log2 = p.scale_log2;
    pp.group_start = options->prefix_group_start;
    pp.members = options->prefix_members;
    pp.shared_blocks = options->shared_blocks;
    pp.pml = reinterpret_cast<float*>(ws + pl.pml_off);
    pp.pacc = reinterpret_cast<float*>(ws + pl.pacc_off);
    pp.n_members = options->num_prefix_members;
    pp.max_group_size = options->max_group_size;
    pp.max_shared_blocks = options->max_shared_blocks;
    pp.splits = pl.splits;
    pp.per_split = pl.per_split;
    pp.gt = g.shape.heads_per_warp;
    if (launch_prefix(pp, options->num_prefix_groups, s) != cudaSuccess) return PKV_ERR_CUDA;
    p.shared_blocks = options->shared_blocks;
    p.ws_pml = pp.pml;
    p.ws_pacc = pp.pacc;
    p.prefix_splits = pl.splits;
    p.max_shared_blocks = options->max_shared_blocks;
  }
  return launch_decode(p, g.shape, s) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_paged_attention_prefill(const pkv_cache_desc* desc, void* out, const void* q, int32_t num_seqs,
                                       int32_t num_q_heads, const int32_t* cu_q_lens, int32_t total_q,
                                       int32_t max_q_len, const int32_t* block_tables, int32_t max_blocks_per_seq,
                                       const int32_t* context_lens, int32_t max_context_len, float softmax_scale,
                                       int32_t* dev_error, pkv_stream_t stream) {
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || total_q < 0 || max_q_len < 0 || max_context_len < 0)
    return PKV_ERR_INVALID_ARG;
  if (num_q_heads % desc->num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
  if (!prefill_supported(desc->k_dtype, desc->v_dtype, desc->block_size, desc->head_dim)) return PKV_ERR_UNSUPPORTED;
  if (num_seqs == 0 || total_q == 0 || max_q_len == 0) return PKV_OK;
  if (out == nullptr || q == nullptr || cu_q_lens == nullptr || block_tables == nullptr || context_lens == nullptr)
    return PKV_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(cu_q_lens, 4) || !aligned(block_tables, 4) ||
      !aligned(context_lens, 4))
    return PKV_ERR_INVALID_ARG;
  if (max_blocks_per_seq <= 0) return PKV_ERR_INVALID_ARG;
  if (dev_error != nullptr && !aligned(dev_error, 4)) return PKV_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return PKV_ERR_INVALID_ARG;
  const int32_t group = num_q_heads / desc->num_kv_heads;
  const int64_t chunks = ((int64_t)max_q_len * group + 127) / 128;
  if (num_seqs > 65535 || desc->num_kv_heads > 65535 || chunks > INT32_MAX) return PKV_ERR_UNSUPPORTED;
  PrefillParams p;
  p.k_codes = desc->k_codes;
  p.v_codes = desc->v_codes;
  p.k_scale = desc->k_scale;
  p.v_scale = desc->v_scale;
  p.v_zp = desc->v_zp;
  p.q = static_cast<const __half*>(q);
  p.out = static_cast<__half*>(out);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.cu_q_lens = cu_q_lens;
  p.dev_error = dev_error;
  p.num_seqs = num_seqs;
  p.num_blocks = desc->num_blocks;
  p.num_kv_heads = desc->num_kv_heads;
  p.num_q_heads = num_q_heads;
  p.group = group;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_context_len = max_context_len;
  p.max_q_len = max_q_len;
  p.total_q = total_q;
  p.block_size = desc->block_size;
  p.v_dtype = desc->v_dtype;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;  // log2(e)
  return launch_prefill(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_copy_blocks(const pkv_cache_desc* desc, const int32_t* block_mapping, int32_t n_pairs,
                           int32_t* dev_error, pkv_stream_t stream) {
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  if (n_pairs < 0) return PKV_ERR_INVALID_ARG;
  if (n_pairs == 0) return PKV_OK;
  CopyParams p;
  st = make_copy_params(desc, block_mapping, n_pairs, dev_error, &p);
  if (st != PKV_OK) return st;
  return launch_copy(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_decode_step(const pkv_cache_desc* desc, const int32_t* block_mapping, int32_t n_pairs, const void* k_new,
                           const void* v_new, const int64_t* slot_mapping, int32_t T, void* out, const void* q,
                           int32_t num_seqs, int32_t num_q_heads, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t max_context_len,
                           float softmax_scale, int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                           int32_t* dev_error, pkv_stream_t stream) {
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  if (n_pairs < 0 || T < 0) return PKV_ERR_INVALID_ARG;
  if (!decode_supported(desc->k_dtype, desc->v_dtype, desc->block_size, desc->head_dim)) return PKV_ERR_UNSUPPORTED;
  DecodeGeometry g;
  st = decode_geometry(desc, num_seqs, num_q_heads, max_context_len, partition_tokens, &g);
  if (st != PKV_OK) return st;
  StepParams sp = {};
  sp.fused = 1;
  if (n_pairs > 0) {
    st = make_copy_params(desc, block_mapping, n_pairs, dev_error, &sp.copy);
    if (st != PKV_OK) return st;
  }
  if (T > 0) {
    st = make_store_params(desc, k_new, v_new, slot_mapping, T, dev_error, &sp.store);
    if (st != PKV_OK) return st;
  }
  DecodeParams p;
  if (num_seqs > 0) {
    st = make_decode_params(desc, g, out, q, num_seqs, num_q_heads, block_tables, max_blocks_per_seq, context_lens,
                            max_context_len, softmax_scale, workspace, workspace_bytes, dev_error, &p);
    if (st != PKV_OK) return st;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (num_seqs == 0 || (n_pairs == 0 && T == 0)) {  // nothing to fuse: the separate launches
    if (n_pairs > 0 && launch_copy(sp.copy, s) != cudaSuccess) return PKV_ERR_CUDA;
    if (T > 0 && launch_store(sp.store, s) != cudaSuccess) return PKV_ERR_CUDA;
    if (num_seqs > 0 && launch_decode(p, g.shape, s) != cudaSuccess) return PKV_ERR_CUDA;
    return PKV_OK;
  }
  sp.bar = p.ws_count + (size_t)num_seqs * (num_q_heads / g.shape.heads_per_warp);
  return launch_decode_step(p, sp, g.shape, s) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_swap_blocks(const pkv_cache_desc* device_pool, const pkv_cache_desc* host_pool,
                           const int32_t* block_mapping, int32_t n_pairs, int32_t direction, int32_t* dev_error,
                           pkv_stream_t stream) {
  pkv_status st = check_desc(device_pool);
  if (st != PKV_OK) return st;
  st = check_desc(host_pool);
  if (st != PKV_OK) return st;
  const pkv_cache_desc *dv = device_pool, *hv = host_pool;
  if (dv->block_size != hv->block_size || dv->num_kv_heads != hv->num_kv_heads || dv->head_dim != hv->head_dim ||
      dv->k_dtype != hv->k_dtype || dv->v_dtype != hv->v_dtype)
    return PKV_ERR_INVALID_ARG;
  if (direction != PKV_SWAP_OUT && direction != PKV_SWAP_IN) return PKV_ERR_INVALID_ARG;
  if (n_pairs < 0) return PKV_ERR_INVALID_ARG;
  if (n_pairs == 0) return PKV_OK;
  if (block_mapping == nullptr || !aligned(block_mapping, 4)) return PKV_ERR_INVALID_ARG;
  if (dev_error != nullptr && !aligned(dev_error, 4)) return PKV_ERR_INVALID_ARG;
  // where every array lives, as the device sees it (nothing is launched unless all check out)
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  const void* arr_d[5] = {dv->k_codes, dv->v_codes, dv->k_scale, dv->v_scale, dv->v_zp};
  const void* arr_h[5] = {hv->k_codes, hv->v_codes, hv->k_scale, hv->v_scale, hv->v_zp};
  const void* view_d[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  const void* view_h[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  for (int i = 0; i < 5; ++i) {
    const size_t nd = pool_array_bytes(dv, i), nh = pool_array_bytes(hv, i);
    if (nd == 0) continue;  // the side has no such array (FP16 scales, zero points of INT8)
    view_d[i] = device_view(arr_d[i], nd, false);
    view_h[i] = device_view(arr_h[i], nh, true);
    if (view_d[i] == nullptr || view_h[i] == nullptr) return PKV_ERR_INVALID_ARG;
  }
  const void* map_view = device_view_any(block_mapping, (size_t)n_pairs * 2 * sizeof(int32_t));
  if (map_view == nullptr) return PKV_ERR_INVALID_ARG;
  int32_t* err_view = nullptr;
  if (dev_error != nullptr) {
    err_view = static_cast<int32_t*>(const_cast<void*>(device_view_any(dev_error, sizeof(int32_t))));
    if (err_view == nullptr) return PKV_ERR_INVALID_ARG;
  }
  const bool out = direction == PKV_SWAP_OUT;
  const void* const* src = out ? view_d : view_h;
  const void* const* dst = out ? view_h : view_d;
  SwapParams p;
  p.src_k = static_cast<const uint8_t*>(src[0]);
  p.src_v = static_cast<const uint8_t*>(src[1]);
  p.src_ks = static_cast<const float*>(src[2]);
  p.src_vs = static_cast<const float*>(src[3]);
  p.src_zp = static_cast<const uint8_t*>(src[4]);
  p.dst_k = static_cast<uint8_t*>(const_cast<void*>(dst[0]));
  p.dst_v = static_cast<uint8_t*>(const_cast<void*>(dst[1]));
  p.dst_ks = static_cast<float*>(const_cast<void*>(dst[2]));
  p.dst_vs = static_cast<float*>(const_cast<void*>(dst[3]));
  p.dst_zp = static_cast<uint8_t*>(const_cast<void*>(dst[4]));
  p.block_mapping = static_cast<const int32_t*>(map_view);
  p.dev_error = err_view;
  p.n_pairs = n_pairs;
  p.src_blocks = out ? dv->num_blocks : hv->num_blocks;
  p.dst_blocks = out ? hv->num_blocks : dv->num_blocks;
  p.num_kv_heads = dv->num_kv_heads;
  p.k_block_bytes = (int64_t)dv->num_kv_heads * dv->block_size * row_bytes(dv->k_dtype, dv->head_dim);
  p.v_block_bytes = (int64_t)dv->num_kv_heads * dv->block_size * row_bytes(dv->v_dtype, dv->head_dim);
  return launch_swap(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// ---- decode without caller-provided scratch -------------------------------------------------
// Scratch for pkv_paged_attention_decode_static: one array per device, alive while the library
// is loaded. In host code the name below stands for a host-side shadow, not a device address, so
// the device address is looked up (per device, with that device current) before any use.
static __device__ __align__(256) unsigned char g_static_scratch[PKV_STATIC_SCRATCH_BYTES];

static void* static_scratch_on_current_device(cudaError_t* err) {
  static void* cached[64] = {nullptr};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (cached[dev] == nullptr) {
    void* ptr = nullptr;
    *err = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (*err != cudaSuccess) return nullptr;
    cached[dev] = ptr;
  }
  return cached[dev];
}

pkv_status pkv_paged_attention_decode_static(const pkv_cache_desc* desc, void* out, const void* q, int32_t num_seqs,
                                             int32_t num_q_heads, const int32_t* block_tables,
                                             int32_t max_blocks_per_seq, const int32_t* context_lens,
                                             int32_t max_context_len, float softmax_scale, int32_t partition_tokens,
                                             int32_t* dev_error, pkv_stream_t stream) {
  pkv_status st = check_desc(desc);
  if (st != PKV_OK) return st;
  if (!decode_supported(desc->k_dtype, desc->v_dtype, desc->block_size, desc->head_dim)) return PKV_ERR_UNSUPPORTED;
  DecodeGeometry g;
  st = decode_geometry(desc, num_seqs, num_q_heads, max_context_len, partition_tokens, &g);
  if (st != PKV_OK) return st;
  if (num_seqs == 0) return PKV_OK;
  if (g.workspace_bytes > PKV_STATIC_SCRATCH_BYTES) return PKV_ERR_UNSUPPORTED;  // too large for the array
  cudaError_t err = cudaSuccess;
  void* scratch = static_scratch_on_current_device(&err);
  if (scratch == nullptr) return PKV_ERR_CUDA;
  // every argument is checked before anything is enqueued
  DecodeParams p;
  st = make_decode_params(desc, g, out, q, num_seqs, num_q_heads, block_tables, max_blocks_per_seq, context_lens,
                          max_context_len, softmax_scale, scratch, PKV_STATIC_SCRATCH_BYTES, dev_error, &p);
  if (st != PKV_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the tickets must start at zero: the array holds whatever the previous call left
  if (cudaMemsetAsync(scratch, 0, g.counter_bytes, s) != cudaSuccess) return PKV_ERR_CUDA;
  return launch_decode(p, g.shape, s) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_static_scratch_address(void** device_ptr, size_t* bytes) {
  if (device_ptr == nullptr) return PKV_ERR_INVALID_ARG;
  cudaError_t err = cudaSuccess;
  void* scratch = static_scratch_on_current_device(&err);
  if (scratch == nullptr) return PKV_ERR_CUDA;
  *device_ptr = scratch;
  if (bytes != nullptr) *bytes = PKV_STATIC_SCRATCH_BYTES;
  return PKV_OK;
}

}  // extern "C"
