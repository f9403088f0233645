/*
 * pkv.h -- C ABI of a paged, block-quantized KV cache for decode-phase attention (sm_100a).
 *
 * Sources the operations follow (web pages; cited by page and section):
 *   [tbr8]      tbr8.org, "如何通过 PagedAttention 与分块量化结合：解决移动端内存碎片化导致的长文本 OOM"
 *               (PagedAttention + group-wise block quantization against long-context OOM on phones).
 *   [deepinsea] deepinsea.top, "PagedAttention 内存管理深度解析" (PagedAttention memory management).
 *   [yunthe]    yunthe.com, "LLM推理显存优化KV Cache量化与PagedAttention实现详解"
 *               (KV-cache quantization and PagedAttention).
 *
 * What lives where
 *   - The KV cache is a pool of fixed-size physical blocks ([tbr8] §2 "PagedAttention 虚拟化管理";
 *     [yunthe] section "PagedAttention分页注意力机制与vLLM实现", block_table data structure).
 *     A block holds block_size tokens (16 or 32, [deepinsea] section "块大小选择") of every KV head.
 *   - Each (block, KV head) tile is quantized on its own ([tbr8] §3 "分块量化", §4 store_kv):
 *     K is INT8 symmetric with scale = absmax/127; V is INT8 symmetric or INT4 asymmetric with
 *     Q(x) = clamp(round(x/scale + zp), 0, 2^bits - 1) and x_hat = (Q - zp) * scale
 *     ([yunthe] section "KV Cache量化技术原理", quantize and dequantize formulas; K INT8 / V INT4
 *     split from [tbr8] §5 item 1). An unquantized FP16 cache is supported for comparison
 *     ([yunthe] section "vLLM推理引擎部署", --kv-cache-dtype fp16 vs int8).
 *   - Dequantization happens inside the attention kernel; no fp16 copy of the cache is ever
 *     written ([tbr8] §5 item 2, fused QuantizedPagedAttention operator).
 *
 * Device memory layout (all row-major, all owned by the caller):
 *   k_codes  [num_blocks][num_kv_heads][block_size][head_dim]   int8   (PKV_INT8_SYM)
 *                                                              fp16   (PKV_FP16)
 *                                                              E4M3   (PKV_FP8_E4M3)
 *   v_codes  [num_blocks][num_kv_heads][block_size][head_dim]   int8 / fp16 / E4M3
 *            [num_blocks][num_kv_heads][block_size][head_dim/2] uint8  (PKV_INT4_ASYM):
 *            byte j of a token row = code[2j] | code[2j+1] << 4 (low nibble = even dim)
 *   k_scale, v_scale [num_blocks][num_kv_heads] fp32   (NULL for an FP16 cache side)
 *   v_zp     [num_blocks][num_kv_heads] uint8           (PKV_INT4_ASYM only, else NULL)
 *   q, out   [num_seqs][num_q_heads][head_dim] fp16
 *   block_tables [num_seqs][max_blocks_per_seq] int32: logical block i of sequence s lives in
 *            physical block block_tables[s][i]
 *   context_lens [num_seqs] int32 (tokens to attend over, including the token just stored)
 *   slot_mapping [T] int64: slot = physical_block * block_size + offset; a negative slot skips
 *            that token
 *   new k, v [T][num_kv_heads][head_dim] fp16
 *
 * Conventions
 *   - Every GPU entry point only enqueues work on `stream` and returns. PKV_OK means the launch
 *     was accepted; argument errors are detected on the host before anything is launched and
 *     leave all buffers untouched.
 *   - The library allocates no device memory. Its only global state is one file-scope device
 *     array (PKV_STATIC_SCRATCH_BYTES per GPU, alive while the library is loaded) that
 *     pkv_paged_attention_decode_static uses instead of a workspace, plus per-device caches of
 *     launch facts (SM count, that array's address). Every other call takes its scratch space
 *     from a caller-provided workspace (size from pkv_decode_workspace_size).
 *   - Data errors that can only be seen on the device (a bad block id in a table, a bad slot)
 *     never trap: the offending work is skipped and, if `dev_error` is non-NULL, the first error
 *     code (PKV_DEVERR_*) is stored there with an atomic compare-and-swap (caller zeroes it).
 *   - A cudaStream_t may be passed wherever pkv_stream_t is expected (same type).
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

struct CUstream_st;
typedef struct CUstream_st* pkv_stream_t; /* identical to cudaStream_t; NULL = legacy stream */

typedef enum pkv_status {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, bad size, inconsistent shapes */
  PKV_ERR_UNSUPPORTED = 2,    /* well-formed but not built: dtype combination, head_dim, ... */
  PKV_ERR_OUT_OF_BLOCKS = 3,  /* host allocator: not enough free blocks */
  PKV_ERR_CUDA = 4,           /* a CUDA launch or query failed */
  PKV_ERR_DEVICE_TIMEOUT = 5  /* reserved: a bounded device-side wait gave up */
} pkv_status;

typedef enum pkv_dtype {
  PKV_FP16 = 0,      /* unquantized half precision */
  PKV_INT8_SYM = 1,  /* int8 codes in [-127, 127], x_hat = code * scale */
  PKV_INT4_ASYM = 2, /* uint4 codes in [0, 15], x_hat = (code - zp) * scale (V only) */
  PKV_FP8_E4M3 = 3   /* E4M3 bytes (sign, 4 exponent bits with bias 7, 3 mantissa bits, largest
                        finite 448), x_hat = value(code) * scale, scale = absmax / 448; K and V
                        both FP8 or neither ([yunthe] "vLLM推理引擎部署与KV Cache量化配置实战":
                        --kv-cache-dtype fp8 uses the E4M3 format) */
} pkv_dtype;

/* Device-side error codes written to *dev_error (first one wins). */
enum {
  PKV_DEVERR_NONE = 0,
  PKV_DEVERR_BLOCK_ID = 1,     /* block id in a table / mapping outside [0, num_blocks) */
  PKV_DEVERR_SLOT = 2,         /* slot_mapping entry beyond num_blocks * block_size */
  PKV_DEVERR_SLOT_GROUP = 3,   /* tokens bound for one block are not consecutive offsets */
  PKV_DEVERR_CONTEXT_LEN = 4,  /* context_len < 0, > max_context_len or > max_blocks*block_size */
  PKV_DEVERR_TIMEOUT = 5,      /* a bounded wait on an asynchronous copy gave up */
  PKV_DEVERR_SEQ_ORDER = 6,    /* a walk-order entry outside [0, num_seqs) */
  PKV_DEVERR_SHARED = 7        /* a shared-prefix group or shared block count out of range */
};

/* Describes one layer's cache pool. Pointers are device pointers, 16-byte aligned. */
typedef struct pkv_cache_desc {
  int32_t num_blocks;    /* nb: physical blocks in the pool */
  int32_t block_size;    /* bs: tokens per block, 16 or 32 */
  int32_t num_kv_heads;  /* Hkv */
  int32_t head_dim;      /* D: 64, 128 or 256 */
  int32_t k_dtype;       /* pkv_dtype: PKV_INT8_SYM, PKV_FP16 or PKV_FP8_E4M3 */
  int32_t v_dtype;       /* pkv_dtype: PKV_INT8_SYM, PKV_INT4_ASYM, PKV_FP16 or PKV_FP8_E4M3 */
  void* k_codes;
  void* v_codes;
  float* k_scale;        /* required when k_dtype != PKV_FP16 */
  float* v_scale;        /* required when v_dtype != PKV_FP16 */
  uint8_t* v_zp;         /* required when v_dtype == PKV_INT4_ASYM */
} pkv_cache_desc;

/* Human-readable name of a status code (static string, never NULL). */
PKV_API const char* pkv_status_string(pkv_status status);

/* Bytes of one (block, head) tile of K or V codes for this descriptor (0 on bad input). */
PKV_API size_t pkv_tile_bytes(const pkv_cache_desc* desc, int32_t which_v);

/*
 * pkv_store_quantized -- quantize T new tokens and scatter them into the pool.
 *
 * Follows [tbr8] §4 (store_kv: scale = absmax/127, codes = x/scale, scale stored per block) and
 * [yunthe] "KV Cache量化技术原理" (Q(x) for the asymmetric INT4 form), with the readings:
 * one scale (and zero point) per (block, KV head); round half to even; codes clamped to
 * [-127, 127] (INT8) or [0, 15] (INT4); INT4 range [min(0, min x), max(0, max x)],
 * scale = (hi - lo)/15, zp = clamp(rint(-lo/scale), 0, 15); scale 0 encodes an all-zero tile.
 * FP8 E4M3: scale = absmax/448, code = E4M3(x/scale) rounded to nearest even and saturated; new
 * values fit a stored scale when every |x/scale| <= 448.
 * All code arithmetic is IEEE binary32, round to nearest even, one rounding per operation.
 *
 * Tokens of one call that land in the same block must be adjacent in slot_mapping with
 * consecutive increasing offsets (a "group"); a block may appear in at most one group per call.
 * For a group at offsets o0..o1 of block b and each KV head:
 *   o0 == 0:  the tile's scale (and zp) is derived from the group alone; codes [o0, o1] written.
 *   o0 > 0:   if every new value is representable under the stored scale/zp ("fits"), new codes
 *             use it and offsets < o0 are untouched; otherwise the tile is rebuilt: old codes at
 *             offsets < o0 are dequantized in binary32, a new scale/zp is derived from them plus
 *             the new values, and offsets 0..o1 are requantized.
 * FP16 sides are copied as is.
 *
 *   k_new, v_new  device fp16 [T][num_kv_heads][head_dim]
 *   slot_mapping  device int64 [T]; negative = skip; >= num_blocks*block_size -> PKV_DEVERR_SLOT
 *   dev_error     device int32 or NULL
 * Returns PKV_OK, PKV_ERR_INVALID_ARG, PKV_ERR_UNSUPPORTED or PKV_ERR_CUDA. T == 0 is a no-op.
 */
PKV_API pkv_status pkv_store_quantized(const pkv_cache_desc* desc, const void* k_new, const void* v_new,
                               const int64_t* slot_mapping, int32_t T, int32_t* dev_error,
                               pkv_stream_t stream);

/*
 * pkv_decode_workspace_size -- bytes of scratch pkv_paged_attention_decode (and pkv_decode_step)
 * needs for these sizes: one ticket per (sequence, head group) and two barrier counters, plus one
 * partial (max, sum, fp32 accumulator) slot per (sequence, head group) and per worker warp; never
 * a dequantized copy of the cache.
 * The value depends on the current device (its SM count sets the number of worker warps).
 * Returns PKV_ERR_INVALID_ARG on bad sizes.
 */
PKV_API pkv_status pkv_decode_workspace_size(const pkv_cache_desc* desc, int32_t num_seqs,
                                             int32_t num_q_heads, int32_t max_context_len,
                                             int32_t partition_tokens, size_t* bytes);

/*
 * pkv_decode_partitioning -- how the decode call splits the work for these sizes: the number of
 * worker warps (each takes an equal share of all KV blocks) and of persistent CTAs on the
 * current device. Either output pointer may be NULL.
 */
PKV_API pkv_status pkv_decode_partitioning(const pkv_cache_desc* desc, int32_t num_seqs,
                                           int32_t num_q_heads, int32_t max_context_len,
                                           int32_t partition_tokens, int32_t* num_workers_out,
                                           int32_t* num_ctas_out);

/*
 * pkv_paged_attention_decode -- one decode step of attention over the paged, quantized cache.
 *
 * For every sequence s and query head h (KV head g = h / (num_q_heads / num_kv_heads)):
 *   token t < L_s lives at physical block b = block_tables[s][t / bs], offset t % bs
 *   ([yunthe] "PagedAttention分页注意力机制" block_table; [tbr8] §2);
 *   k_hat = code * k_scale[b][g]; v_hat = (code - zp) * v_scale[b][g] ([yunthe] x_hat formula);
 *   z_t = softmax_scale * dot(q[s][h], k_hat_t); out[s][h] = sum_t softmax(z)_t * v_hat_t,
 *   written as fp16 (round to nearest). L_s == 0 gives out = 0.
 * Work split: all KV blocks of the batch form one stream, ordered (sequence, head group, block),
 * cut into equal contiguous shares for a persistent set of worker warps, so any length mix is
 * balanced. A (sequence, head group) cut between warps gets one partial per warp in the
 * workspace and the last of them to finish merges them, all in one kernel launch.
 * partition_tokens 0 uses every resident warp of the device; a positive multiple of block_size
 * asks for about one worker per partition_tokens tokens of the largest possible work
 * (num_seqs * heads * max_context_len), i.e. fewer workers and fewer cuts.
 *
 *   q            device fp16 [num_seqs][num_q_heads][head_dim]
 *   out          device fp16 [num_seqs][num_q_heads][head_dim]
 *   block_tables device int32 [num_seqs][max_blocks_per_seq]
 *   context_lens device int32 [num_seqs]; each <= max_context_len (host bound used to size the
 *                grid) and <= max_blocks_per_seq * block_size, else PKV_DEVERR_CONTEXT_LEN and the
 *                sequence is clamped
 *   workspace    device, >= pkv_decode_workspace_size(...) bytes, 16-byte aligned. It must be
 *                zero-filled before its first use: every call that completes leaves its tickets
 *                at zero again, so one zeroing serves any number of later calls (zero it again
 *                after a PKV_DEVERR_TIMEOUT). Calls that share a workspace must not overlap on
 *                the GPU.
 *   dev_error    device int32 or NULL
 * num_q_heads must be a multiple of num_kv_heads. The pool may hold at most 2^31 - 1 token rows
 * per cache side (num_blocks * num_kv_heads * block_size): the tile copies address rows with a
 * signed 32-bit coordinate. A larger pool gives PKV_ERR_UNSUPPORTED.
 *
 * Ordering with the preceding work on `stream`: the kernel is launched with programmatic stream
 * serialization, so it may start while the previous kernel on the stream is still running (the
 * store of the step's new tokens, which lets the decode's set-up overlap it). Before it waits
 * for that kernel to complete it reads only context_lens, block_tables and q (and prefetches q);
 * every read of the pool (codes, scales, zero points) and every write comes after the wait.
 * So context_lens, block_tables and q must be complete before the previous kernel on the stream
 * starts: written by an earlier kernel or copy, not by the kernel immediately before this call
 * when that kernel lets its dependents start early (griddepcontrol.launch_dependents). A
 * stream-ordered copy, memset or event wait in between is enough.
 */
PKV_API pkv_status pkv_paged_attention_decode(const pkv_cache_desc* desc, void* out, const void* q,
                                      int32_t num_seqs, int32_t num_q_heads,
                                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                                      const int32_t* context_lens, int32_t max_context_len,
                                      float softmax_scale, int32_t partition_tokens,
                                      void* workspace, size_t workspace_bytes, int32_t* dev_error,
                                      pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_ex -- pkv_paged_attention_decode with options; the same arguments,
 * results and ordering rules, plus:
 *
 * Walk order. seq_order: device int32 [num_seqs] or NULL: the order in which the decode walks the
 *   sequences (a permutation of 0 .. num_seqs-1; results do not depend on it). A caller that knows
 *   which sequences share physical blocks (beam candidates forked from one parent, [deepinsea]
 *   "Copy-on-Write 机制"; requests on a common prefix, [yunthe] "PagedAttention分页注意力机制与vLLM
 *   实现") lists them next to each other, so that the shared blocks are read from memory once and
 *   found in L2 by the neighbours. An entry outside [0, num_seqs) leaves that position empty and
 *   sets PKV_DEVERR_SEQ_ORDER; a repeated entry makes that sequence's outputs unspecified.
 *
 * Shared-prefix decode (num_prefix_groups > 0). Sequences that share their first blocks (one
 *   physical copy, [yunthe] "PagedAttention分页注意力机制与vLLM实现" and "Prefix Caching与多轮对话场景
 *   优化实践") are given as groups: group i's members are prefix_members[prefix_group_start[i] ..
 *   prefix_group_start[i+1]), and shared_blocks[s] is the number of leading blocks sequence s shares
 *   with its group (0 for a sequence in no group). A first pass reads each shared block once per
 *   group and multiplies it against the queries of every member (integer tensor cores on the int8
 *   codes, the prefill kernel's prefix mode), leaving partial softmax states in the workspace; the
 *   decode then walks only each sequence's own blocks and merges the two. Requirements (not
 *   checked on the device; breaking them gives unspecified outputs, never a fault): the members of
 *   a group have the same shared_blocks value and the same table entries for those blocks; every
 *   sequence with shared_blocks > 0 is a member of exactly one group. A shared count that leaves
 *   no block of the sequence to the decode is clamped to leave its last block, and reported with
 *   PKV_DEVERR_SHARED. Built for INT8 K with INT8 or INT4 V and head_dim 128 (else
 *   PKV_ERR_UNSUPPORTED). The workspace must then be pkv_decode_ex_workspace_size(...) bytes.
 *   max_group_size and max_shared_blocks are host bounds (they size the first pass's grid); groups
 *   or counts above them are reported (PKV_DEVERR_SHARED) and their shared part left out.
 *   prefix_group_start, prefix_members and shared_blocks are read like block_tables (before the
 *   decode waits for the preceding kernel).
 *
 * options may be NULL (the plain decode). struct_bytes must be sizeof(pkv_decode_options) as the
 * caller compiled it.
 */
typedef struct pkv_decode_options {
  size_t struct_bytes;
  const int32_t* seq_order;
  int32_t num_prefix_groups;
  int32_t num_prefix_members;          /* prefix_group_start[num_prefix_groups] */
  int32_t max_group_size;
  int32_t max_shared_blocks;
  const int32_t* prefix_group_start;   /* device int32 [num_prefix_groups + 1] */
  const int32_t* prefix_members;       /* device int32 [num_prefix_members] */
  const int32_t* shared_blocks;        /* device int32 [num_seqs] */
} pkv_decode_options;
PKV_API pkv_status pkv_paged_attention_decode_ex(const pkv_cache_desc* desc, void* out, const void* q,
                                                 int32_t num_seqs, int32_t num_q_heads,
                                                 const int32_t* block_tables, int32_t max_blocks_per_seq,
                                                 const int32_t* context_lens, int32_t max_context_len,
                                                 float softmax_scale, int32_t partition_tokens,
                                                 const pkv_decode_options* options, void* workspace,
                                                 size_t workspace_bytes, int32_t* dev_error, pkv_stream_t stream);
/* Workspace bytes of pkv_paged_attention_decode_ex with these options (options may be NULL). */
PKV_API pkv_status pkv_decode_ex_workspace_size(const pkv_cache_desc* desc, int32_t num_seqs, int32_t num_q_heads,
                                                int32_t max_context_len, int32_t partition_tokens,
                                                const pkv_decode_options* options, size_t* bytes);

/*
 * pkv_paged_attention_prefill -- chunked prefill: causal attention of each sequence's new tokens
 * over the paged, quantized cache, after pkv_store_quantized has stored their K/V
 * ([yunthe] section "Prefix Caching与多轮对话场景优化实践": with the prefix cached, only the new
 * tokens are computed; [tbr8] §5 item 2: dequantization inside the attention operator).
 *
 * Sequence s has q_len = cu_q_lens[s+1] - cu_q_lens[s] query rows q[cu_q_lens[s] + i], the last
 * q_len of its context_lens[s] tokens; the query at position p = context_lens[s] - q_len + i
 * attends to tokens 0 .. p (k_hat, v_hat and the logit scale as in pkv_paged_attention_decode):
 *   out[row][h] = sum_{t <= p} softmax_t(softmax_scale * q[row][h] . k_hat_t) * v_hat_t   (fp16)
 *   q, out        device fp16 [total_q][num_q_heads][head_dim]
 *   cu_q_lens     device int32 [num_seqs + 1], non-decreasing, cu_q_lens[0] = 0,
 *                 cu_q_lens[num_seqs] = total_q; every q_len <= max_q_len (host bound: grid size)
 *   context_lens  device int32 [num_seqs]; q_len <= context_len <= min(max_context_len,
 *                 max_blocks_per_seq * block_size), else PKV_DEVERR_CONTEXT_LEN (rows of a chunk
 *                 longer than its context are zeroed; a longer context is clamped)
 * Built for INT8 K with INT8 or INT4 V, head_dim 128, block size 16 or 32 (else
 * PKV_ERR_UNSUPPORTED). q.k runs on the integer tensor cores with q split into exact byte planes;
 * p.v on the fp16 tensor cores, each V code converted once per 128 query columns. No workspace.
 */
PKV_API pkv_status pkv_paged_attention_prefill(const pkv_cache_desc* desc, void* out, const void* q,
                                               int32_t num_seqs, int32_t num_q_heads, const int32_t* cu_q_lens,
                                               int32_t total_q, int32_t max_q_len, const int32_t* block_tables,
                                               int32_t max_blocks_per_seq, const int32_t* context_lens,
                                               int32_t max_context_len, float softmax_scale, int32_t* dev_error,
                                               pkv_stream_t stream);

/*
 * pkv_decode_step -- one decode step in a single kernel launch: exactly
 *   pkv_copy_blocks(desc, block_mapping, n_pairs, ...); then
 *   pkv_store_quantized(desc, k_new, v_new, slot_mapping, T, ...); then
 *   pkv_paged_attention_decode(desc, out, q, num_seqs, ...)
 * on `stream`, with the same arguments, layouts, results and error behaviour as those three
 * calls (each part may be empty: n_pairs == 0, T == 0). The pages describe the three operations;
 * running them as one launch is this library's own arrangement for latency: every warp of the
 * decode grid first takes part in the copies and the stores, a grid-wide barrier separates the
 * phases, and the decode's set-up (lengths, block tables) overlaps the stores. The kernel is
 * launched cooperatively (all CTAs resident); PKV_ERR_CUDA if the device refuses that.
 * The workspace is the decode's (pkv_decode_workspace_size), zero-filled before first use as
 * there; its barrier counters, like the tickets, are left at zero by every call that completes.
 */
PKV_API pkv_status pkv_decode_step(const pkv_cache_desc* desc, const int32_t* block_mapping, int32_t n_pairs,
                                   const void* k_new, const void* v_new, const int64_t* slot_mapping, int32_t T,
                                   void* out, const void* q, int32_t num_seqs, int32_t num_q_heads,
                                   const int32_t* block_tables, int32_t max_blocks_per_seq,
                                   const int32_t* context_lens, int32_t max_context_len, float softmax_scale,
                                   int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                                   int32_t* dev_error, pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_static -- the same decode as pkv_paged_attention_decode, for
 * callers that cannot hand the library any scratch memory: for example a plugin that its host
 * engine gives only the input and output buffers (the engine owns every other byte of device
 * memory), or a serving loop that fixed its memory budget up front and may not allocate per
 * request. The web pages this library follows have no counterpart of this call; it exists only
 * for such callers.
 *
 * It allocates nothing: its scratch is one file-scope device array of PKV_STATIC_SCRATCH_BYTES
 * (8 MiB) that every GPU holds from the moment the library is loaded until the process exits.
 *   - Sizes whose scratch would exceed it (pkv_decode_workspace_size(...) >
 *     PKV_STATIC_SCRATCH_BYTES) are rejected with PKV_ERR_UNSUPPORTED before anything runs; use
 *     pkv_paged_attention_decode with a workspace for those.
 *   - The first call on a device looks up that device's address of the array (with the device
 *     current), so make that first call before any stream capture begins.
 *   - All calls share the array and it keeps the last call's contents; each call clears, on its
 *     stream, the part that must start at zero. Calls whose executions overlap on the GPU (any
 *     streams, any threads) race on the array and give undefined results: serialise them.
 *   - Every argument is checked before anything is enqueued: a call that returns an error has
 *     written nothing, not even the array.
 * Arguments and results are those of pkv_paged_attention_decode without the workspace.
 */
#define PKV_STATIC_SCRATCH_BYTES (8u << 20)
PKV_API pkv_status pkv_paged_attention_decode_static(
    const pkv_cache_desc* desc, void* out, const void* q, int32_t num_seqs, int32_t num_q_heads,
    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
    int32_t max_context_len, float softmax_scale, int32_t partition_tokens, int32_t* dev_error,
    pkv_stream_t stream);

/*
 * pkv_static_scratch_address -- the current device's address of the array that
 * pkv_paged_attention_decode_static uses, and its size in bytes (either output may be NULL
 * except device_ptr). For diagnostics and tests, e.g. to check that the call clears what must
 * start at zero whatever an earlier call or a stray write left there. Like that call, the first
 * use on a device looks the address up with the device current. The pages have no counterpart.
 */
PKV_API pkv_status pkv_static_scratch_address(void** device_ptr, size_t* bytes);

/*
 * pkv_copy_blocks -- copy-on-write block copies ([deepinsea] section "Copy-on-Write 机制";
 * [yunthe] "PagedAttention分页注意力机制", fork writes new tokens into new blocks).
 * For each pair (src, dst) in block_mapping, copies every head's K codes, V codes, scales and
 * zero points of block src into block dst. Pairs must not chain (no dst is another pair's src)
 * and no dst may repeat. An id outside [0, num_blocks) skips the pair and sets
 * PKV_DEVERR_BLOCK_ID.
 *   block_mapping device int32 [n_pairs][2] = {src, dst}
 */
PKV_API pkv_status pkv_copy_blocks(const pkv_cache_desc* desc, const int32_t* block_mapping,
                           int32_t n_pairs, int32_t* dev_error, pkv_stream_t stream);

/*
 * pkv_swap_blocks -- move whole blocks between the device pool and a pool in host memory
 * ([deepinsea] section "Swap 机制": when device memory runs short, KV blocks are swapped out to
 * CPU memory and back in later; the transfer is slow, so it is a fallback, not a routine step).
 *
 * For each pair (src, dst) of block_mapping, every head's K codes, V codes, scales and zero points
 * of block src of the source pool are copied into block dst of the destination pool:
 *   direction PKV_SWAP_OUT: device_pool -> host_pool (src is a device block id, dst a host id)
 *   direction PKV_SWAP_IN:  host_pool -> device_pool (src is a host block id, dst a device id)
 * The two pools must have the same block_size, num_kv_heads, head_dim and dtypes; num_blocks may
 * differ. The host pool's arrays must be page-locked host memory that the device can address
 * (cudaHostAlloc / cudaMallocHost, or cudaHostRegister with cudaHostRegisterMapped), every byte of
 * each array; the device pool's arrays must be memory of the current device. Both are checked on
 * the host (both ends of every array) before anything is launched: PKV_ERR_INVALID_ARG otherwise,
 * never a fault. One kernel moves all pairs, however scattered the ids (reads and writes of host
 * memory cross the host link directly, many 16-byte accesses in flight). Ids outside their pool
 * skip the pair and set PKV_DEVERR_BLOCK_ID. Destinations must not repeat.
 *   block_mapping int32 [n_pairs][2] = {src, dst}, in device memory or mapped page-locked host memory
 *   dev_error     device int32 (or mapped host int32) or NULL
 * Host-side bookkeeping stays with the caller: a pkv_allocator per pool (release the device ids
 * after a swap-out completes, the host ids after a swap-in).
 */
typedef enum pkv_swap_dir { PKV_SWAP_OUT = 0, PKV_SWAP_IN = 1 } pkv_swap_dir;
PKV_API pkv_status pkv_swap_blocks(const pkv_cache_desc* device_pool, const pkv_cache_desc* host_pool,
                                   const int32_t* block_mapping, int32_t n_pairs, int32_t direction,
                                   int32_t* dev_error, pkv_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Host block allocator: free list plus per-block reference counts, host memory only.
 * Ceil-division sizing and the out-of-blocks failure follow [deepinsea] "分页机制设计"
 * (BlockManager.allocate returns False when short); release-on-refcount follows [tbr8] §5
 * item 3; fork/copy-on-write follows [deepinsea] "Copy-on-Write 机制". The free list is LIFO.
 * A handle is not thread-safe.
 * ------------------------------------------------------------------------------------------ */
typedef struct pkv_allocator pkv_allocator;

/* Number of blocks needed for num_tokens tokens: ceil(num_tokens / block_size); -1 if invalid. */
PKV_API int32_t pkv_blocks_for_tokens(int64_t num_tokens, int32_t block_size);

PKV_API pkv_status pkv_alloc_create(int32_t num_blocks, pkv_allocator** out_handle);
PKV_API void pkv_alloc_destroy(pkv_allocator* h);
PKV_API int32_t pkv_alloc_num_free(const pkv_allocator* h);
/* Reference count of a block (0 = free); -1 for an id out of range. */
PKV_API int32_t pkv_alloc_refcount(const pkv_allocator* h, int32_t block_id);
/* Take n blocks (refcount 1 each) into ids[0..n). All-or-nothing: PKV_ERR_OUT_OF_BLOCKS if
 * fewer than n are free, in which case nothing is taken. */
PKV_API pkv_status pkv_alloc_blocks(pkv_allocator* h, int32_t n, int32_t* ids);
/* Share n blocks with another sequence: refcount += 1 each. Ids must be allocated. */
PKV_API pkv_status pkv_alloc_fork(pkv_allocator* h, const int32_t* ids, int32_t n);
/* Drop one reference from each of n blocks; a block returns to the free list at 0. All or nothing:
 * PKV_ERR_INVALID_ARG (and no change) if an id is out of range or listed more often than it has
 * references. Cost O(n log n) in the ids, independent of the pool size. */
PKV_API pkv_status pkv_alloc_release(pkv_allocator* h, const int32_t* ids, int32_t n);
/* Make block_id private before a write. If its refcount is 1, *new_id = block_id and nothing
 * changes. Otherwise a fresh block is taken (*new_id), the old block's refcount drops by one,
 * and the caller must copy old -> new (pkv_copy_blocks) before writing. */
PKV_API pkv_status pkv_alloc_cow(pkv_allocator* h, int32_t block_id, int32_t* new_id);

/* ------------------------------------------------------------------------------------------
 * Automatic prefix caching (host memory only): an index from token blocks to physical blocks
 * ([yunthe] section "Prefix Caching与多轮对话场景优化实践": a new request first looks for blocks in
 * the pool that already hold its prefix and, on a hit, maps onto them and computes only its new
 * tokens; section "PagedAttention分页注意力机制与vLLM实现": requests with the same prefix share
 * physical blocks). Only whole blocks are cached. A block is identified by its block_size token
 * ids together with all the tokens before it: lookups hash that and then compare it exactly, so a
 * hash collision never gives a false hit. The cache holds one reference on every block it
 * indexes, through the pool's pkv_allocator (which must outlive it); a block that only the cache
 * references is kept for later hits and evicted least recently used first when pkv_prefix_alloc
 * needs room; evicting a block drops the cached blocks that follow it too. Not thread-safe.
 * ------------------------------------------------------------------------------------------ */
typedef struct pkv_prefix_cache pkv_prefix_cache;

PKV_API pkv_status pkv_prefix_cache_create(pkv_allocator* alloc, int32_t block_size, pkv_prefix_cache** out);
/* Drops every entry (releasing the cache's references) and frees the handle. */
PKV_API void pkv_prefix_cache_destroy(pkv_prefix_cache* pc);
/* Cached blocks; cached blocks that only the cache references (evictable). -1 on NULL. */
PKV_API int32_t pkv_prefix_cache_size(const pkv_prefix_cache* pc);
PKV_API int32_t pkv_prefix_cache_evictable(const pkv_prefix_cache* pc);
/* The longest cached prefix of tokens[0, n_tokens) in whole blocks, at most max_blocks: the
 * physical ids go to block_ids[0, *n_matched), and each of them gains one reference that the
 * caller owns (release it with pkv_alloc_release when the sequence ends). */
PKV_API pkv_status pkv_prefix_match(pkv_prefix_cache* pc, const int32_t* tokens, int64_t n_tokens,
                                    int32_t* block_ids, int32_t max_blocks, int32_t* n_matched);
/* Registers the whole blocks of a sequence once their K/V are stored: block_ids[i] holds tokens
 * [i*block_size, (i+1)*block_size). Blocks whose content (with their prefix) is already cached
 * are left as they are; the cache takes one reference on each newly registered block. The ids
 * must be allocated (PKV_ERR_INVALID_ARG, and no change, otherwise). */
PKV_API pkv_status pkv_prefix_insert(pkv_prefix_cache* pc, const int32_t* tokens, int64_t n_tokens,
                                     const int32_t* block_ids, int32_t n_blocks);
/* Takes n fresh blocks (refcount 1) from the allocator, evicting least recently used blocks that
 * only the cache references when too few are free. All or nothing: PKV_ERR_OUT_OF_BLOCKS, with
 * no eviction, when even evicting every such block would not free enough. */
PKV_API pkv_status pkv_prefix_alloc(pkv_prefix_cache* pc, int32_t n, int32_t* ids);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
