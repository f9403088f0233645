/*
 * oracle.h -- declarations of the CPU oracle (test infrastructure only; see oracle.c).
 * Independent of the GPU library: its own types, its own constants, host memory only.
 */
#ifndef PKV_ORACLE_H
#define PKV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_FP16 = 0, ORACLE_INT8_SYM = 1, ORACLE_INT4_ASYM = 2, ORACLE_FP8_E4M3 = 3 };

/* error codes reported by the oracle for malformed inputs (first one wins) */
enum {
  ORACLE_DEVERR_BLOCK_ID = 1,
  ORACLE_DEVERR_SLOT = 2,
  ORACLE_DEVERR_SLOT_GROUP = 3,
  ORACLE_DEVERR_CONTEXT_LEN = 4
};

/* One layer's pool in host memory, same row-major layout as the device pool:
 *   codes [num_blocks][num_kv_heads][block_size][row] with row = head_dim int8 (INT8),
 *         head_dim fp16 bit patterns (FP16), head_dim/2 packed nibbles (INT4) or head_dim
 *         E4M3 bytes (FP8);
 *   scales / zero points [num_blocks][num_kv_heads]. */
typedef struct oracle_cache {
  int32_t num_blocks, block_size, num_kv_heads, head_dim;
  int32_t k_dtype, v_dtype;
  void* k_codes;
  void* v_codes;
  float* k_scale;
  float* v_scale;
  uint8_t* v_zp;
} oracle_cache;

/* Quantize and scatter T tokens (fp16 bit patterns [T][H][D]). Returns 0, an error code
 * (first malformed input seen), or -1 for an unsupported descriptor. */
int32_t oracle_store(const oracle_cache* c, const uint16_t* k_new, const uint16_t* v_new,
                     const int64_t* slot_mapping, int32_t T);

/* Copy whole blocks: pairs {src, dst}. */
int32_t oracle_copy_blocks(const oracle_cache* c, const int32_t* block_mapping, int32_t n_pairs);

/* The E4M3 value of a code (binary64, exact; NaN for the NaN codes), and the code of a binary32
 * value (round to nearest, ties to even, saturating at +-448), from the format's definition. */
double oracle_fp8_e4m3_decode(uint8_t code);
uint8_t oracle_fp8_e4m3_encode(float x);

/* Decode attention in binary64. q: fp16 bit patterns [S][Hq][D]; out: double [S][Hq][D]. */
int32_t oracle_decode(const oracle_cache* c, const uint16_t* q, int32_t num_seqs, int32_t num_q_heads,
                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                      const int32_t* context_lens, int32_t max_context_len, float softmax_scale,
                      double* out, int32_t num_threads);

/* Chunked prefill: causal attention of each sequence's last q_len context tokens (queries
 * q [T][Hq][D], T = cu_q_lens[num_seqs], rows of sequence s at cu_q_lens[s] ..) over its cached
 * tokens; out: double [T][Hq][D]. */
int32_t oracle_prefill(const oracle_cache* c, const uint16_t* q, int32_t num_seqs, int32_t num_q_heads,
                       const int32_t* cu_q_lens, const int32_t* block_tables, int32_t max_blocks_per_seq,
                       const int32_t* context_lens, float softmax_scale, double* out, int32_t num_threads);

#ifdef __cplusplus
}
#endif

#endif
