/*
 * oracle.c -- plain, slow, obviously correct CPU implementation of the paged block-quantized
 * KV-cache path: quantize + scatter (store), block copy (copy-on-write), and decode attention.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the oracle the GPU library is checked against; it
 * shares no code, header, table or helper with the GPU library and is never called by it.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 *
 * Sources (web pages, cited by page and section):
 *   [tbr8]      tbr8.org, "如何通过 PagedAttention 与分块量化结合：解决移动端内存碎片化导致的长文本 OOM"
 *   [deepinsea] deepinsea.top, "PagedAttention 内存管理深度解析"
 *   [yunthe]    yunthe.com, "LLM推理显存优化KV Cache量化与PagedAttention实现详解"
 *
 * Arithmetic
 *   - Quantization (codes, scales, zero points): IEEE-754 binary32, round to nearest even, one
 *     rounding per operation. Build with -ffp-contract=off and without fast-math so that the
 *     compiler neither fuses a*b+c nor reorders anything. rintf() rounds half to even in the
 *     default rounding mode.
 *   - Attention: binary64 throughout (dequantized values, dot products, exp, sums).
 *
 * Readings where the pages leave a step open (each repeated where it is used):
 *   R1 rounding is round-half-to-even ([yunthe] writes round(); [tbr8] §4's cast truncates)
 *   R2 one scale (and zero point) per (block, KV head) ([tbr8] §4 stores one scale per block
 *      index of a [blocks, heads, 1, 1] tensor)
 *   R3 scales are stored and computed in binary32
 *   R4 INT8 symmetric codes lie in [-127, 127] with zero point 0
 *   R5 INT4 range is [min(0, min x), max(0, max x)], scale (hi-lo)/15, zp = clamp(rint(-lo/s),0,15)
 *   R6 appending to a partly filled block: keep the stored scale if every new value fits,
 *      else dequantize the old codes and requantize the whole tile   -- parity unpinned by the
 *      pages (they only ever quantize whole blocks); pinned here only by internal invariants
 *   R7 scale 0 means an all-zero tile: codes 0 (INT8) / zp 0, codes 0 (INT4)
 *   R8 INT4 nibbles packed along head_dim, low nibble = even dimension
 *   R10 context_lens include the token just stored
 *   R11 context_len 0 gives a zero output; a negative slot skips the token
 *   R15 FP8 E4M3 ([yunthe] "vLLM推理引擎部署与KV Cache量化配置实战": the fp8 cache mode uses E4M3):
 *      one binary32 scale per (block, KV head), scale = absmax / 448 (the largest finite E4M3
 *      magnitude), code = E4M3(x / scale) rounded to nearest, ties to even, saturating; scale 0
 *      gives codes 0; x_hat = value(code) * scale. Appending: new values fit when every
 *      |x / scale_old| <= 448, else the tile is rebuilt as for INT8 (old values dequantized in
 *      binary32, scale from old and new together)
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---- IEEE-754 binary16 -> binary64, from the format's definition (exact) ---- */
static double half_bits_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int exponent = (h >> 10) & 0x1f;
  int mantissa = h & 0x3ff;
  double v;
  if (exponent == 0) {
    v = ldexp((double)mantissa, -24); /* subnormal: m * 2^-24 */
  } else if (exponent == 31) {
    v = mantissa ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + mantissa), exponent - 25); /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

static void record_error(int32_t* err, int32_t code) {
  if (*err == 0) *err = code;
}

/* ---- symmetric INT8: scale = absmax / 127 ([tbr8] §4 store_kv), codes round(x / scale) ---- */
static int8_t quant_sym(float x, float s) {
  if (s == 0.0f) return 0; /* R7 */
  float r = rintf(x / s);   /* R1 */
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f; /* R4 */
  return (int8_t)r;
}

/* One (block, head) tile, symmetric INT8. tile: [bs][d] codes; new_x: [n][d] values for
 * offsets o0 .. o0+n-1. */
static void store_tile_sym(int8_t* tile, float* scale, int d, int o0, int n, const float* new_x) {
  float m_new = 0.0f;
  for (int i = 0; i < n * d; ++i) {
    float a = fabsf(new_x[i]);
    if (a > m_new) m_new = a;
  }
  if (o0 == 0) {
    float s = m_new / 127.0f;
    for (int i = 0; i < n * d; ++i) tile[i] = quant_sym(new_x[i], s);
    *scale = s;
    return;
  }
  /* R6: append into a partly filled tile */
  float s_old = *scale;
  int fits = 1;
  for (int i = 0; i < n * d && fits; ++i) {
    if (s_old == 0.0f) {
      fits = (new_x[i] == 0.0f);
    } else {
      float r = rintf(new_x[i] / s_old);
      fits = (r <= 127.0f && r >= -127.0f);
    }
  }
  int8_t* new_tile = tile + (size_t)o0 * d;
  if (fits) {
    for (int i = 0; i < n * d; ++i) new_tile[i] = quant_sym(new_x[i], s_old);
    return;
  }
  /* rebuild: old codes dequantized in binary32, scale from old and new values together */
  int n_old = o0 * d;
  float* xh = (float*)malloc(sizeof(float) * (size_t)(n_old > 0 ? n_old : 1));
  float m_old = 0.0f;
  for (int i = 0; i < n_old; ++i) {
    xh[i] = (float)tile[i] * s_old; /* x_hat = Q * scale, [yunthe] with zp 0 */
    float a = fabsf(xh[i]);
    if (a > m_old) m_old = a;
  }
  float s = (m_old > m_new ? m_old : m_new) / 127.0f;
  for (int i = 0; i < n_old; ++i) tile[i] = quant_sym(xh[i], s);
  for (int i = 0; i < n * d; ++i) new_tile[i] = quant_sym(new_x[i], s);
  *scale = s;
  free(xh);
}

/* ---- asymmetric INT4: Q(x) = clamp(round(x/scale + zp), 0, 15), [yunthe] quantize formula ---- */
static void derive_asym(float lo, float hi, float* s_out, int* zp_out) {
  float s = (hi - lo) / 15.0f; /* R5 */
  int zp = 0;
  if (s != 0.0f) {
    float z = rintf(-lo / s);
    if (z < 0.0f) z = 0.0f;
    if (z > 15.0f) z = 15.0f;
    zp = (int)z;
  }
  *s_out = s;
  *zp_out = zp;
}

static int quant_asym(float x, float s, int zp) {
  if (s == 0.0f) return zp; /* R7 */
  float r = rintf(x / s + (float)zp);
  if (r < 0.0f) r = 0.0f;
  if (r > 15.0f) r = 15.0f;
  return (int)r;
}

/* nibble access, R8: byte j of a row = code[2j] | code[2j+1] << 4 */
static int get_nibble(const uint8_t* row, int dim) {
  uint8_t byte = row[dim / 2];
  return (dim % 2 == 0) ? (byte & 0xF) : (byte >> 4);
}

static void set_nibble(uint8_t* row, int dim, int code) {
  uint8_t* byte = &row[dim / 2];
  if (dim % 2 == 0) {
    *byte = (uint8_t)((*byte & 0xF0) | (code & 0xF));
  } else {
    *byte = (uint8_t)((*byte & 0x0F) | ((code & 0xF) << 4));
  }
}

/* tile: [bs][d/2] packed bytes */
static void store_tile_asym4(uint8_t* tile, float* scale, uint8_t* zp_ptr, int d, int o0, int n,
                             const float* new_x) {
  int row_bytes = d / 2;
  float lo_new = 0.0f, hi_new = 0.0f; /* range always includes 0 (R5) */
  for (int i = 0; i < n * d; ++i) {
    if (new_x[i] < lo_new) lo_new = new_x[i];
    if (new_x[i] > hi_new) hi_new = new_x[i];
  }
  if (o0 == 0) {
    float s;
    int zp;
    derive_asym(lo_new, hi_new, &s, &zp);
    for (int t = 0; t < n; ++t)
      for (int j = 0; j < d; ++j)
        set_nibble(tile + (size_t)t * row_bytes, j, quant_asym(new_x[t * d + j], s, zp));
    *scale = s;
    *zp_ptr = (uint8_t)zp;
    return;
  }
  float s_old = *scale;
  int zp_old = *zp_ptr;
  int fits = 1;
  for (int i = 0; i < n * d && fits; ++i) {
    if (s_old == 0.0f) {
      fits = (new_x[i] == 0.0f);
    } else {
      float r = rintf(new_x[i] / s_old + (float)zp_old);
      fits = (r >= 0.0f && r <= 15.0f);
    }
  }
  if (fits) {
    for (int t = 0; t < n; ++t)
      for (int j = 0; j < d; ++j)
        set_nibble(tile + (size_t)(o0 + t) * row_bytes, j, quant_asym(new_x[t * d + j], s_old, zp_old));
    return;
  }
  int n_old = o0 * d;
  float* xh = (float*)malloc(sizeof(float) * (size_t)(n_old > 0 ? n_old : 1));
  float lo = lo_new, hi = hi_new;
  for (int t = 0; t < o0; ++t) {
    for (int j = 0; j < d; ++j) {
      int q = get_nibble(tile + (size_t)t * row_bytes, j);
      float v = (float)(q - zp_old) * s_old; /* x_hat = (Q - zp) * scale, [yunthe] */
      xh[t * d + j] = v;
      if (v < lo) lo = v;
      if (v > hi) hi = v;
    }
  }
  float s;
  int zp;
  derive_asym(lo, hi, &s, &zp);
  for (int t = 0; t < o0; ++t)
    for (int j = 0; j < d; ++j)
      set_nibble(tile + (size_t)t * row_bytes, j, quant_asym(xh[t * d + j], s, zp));
  for (int t = 0; t < n; ++t)
    for (int j = 0; j < d; ++j)
      set_nibble(tile + (size_t)(o0 + t) * row_bytes, j, quant_asym(new_x[t * d + j], s, zp));
  *scale = s;
  *zp_ptr = (uint8_t)zp;
  free(xh);
}

/* ---- FP8 E4M3 (R15). The format: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; the
 * exponent field 0 holds subnormals m * 2^-9, fields 1..15 hold (1 + m/8) * 2^(e-7), except that
 * the all-ones pattern S.1111.111 is NaN; there are no infinities, so the largest finite
 * magnitude is 1.75 * 2^8 = 448. ---- */
double oracle_fp8_e4m3_decode(uint8_t code) {
  int sign = code >> 7, e = (code >> 3) & 0xF, m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);
  else v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  return sign ? -v : v;
}

/* Nearest representable magnitude by comparing with every finite one (codes 0..126 ascend in
 * value); of two equally near, the one with an even mantissa (its lowest bit 0). Magnitudes past
 * 448 go to 448 (saturation). The sign is the sign bit of x. */
uint8_t oracle_fp8_e4m3_encode(float x) {
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);
  int best = 0;
  double best_d = a;
  for (int c = 1; c <= 126; ++c) {
    double d = fabs(oracle_fp8_e4m3_decode((uint8_t)c) - a);
    if (d < best_d || (d == best_d && (c & 1) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return (uint8_t)(sign | best);
}

static uint8_t quant_fp8(float x, float s) {
  if (s == 0.0f) return 0; /* R7 */
  return oracle_fp8_e4m3_encode(x / s);
}

/* One (block, head) tile of E4M3 codes: [bs][d] bytes; new_x: [n][d] values for offsets o0.. */
static void store_tile_fp8(uint8_t* tile, float* scale, int d, int o0, int n, const float* new_x) {
  float m_new = 0.0f;
  for (int i = 0; i < n * d; ++i) {
    float a = fabsf(new_x[i]);
    if (a > m_new) m_new = a;
  }
  if (o0 == 0) {
    float s = m_new / 448.0f;
    for (int i = 0; i < n * d; ++i) tile[i] = quant_fp8(new_x[i], s);
    *scale = s;
    return;
  }
  float s_old = *scale;
  int fits = 1;
  for (int i = 0; i < n * d && fits; ++i) {
    if (s_old == 0.0f) fits = (new_x[i] == 0.0f);
    else fits = (fabsf(new_x[i] / s_old) <= 448.0f);
  }
  uint8_t* new_tile = tile + (size_t)o0 * d;
  if (fits) {
    for (int i = 0; i < n * d; ++i) new_tile[i] = quant_fp8(new_x[i], s_old);
    return;
  }
  int n_old = o0 * d;
  float* xh = (float*)malloc(sizeof(float) * (size_t)(n_old > 0 ? n_old : 1));
  float m_old = 0.0f;
  for (int i = 0; i < n_old; ++i) {
    xh[i] = (float)oracle_fp8_e4m3_decode(tile[i]) * s_old; /* exact value, one binary32 product */
    float a = fabsf(xh[i]);
    if (a > m_old) m_old = a;
  }
  float s = (m_old > m_new ? m_old : m_new) / 448.0f;
  for (int i = 0; i < n_old; ++i) tile[i] = quant_fp8(xh[i], s);
  for (int i = 0; i < n * d; ++i) new_tile[i] = quant_fp8(new_x[i], s);
  *scale = s;
  free(xh);
}

static size_t code_row_bytes(int dtype, int d) {
  if (dtype == ORACLE_FP16) return (size_t)d * 2;
  if (dtype == ORACLE_INT8_SYM || dtype == ORACLE_FP8_E4M3) return (size_t)d;
  return (size_t)d / 2;
}

static int dtypes_ok(const oracle_cache* c) {
  if (c->k_dtype != ORACLE_FP16 && c->k_dtype != ORACLE_INT8_SYM && c->k_dtype != ORACLE_FP8_E4M3) return 0;
  if (c->v_dtype != ORACLE_FP16 && c->v_dtype != ORACLE_INT8_SYM && c->v_dtype != ORACLE_INT4_ASYM &&
      c->v_dtype != ORACLE_FP8_E4M3)
    return 0;
  return 1;
}

/* Store one side (K or V) of one group for one head. */
static void store_side(const oracle_cache* c, int which_v, int block, int head, int o0, int n,
                       const uint16_t* src, const float* vals) {
  int dtype = which_v ? c->v_dtype : c->k_dtype;
  size_t row = code_row_bytes(dtype, c->head_dim);
  uint8_t* base = (uint8_t*)(which_v ? c->v_codes : c->k_codes);
  uint8_t* tile = base + ((size_t)block * c->num_kv_heads + head) * c->block_size * row;
  size_t meta = (size_t)block * c->num_kv_heads + head;
  if (dtype == ORACLE_FP16) {
    /* unquantized side: the fp16 bits are stored as given */
    for (int t = 0; t < n; ++t)
      memcpy(tile + (size_t)(o0 + t) * row, src + (size_t)t * c->head_dim, row);
  } else if (dtype == ORACLE_INT8_SYM) {
    float* scale = which_v ? &c->v_scale[meta] : &c->k_scale[meta];
    store_tile_sym((int8_t*)tile, scale, c->head_dim, o0, n, vals);
  } else if (dtype == ORACLE_FP8_E4M3) {
    float* scale = which_v ? &c->v_scale[meta] : &c->k_scale[meta];
    store_tile_fp8(tile, scale, c->head_dim, o0, n, vals);
  } else {
    store_tile_asym4(tile, &c->v_scale[meta], &c->v_zp[meta], c->head_dim, o0, n, vals);
  }
}

int32_t oracle_store(const oracle_cache* c, const uint16_t* k_new, const uint16_t* v_new,
                     const int64_t* slot_mapping, int32_t T) {
  int32_t err = 0;
  if (!dtypes_ok(c)) return -1;
  const int bs = c->block_size, H = c->num_kv_heads, d = c->head_dim;
  const int64_t num_slots = (int64_t)c->num_blocks * bs;
  float* vals = (float*)malloc(sizeof(float) * (size_t)bs * d);
  uint16_t* raw = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)bs * d);
  int32_t t = 0;
  while (t < T) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) { /* R11: padding */
      ++t;
      continue;
    }
    if (slot >= num_slots) {
      record_error(&err, ORACLE_DEVERR_SLOT);
      ++t;
      continue;
    }
    /* a group: the maximal run of following tokens whose slots are valid and in the same block */
    int64_t block = slot / bs;
    int32_t end = t + 1;
    int consecutive = 1;
    while (end < T && slot_mapping[end] >= 0 && slot_mapping[end] < num_slots &&
           slot_mapping[end] / bs == block) {
      if (slot_mapping[end] != slot_mapping[end - 1] + 1) consecutive = 0;
      ++end;
    }
    if (!consecutive) {
      record_error(&err, ORACLE_DEVERR_SLOT_GROUP);
      t = end;
      continue;
    }
    int o0 = (int)(slot % bs);
    int n = end - t;
    for (int h = 0; h < H; ++h) {
      for (int side = 0; side < 2; ++side) {
        const uint16_t* src_all = side ? v_new : k_new;
        for (int i = 0; i < n; ++i) {
          const uint16_t* src = src_all + ((size_t)(t + i) * H + h) * d;
          for (int j = 0; j < d; ++j) {
            raw[i * d + j] = src[j];
            vals[i * d + j] = (float)half_bits_to_double(src[j]); /* exact widening */
          }
        }
        store_side(c, side, (int)block, h, o0, n, raw, vals);
      }
    }
    t = end;
  }
  free(vals);
  free(raw);
  return err;
}

int32_t oracle_copy_blocks(const oracle_cache* c, const int32_t* block_mapping, int32_t n_pairs) {
  int32_t err = 0;
  if (!dtypes_ok(c)) return -1;
  const int H = c->num_kv_heads;
  size_t k_block = (size_t)H * c->block_size * code_row_bytes(c->k_dtype, c->head_dim);
  size_t v_block = (size_t)H * c->block_size * code_row_bytes(c->v_dtype, c->head_dim);
  for (int32_t p = 0; p < n_pairs; ++p) {
    int32_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
    if (src < 0 || src >= c->num_blocks || dst < 0 || dst >= c->num_blocks) {
      record_error(&err, ORACLE_DEVERR_BLOCK_ID);
      continue;
    }
    memcpy((uint8_t*)c->k_codes + (size_t)dst * k_block, (uint8_t*)c->k_codes + (size_t)src * k_block, k_block);
    memcpy((uint8_t*)c->v_codes + (size_t)dst * v_block, (uint8_t*)c->v_codes + (size_t)src * v_block, v_block);
    if (c->k_dtype != ORACLE_FP16)
      memcpy(c->k_scale + (size_t)dst * H, c->k_scale + (size_t)src * H, sizeof(float) * H);
    if (c->v_dtype != ORACLE_FP16)
      memcpy(c->v_scale + (size_t)dst * H, c->v_scale + (size_t)src * H, sizeof(float) * H);
    if (c->v_dtype == ORACLE_INT4_ASYM)
      memcpy(c->v_zp + (size_t)dst * H, c->v_zp + (size_t)src * H, (size_t)H);
  }
  return err;
}

/* Dequantized value of dimension j of token `off` in (block, head), as binary64.
 * k_hat = Q * scale; v_hat = (Q - zp) * scale ([yunthe] x_hat formula); fp16 as stored. */
static double dequant(const oracle_cache* c, int which_v, int block, int head, int off, int j) {
  int dtype = which_v ? c->v_dtype : c->k_dtype;
  size_t row = code_row_bytes(dtype, c->head_dim);
  const uint8_t* base = (const uint8_t*)(which_v ? c->v_codes : c->k_codes);
  const uint8_t* r = base + (((size_t)block * c->num_kv_heads + head) * c->block_size + off) * row;
  size_t meta = (size_t)block * c->num_kv_heads + head;
  if (dtype == ORACLE_FP16) {
    uint16_t bits;
    memcpy(&bits, r + 2 * (size_t)j, 2);
    return half_bits_to_double(bits);
  }
  if (dtype == ORACLE_INT8_SYM) {
    double s = which_v ? (double)c->v_scale[meta] : (double)c->k_scale[meta];
    return (double)((const int8_t*)r)[j] * s;
  }
  if (dtype == ORACLE_FP8_E4M3) { /* x_hat = value(code) * scale (R15) */
    double s = which_v ? (double)c->v_scale[meta] : (double)c->k_scale[meta];
    return oracle_fp8_e4m3_decode(r[j]) * s;
  }
  return ((double)get_nibble(r, j) - (double)c->v_zp[meta]) * (double)c->v_scale[meta];
}

/* Attention of one query row (fp16 bits, head_dim values) over tokens [0, L) of one sequence
 * (its block-table row), KV head g, in binary64: z_t = scale * q . k_hat_t, out = sum_t softmax(z)_t
 * v_hat_t. A block id outside the pool leaves its tokens out and is reported. */
static int32_t attend_row(const oracle_cache* c, const uint16_t* qrow, const int32_t* table_row, int L, int g,
                          float softmax_scale, double* o) {
  const int d = c->head_dim, bs = c->block_size;
  int32_t local_err = 0;
  for (int j = 0; j < d; ++j) o[j] = 0.0;
  double qv[512];
  for (int j = 0; j < d; ++j) qv[j] = half_bits_to_double(qrow[j]);
  /* logits z_t = scale * q . k_hat_t for every valid token */
  double* z = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  int* valid = (int*)malloc(sizeof(int) * (size_t)(L > 0 ? L : 1));
  double zmax = -INFINITY;
  for (int t = 0; t < L; ++t) {
    int block = table_row[t / bs];
    valid[t] = (block >= 0 && block < c->num_blocks);
    if (!valid[t]) {
      local_err = ORACLE_DEVERR_BLOCK_ID;
      continue;
    }
    double dot = 0.0;
    for (int j = 0; j < d; ++j) dot += qv[j] * dequant(c, 0, block, g, t % bs, j);
    z[t] = (double)softmax_scale * dot;
    if (z[t] > zmax) zmax = z[t];
  }
  /* softmax over the valid tokens, then the weighted sum of v_hat */
  double denom = 0.0;
  for (int t = 0; t < L; ++t) {
    if (!valid[t]) continue;
    double w = exp(z[t] - zmax);
    denom += w;
    int block = table_row[t / bs];
    for (int j = 0; j < d; ++j) o[j] += w * dequant(c, 1, block, g, t % bs, j);
  }
  if (denom > 0.0)
    for (int j = 0; j < d; ++j) o[j] /= denom;
  free(z);
  free(valid);
  return local_err;
}

int32_t oracle_decode(const oracle_cache* c, const uint16_t* q, int32_t num_seqs, int32_t num_q_heads,
                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                      const int32_t* context_lens, int32_t max_context_len, float softmax_scale,
                      double* out, int32_t num_threads) {
  if (!dtypes_ok(c) || c->head_dim > 512) return -1;
  const int H = c->num_kv_heads, d = c->head_dim, bs = c->block_size;
  if (H <= 0 || num_q_heads % H != 0) return -1;
  const int G = num_q_heads / H;
  int32_t err = 0;
  const int64_t pairs = (int64_t)num_seqs * num_q_heads;
  if (num_threads <= 0) num_threads = 1;

#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads)
  for (int64_t sh = 0; sh < pairs; ++sh) {
    const int s = (int)(sh / num_q_heads), h = (int)(sh % num_q_heads);
    const int g = h / G; /* query head h reads KV head h / G */
    int32_t local_err = 0;
    int L = context_lens[s];
    if (L < 0 || L > max_context_len || L > max_blocks_per_seq * bs) {
      local_err = ORACLE_DEVERR_CONTEXT_LEN;
      if (L < 0) L = 0;
      if (L > max_context_len) L = max_context_len;
      if (L > max_blocks_per_seq * bs) L = max_blocks_per_seq * bs;
    }
    int32_t row_err = attend_row(c, q + (size_t)sh * d, block_tables + (size_t)s * max_blocks_per_seq, L, g,
                                 softmax_scale, out + (size_t)sh * d);
    if (!local_err) local_err = row_err;
    if (local_err) {
#pragma omp critical
      record_error(&err, local_err);
    }
  }
  return err;
}

/* Chunked prefill ([yunthe] "Prefix Caching与多轮对话场景优化实践": only the new tokens are computed,
 * attending over the cached prefix; [tbr8] §5 item 2: dequantization inside the attention
 * operator). Sequence s contributes q_len = cu_q_lens[s+1] - cu_q_lens[s] query tokens, the last
 * q_len of its context_lens[s] tokens (already stored): the query at position
 * p = context_lens[s] - q_len + i attends causally to tokens [0, p], i.e. it is the decode of that
 * query over a context of p + 1 tokens. */
int32_t oracle_prefill(const oracle_cache* c, const uint16_t* q, int32_t num_seqs, int32_t num_q_heads,
                       const int32_t* cu_q_lens, const int32_t* block_tables, int32_t max_blocks_per_seq,
                       const int32_t* context_lens, float softmax_scale, double* out, int32_t num_threads) {
  if (!dtypes_ok(c) || c->head_dim > 512) return -1;
  const int H = c->num_kv_heads, d = c->head_dim, bs = c->block_size;
  if (H <= 0 || num_q_heads % H != 0) return -1;
  const int G = num_q_heads / H;
  int32_t err = 0;
  if (num_threads <= 0) num_threads = 1;
  const int64_t rows = num_seqs > 0 ? (int64_t)cu_q_lens[num_seqs] * num_q_heads : 0;

#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads)
  for (int64_t rh = 0; rh < rows; ++rh) {
    const int64_t row = rh / num_q_heads;
    const int h = (int)(rh % num_q_heads);
    int s = 0;
    while (s + 1 < num_seqs && cu_q_lens[s + 1] <= row) ++s; /* the sequence holding this row */
    const int q_len = cu_q_lens[s + 1] - cu_q_lens[s];
    const int i = (int)(row - cu_q_lens[s]);
    double* o = out + (size_t)rh * d;
    int32_t local_err = 0;
    int L = context_lens[s] - q_len + i + 1; /* causal: positions 0 .. p */
    if (q_len > context_lens[s] || L < 1) {
      local_err = ORACLE_DEVERR_CONTEXT_LEN;
      for (int j = 0; j < d; ++j) o[j] = 0.0;
    } else {
      if (L > max_blocks_per_seq * bs) {
        local_err = ORACLE_DEVERR_CONTEXT_LEN;
        L = max_blocks_per_seq * bs;
      }
      int32_t row_err = attend_row(c, q + (size_t)rh * d, block_tables + (size_t)s * max_blocks_per_seq, L, h / G,
                                   softmax_scale, o);
      if (!local_err) local_err = row_err;
    }
    if (local_err) {
#pragma omp critical
      record_error(&err, local_err);
    }
  }
  return err;
}
