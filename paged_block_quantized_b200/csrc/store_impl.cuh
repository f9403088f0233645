// store_impl.cuh -- the store's device code: quantize new K/V tokens and scatter them into pool
// blocks, one warp per (token, KV head). Used by the store kernel (store.cu) and by the fused
// decode step (decode_kernel.cuh).
//
// Follows tbr8.org "如何通过 PagedAttention 与分块量化结合：解决移动端内存碎片化导致的长文本 OOM" §4
// (store_kv: scale = absmax / 127 per block, codes = x / scale, one scale stored per block and
// head) and yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section
// "KV Cache量化技术原理" (asymmetric Q(x) = clamp(round(x/scale + zero_point), 0, 2^bits - 1)),
// with K INT8 / V INT4 as the tbr8.org page advises in §5 item 1. Readings where the pages are
// silent: ties round to even; INT8 codes in [-127, 127]; INT4 range [min(0, min x), max(0, max x)],
// scale = (hi - lo) / 15, zp = clamp(rint(-lo / scale), 0, 15); scale 0 encodes an all-zero tile;
// nibbles packed along head_dim, low nibble = even dim; appending into a partly filled tile keeps
// the stored scale when every new value fits and otherwise rebuilds the tile from the
// dequantized old codes plus the new values.
//
// Bit-exactness: every arithmetic step is an explicit IEEE binary32 round-to-nearest intrinsic
// (__fdiv_rn, __fmul_rn, __fadd_rn, __fsub_rn) so nvcc cannot contract or reorder it, and
// __float2int_rn rounds half to even. Maxima and minima are order independent. Two shortcuts
// give the same results as the element-wise rule, because every step involved (x / s, + zp,
// code * s, rint) is monotone for s >= 0 and round-to-nearest is symmetric about zero:
//  - "every new value fits" is decided from the extremes alone: |x| <= m gives
//    |rint(x / s)| <= rint(m / s), and lo <= x <= hi brackets rint(x / s + zp);
//  - a rebuild's range over the dequantized old values comes from the largest |code| (INT8) or
//    the smallest and largest code (INT4), and requantizing an old code depends on the code
//    alone, so each tile's old codes go through a 256-entry table built once per rebuild.
//
// FP8 E4M3 (yunthe.com, same page, section "vLLM推理引擎部署与KV Cache量化配置实战": the fp8 cache
// mode stores E4M3 values): scale = absmax / 448 per (block, head), code = E4M3(x / scale) rounded
// to nearest even and saturated (the hardware conversion), new values fit a stored scale when
// |x / scale| <= 448; a rebuild requantizes old codes through the same kind of 256-entry table
// (an E4M3 code's requantized value depends on the code alone).
//
// Work split: one warp per (token, KV head). The warp of the first token of a group (the run of
// tokens bound for one block) does the whole group; the others return at once.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace pkv {
namespace store_detail {
namespace {

constexpr uint32_t kFull = 0xffffffffu;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fminf(v, __shfl_xor_sync(kFull, v, off));
  return v;
}

// 4 fp16 values at p (8-byte aligned) -> floats (exact widening)
__device__ __forceinline__ void load4(const __half* p, float f[4]) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
  f[0] = a.x;
  f[1] = a.y;
  f[2] = b.x;
  f[3] = b.y;
}

// symmetric: 0 if s == 0, else clamp(rint(x / s), -127, 127)
__device__ __forceinline__ int quant_sym(float x, float s) {
  if (s == 0.0f) return 0;
  const int r = __float2int_rn(__fdiv_rn(x, s));
  return min(127, max(-127, r));
}

// asymmetric 4-bit: zp if s == 0, else clamp(rint(x / s + zp), 0, 15)
__device__ __forceinline__ int quant_asym(float x, float s, int zp) {
  if (s == 0.0f) return zp;
  const int r = __float2int_rn(__fadd_rn(__fdiv_rn(x, s), (float)zp));
  return min(15, max(0, r));
}

__device__ __forceinline__ void derive_asym(float lo, float hi, float& s, int& zp) {
  s = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
  zp = 0;
  if (s != 0.0f) zp = min(15, max(0, __float2int_rn(__fdiv_rn(-lo, s))));
}

// Do new values with largest magnitude m all fit a stored INT8 scale? (|rint(m / s)| <= 127; a zero
// scale holds zeros only)
__device__ __forceinline__ bool fits_sym(float m, float s_old) {
  if (s_old == 0.0f) return m == 0.0f;
  return __float2int_rn(__fdiv_rn(m, s_old)) <= 127;
}

// Do new values in [lo, hi] all fit a stored INT4 scale and zero point?
__device__ __forceinline__ bool fits_asym(float lo, float hi, float s_old, int zp_old) {
  if (s_old == 0.0f) return lo == 0.0f && hi == 0.0f;
  const int r_lo = __float2int_rn(__fadd_rn(__fdiv_rn(lo, s_old), (float)zp_old));
  const int r_hi = __float2int_rn(__fadd_rn(__fdiv_rn(hi, s_old), (float)zp_old));
  return r_lo >= 0 && r_hi <= 15;
}

// E4M3 code of x / s (nearest even, saturated at +-448); 0 if s == 0
__device__ __forceinline__ uint32_t quant_fp8(float x, float s) {
  if (s == 0.0f) return 0u;
  return (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(x, s), __NV_SATFINITE, __NV_E4M3);
}
// value of an E4M3 code (exact in binary32)
__device__ __forceinline__ float fp8_value(uint32_t code) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3)));
}
// Do new values with largest magnitude m all fit a stored E4M3 scale? (|m / s| <= 448)
__device__ __forceinline__ bool fits_fp8(float m, float s_old) {
  if (s_old == 0.0f) return m == 0.0f;
  return __fdiv_rn(m, s_old) <= 448.0f;
}

// four bytes of w through a 256-entry table (after xor-ing w with flip)
__device__ __forceinline__ uint32_t translate4(uint32_t w, uint32_t flip, const uint8_t* tbl) {
  const uint32_t x = w ^ flip;
  return (uint32_t)tbl[x & 0xffu] | ((uint32_t)tbl[(x >> 8) & 0xffu] << 8) |
         ((uint32_t)tbl[(x >> 16) & 0xffu] << 16) | ((uint32_t)tbl[x >> 24] << 24);
}
__device__ __forceinline__ uint4 translate16(uint4 v, uint32_t flip, const uint8_t* tbl) {
  return make_uint4(translate4(v.x, flip, tbl), translate4(v.y, flip, tbl), translate4(v.z, flip, tbl),
                    translate4(v.w, flip, tbl));
}

// Per-byte comparisons of four packed values in 0 .. 15 (one per byte): (a | 16) - b keeps each
// byte in 1 .. 31 (no borrow into the next byte), and its bit 4 says a >= b.
__device__ __forceinline__ uint32_t nibble_ge(uint32_t a, uint32_t b) {
  return (((a | 0x10101010u) - b) >> 4 & 0x01010101u) * 0xFFu;  // 0xFF in each byte where a >= b
}
__device__ __forceinline__ uint32_t bitsel(uint32_t m, uint32_t a, uint32_t b) { return (a & m) | (b & ~m); }

// largest |code| among the 16 INT8 codes of v
__device__ __forceinline__ int32_t absmax16(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  int32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int32_t x = (int32_t)w[i];
    m = max(m, max(max(abs((int32_t)(int8_t)x), abs((int32_t)(int8_t)(x >> 8))),
                   max(abs((int32_t)(int8_t)(x >> 16)), abs(x >> 24))));
  }
  return m;
}

// per-byte smallest / largest of the 32 nibble codes of v, folded into mn / mx
__device__ __forceinline__ void nibble_minmax32(uint4 v, uint32_t& mn, uint32_t& mx) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t l4 = w[i] & 0x0F0F0F0Fu, h4 = (w[i] >> 4) & 0x0F0F0F0Fu;
    const uint32_t ge = nibble_ge(l4, h4);
    const uint32_t hi = bitsel(ge, l4, h4), lo = bitsel(ge, h4, l4);
    mx = bitsel(nibble_ge(mx, hi), mx, hi);
    mn = bitsel(nibble_ge(mn, lo), lo, mn);
  }
}

// A rebuild reads a tile's old rows as 16-byte vectors, kChunkVecs at a time: vector e of chunk c
// is c * kChunkVecs + j * 32 + lane for j < 4, so each j is one coalesced 512-byte access and the
// four loads of a chunk are in flight together. The per-vector work runs in a loop that is not
// unrolled, over v[0] with the registers rotated, which keeps the code small.
constexpr int kChunkVecs = 128;

__device__ __forceinline__ void load_chunk(const uint4* v16, int nvec, int c, int lane, uint4 v[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = c * kChunkVecs + j * 32 + lane;
    v[j] = e < nvec ? v16[e] : make_uint4(0u, 0u, 0u, 0u);
  }
}
__device__ __forceinline__ void rotate(uint4 v[4]) {
  const uint4 t = v[0];
  v[0] = v[1];
  v[1] = v[2];
  v[2] = v[3];
  v[3] = t;
}

// Requantize the old rows in place through tbl: chunks again (a single chunk is still in v).
__device__ __forceinline__ void requant_rows(uint4* v16, int nvec, int nchunks, uint32_t flip, const uint8_t* tbl,
                                             int lane, uint4 v[4]) {
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    if (nchunks > 1) load_chunk(v16, nvec, c, lane, v);
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      const int e = c * kChunkVecs + j * 32 + lane;
      if (e < nvec) v16[e] = translate16(v[0], flip, tbl);
      rotate(v);
    }
  }
}

// Rebuild of the old rows [0, o0) of an INT8 tile (rows of d codes) for values that do not fit
// the stored scale s_old: x_hat = code * s_old (binary32), new scale = max(max |x_hat|, m_new) / 127,
// old codes requantized to it. Returns the new scale. tbl: 256 bytes of this warp's shared memory.
__device__ __noinline__ float rebuild_sym(int8_t* tile, int d, int o0, float s_old, float m_new, uint8_t* tbl, int lane) {
  uint4* v16 = reinterpret_cast<uint4*>(tile);
  const int nvec = o0 * d / 16;
  const int nchunks = (nvec + kChunkVecs - 1) / kChunkVecs;
  uint4 v[4];
  int32_t amax = 0;  // largest |code| (vectors past the end read as zeros)
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    load_chunk(v16, nvec, c, lane, v);
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      amax = max(amax, absmax16(v[0]));
      rotate(v);
    }
  }
  const int32_t qmax = __reduce_max_sync(kFull, amax);
  const float m_old = __fmul_rn((float)qmax, s_old);
  const float s = __fdiv_rn(fmaxf(m_old, m_new), 127.0f);
  // table entry (code + 128): the code's requantized value; lane l fills entries 8l .. 8l+7
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int code = lane * 8 + j - 128;
    const uint32_t c = (uint32_t)(quant_sym(__fmul_rn((float)code, s_old), s) & 0xff);
    if (j < 4) lo |= c << (8 * j); else hi |= c << (8 * (j - 4));
  }
  reinterpret_cast<uint2*>(tbl)[lane] = make_uint2(lo, hi);
  __syncwarp();
  requant_rows(v16, nvec, nchunks, 0x80808080u, tbl, lane, v);  // byte b holds code (int8)b: entry b ^ 0x80
  __syncwarp();
  return s;
}

// largest magnitude field (code & 0x7f) among the 16 E4M3 codes of v: E4M3 magnitudes ascend with
// their 7-bit pattern, so this code has the largest |value|
__device__ __forceinline__ uint32_t fp8_magmax16(uint4 v) {
  const uint32_t w[4] = {v.x & 0x7f7f7f7fu, v.y & 0x7f7f7f7fu, v.z & 0x7f7f7f7fu, v.w & 0x7f7f7f7fu};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(max(m, max(w[i] & 0xffu, (w[i] >> 8) & 0xffu)), max((w[i] >> 16) & 0xffu, w[i] >> 24));
  return m;
}

// Rebuild of the old rows [0, o0) of an E4M3 tile (rows of d codes) for values that do not fit:
// x_hat = value(code) * s_old (binary32), new scale = max(max |x_hat|, m_new) / 448, old codes
// requantized through a table. Returns the new scale.
__device__ __noinline__ float rebuild_fp8(uint8_t* tile, int d, int o0, float s_old, float m_new, uint8_t* tbl,
                                          int lane) {
  uint4* v16 = reinterpret_cast<uint4*>(tile);
  const int nvec = o0 * d / 16;
  const int nchunks = (nvec + kChunkVecs - 1) / kChunkVecs;
  uint4 v[4];
  uint32_t qmax = 0;
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    load_chunk(v16, nvec, c, lane, v);
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      qmax = max(qmax, fp8_magmax16(v[0]));
      rotate(v);
    }
  }
  qmax = __reduce_max_sync(kFull, qmax);
  const float m_old = __fmul_rn(fp8_value(qmax), s_old);
  const float s = __fdiv_rn(fmaxf(m_old, m_new), 448.0f);
  // table entry b: the requantized code of code b; lane l fills entries 8l .. 8l+7
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t b = (uint32_t)(lane * 8 + j);
    const uint32_t c = quant_fp8(__fmul_rn(fp8_value(b), s_old), s);
    if (j < 4) lo |= c << (8 * j); else hi |= c << (8 * (j - 4));
  }
  reinterpret_cast<uint2*>(tbl)[lane] = make_uint2(lo, hi);
  __syncwarp();
  requant_rows(v16, nvec, nchunks, 0u, tbl, lane, v);
  __syncwarp();
  return s;
}

// Rebuild of the old rows [0, o0) of an INT4 tile (rows of d / 2 bytes) for values that do not
// fit: x_hat = (code - zp_old) * s_old (binary32), range [min(lo_new, x_hat), max(hi_new, x_hat)],
// new scale and zero point from it, old codes requantized. tbl: 256 bytes of shared memory.
__device__ __noinline__ void rebuild_asym4(uint8_t* tile, int d, int o0, float s_old, int zp_old, float lo_new,
                                           float hi_new, uint8_t* tbl, int lane, float& s_out, int& zp_out) {
  uint4* v16 = reinterpret_cast<uint4*>(tile);
  const int nvec = o0 * d / 32;
  const int nchunks = (nvec + kChunkVecs - 1) / kChunkVecs;
  uint4 v[4];
  uint32_t mn = 0x0F0F0F0Fu, mx = 0u;  // per byte: smallest / largest code seen
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    load_chunk(v16, nvec, c, lane, v);
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      if (c * kChunkVecs + j * 32 + lane < nvec) nibble_minmax32(v[0], mn, mx);
      rotate(v);
    }
  }
  // a lane with no old vectors keeps 15 / 0, which leave the warp's minimum / maximum alone
  const uint32_t qmin =
      __reduce_min_sync(kFull, min(min(mn & 0xffu, (mn >> 8) & 0xffu), min((mn >> 16) & 0xffu, mn >> 24)));
  const uint32_t qmax =
      __reduce_max_sync(kFull, max(max(mx & 0xffu, (mx >> 8) & 0xffu), max((mx >> 16) & 0xffu, mx >> 24)));
  const float lo = fminf(lo_new, __fmul_rn((float)((int)qmin - zp_old), s_old));
  const float hi = fmaxf(hi_new, __fmul_rn((float)((int)qmax - zp_old), s_old));
  float s;
  int zp;
  derive_asym(lo, hi, s, zp);
  // lane k < 16: requantized value of code k; byte table entry b = T[b & 15] | T[b >> 4] << 4
  const int t_k = quant_asym(__fmul_rn((float)((lane & 15) - zp_old), s_old), s, zp);
  const uint32_t t_hi = (uint32_t)__shfl_sync(kFull, t_k, lane >> 1);  // b >> 4 for b = 8 lane + j
  uint32_t lo_w = 0, hi_w = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t t_lo = (uint32_t)__shfl_sync(kFull, t_k, (lane * 8 + j) & 15);
    const uint32_t c = t_lo | (t_hi << 4);
    if (j < 4) lo_w |= c << (8 * j); else hi_w |= c << (8 * (j - 4));
  }
  reinterpret_cast<uint2*>(tbl)[lane] = make_uint2(lo_w, hi_w);
  __syncwarp();
  requant_rows(v16, nvec, nchunks, 0u, tbl, lane, v);
  __syncwarp();
  s_out = s;
  zp_out = zp;
}

// Values of the group for one head: element e of token i at src + i * row_stride + e.
struct GroupSrc {
  const __half* base;  // token 0 of the group, this head
  int64_t row_stride;  // elements between tokens (num_kv_heads * head_dim)
  int n;               // tokens in the group
  int d;               // head_dim
};

// ---- groups of several tokens (prefill chunks): INT8 symmetric side of one (block, head) tile ----
__device__ __noinline__ void store_sym(const GroupSrc& src, int8_t* tile, float* scale_ptr, int o0, uint8_t* tbl,
                                       int lane) {
  const int d = src.d, n = src.n;
  const int quads = n * d / 4;
  float m_new = 0.0f;
  for (int e = lane; e < quads; e += 32) {
    const int i = (4 * e) / d, j = (4 * e) % d;
    float f[4];
    load4(src.base + i * src.row_stride + j, f);
#pragma unroll
    for (int u = 0; u < 4; ++u) m_new = fmaxf(m_new, fabsf(f[u]));
  }
  m_new = warp_max(m_new);
  float s;
  if (o0 == 0) {
    s = __fdiv_rn(m_new, 127.0f);
  } else {
    const float s_old = *scale_ptr;
    s = fits_sym(m_new, s_old) ? s_old : rebuild_sym(tile, d, o0, s_old, m_new, tbl, lane);
  }
  int8_t* dst = tile + (size_t)o0 * d;
  for (int e = lane; e < quads; e += 32) {
    const int i = (4 * e) / d, j = (4 * e) % d;
    float f[4];
    load4(src.base + i * src.row_stride + j, f);
    uint32_t out = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) out |= ((uint32_t)(quant_sym(f[u], s) & 0xff)) << (8 * u);
    reinterpret_cast<uint32_t*>(dst)[e] = out;
  }
  if (lane == 0) *scale_ptr = s;
}

// ---- E4M3 side of one (block, head) tile, groups of several tokens ----
__device__ __noinline__ void store_fp8(const GroupSrc& src, uint8_t* tile, float* scale_ptr, int o0, uint8_t* tbl,
                                       int lane) {
  const int d = src.d, n = src.n;
  const int quads = n * d / 4;
  float m_new = 0.0f;
  for (int e = lane; e < quads; e += 32) {
    const int i = (4 * e) / d, j = (4 * e) % d;
    float f[4];
    load4(src.base + i * src.row_stride + j, f);
#pragma unroll
    for (int u = 0; u < 4; ++u) m_new = fmaxf(m_new, fabsf(f[u]));
  }
  m_new = warp_max(m_new);
  float s;
  if (o0 == 0) {
    s = __fdiv_rn(m_new, 448.0f);
  } else {
    const float s_old = *scale_ptr;
    s = fits_fp8(m_new, s_old) ? s_old : rebuild_fp8(tile, d, o0, s_old, m_new, tbl, lane);
  }
  uint8_t* dst = tile + (size_t)o0 * d;
  for (int e = lane; e < quads; e += 32) {
    const int i = (4 * e) / d, j = (4 * e) % d;
    float f[4];
    load4(src.base + i * src.row_stride + j, f);
    uint32_t out = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) out |= quant_fp8(f[u], s) << (8 * u);
    reinterpret_cast<uint32_t*>(dst)[e] = out;
  }
  if (lane == 0) *scale_ptr = s;
}

// ---- INT4 asymmetric side: tile is [bs][d/2] bytes, byte j = code[2j] | code[2j+1] << 4 ----
__device__ __noinline__ void store_asym4(const GroupSrc& src, uint8_t* tile, float* scale_ptr, uint8_t* zp_ptr, int o0,
                                         uint8_t* tbl, int lane) {
  const int d = src.d, n = src.n;
  const int quads = n * d / 4;  // 4 values -> 2 bytes
  float lo = 0.0f, hi = 0.0f;
  for (int e = lane; e < quads; e += 32) {
    const int i = (4 * e) / d, j = (4 * e) % d;
    float f[4];
    load4(src.base + i * src.row_stride + j, f);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      lo = fminf(lo, f[u]);
      hi = fmaxf(hi, f[u]);
    }
  }
  lo = warp_min(lo);
  hi = warp_max(hi);
  float s;
  int zp;
  if (o0 == 0) {
    derive_asym(lo, hi, s, zp);
  } else {
    const float s_old = *scale_ptr;
    const int zp_old = *zp_ptr;
    if (fits_asym(lo, hi, s_old, zp_old)) {
      s = s_old;
      zp = zp_old;
    } else {
      rebuild_asym4(tile, d, o0, s_old, zp_old, lo, hi, tbl, lane, s, zp);
    }
  }
  uint8_t* dst = tile + (size_t)o0 * (d / 2);
  for (int e = lane; e < quads; e += 32) {
    const int i = (4 * e) / d, j = (4 * e) % d;
    float f[4];
    load4(src.base + i * src.row_stride + j, f);
    const uint32_t b0 = (uint32_t)(quant_asym(f[0], s, zp) | (quant_asym(f[1], s, zp) << 4));
    const uint32_t b1 = (uint32_t)(quant_asym(f[2], s, zp) | (quant_asym(f[3], s, zp) << 4));
    reinterpret_cast<uint16_t*>(dst)[e] = (uint16_t)(b0 | (b1 << 8));
  }
  if (lane == 0) {
    *scale_ptr = s;
    *zp_ptr = (uint8_t)zp;
  }
}

// ---- FP16 side: values stored as given ----
__device__ __noinline__ void store_fp16(const GroupSrc& src, __half* tile, int o0, int lane) {
  const int d = src.d, n = src.n;
  const int vecs = n * d / 8;  // 16-byte vectors
  __half* dst = tile + (size_t)o0 * d;
  for (int e = lane; e < vecs; e += 32) {
    const int i = (8 * e) / d, j = (8 * e) % d;
    reinterpret_cast<uint4*>(dst + (size_t)i * d)[j / 8] =
        *reinterpret_cast<const uint4*>(src.base + i * src.row_stride + j);
  }
}

// ---- single-token groups (the decode-step append): the token in registers ----
// A lane holds vpl = head_dim / 32 consecutive values (2, 4 or 8) of the token for one head.
__device__ __forceinline__ void load_halves(const __half* src, int vpl, uint32_t raw[4]) {
  raw[0] = raw[1] = raw[2] = raw[3] = 0;
  if (vpl == 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(src);
    raw[0] = w.x; raw[1] = w.y; raw[2] = w.z; raw[3] = w.w;
  } else if (vpl == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(src);
    raw[0] = w.x; raw[1] = w.y;
  } else {
    raw[0] = *reinterpret_cast<const uint32_t*>(src);
  }
}
__device__ __forceinline__ void halves_to_float(const uint32_t raw[4], float x[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&raw[i]));
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// INT8 symmetric side of a one-token group at offset o0 (s_old: the stored scale when o0 > 0).
__device__ __forceinline__ void append_sym(const float x[8], int vpl, int8_t* tile, float* scale_ptr, float s_old,
                                          int o0, int d, uint8_t* tbl, int lane) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < vpl) m = fmaxf(m, fabsf(x[i]));
  m = warp_max(m);
  float s;
  bool set_scale = true;
  if (o0 == 0) {
    s = __fdiv_rn(m, 127.0f);
  } else if (fits_sym(m, s_old)) {
    s = s_old;
    set_scale = false;
  } else {
    s = rebuild_sym(tile, d, o0, s_old, m, tbl, lane);
  }
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i >= vpl) continue;
    const uint32_t c = (uint32_t)(quant_sym(x[i], s) & 0xff);
    if (i < 4) lo |= c << (8 * i); else hi |= c << (8 * (i - 4));
  }
  int8_t* dst = tile + (size_t)o0 * d + lane * vpl;
  if (vpl == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
  else if (vpl == 4) *reinterpret_cast<uint32_t*>(dst) = lo;
  else *reinterpret_cast<uint16_t*>(dst) = (uint16_t)lo;
  if (set_scale && lane == 0) *scale_ptr = s;
}

// E4M3 side of a one-token group at offset o0 (s_old: the stored scale when o0 > 0).
__device__ __forceinline__ void append_fp8(const float x[8], int vpl, uint8_t* tile, float* scale_ptr, float s_old,
                                          int o0, int d, uint8_t* tbl, int lane) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < vpl) m = fmaxf(m, fabsf(x[i]));
  m = warp_max(m);
  float s;
  bool set_scale = true;
  if (o0 == 0) {
    s = __fdiv_rn(m, 448.0f);
  } else if (fits_fp8(m, s_old)) {
    s = s_old;
    set_scale = false;
  } else {
    s = rebuild_fp8(tile, d, o0, s_old, m, tbl, lane);
  }
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i >= vpl) continue;
    const uint32_t c = quant_fp8(x[i], s);
    if (i < 4) lo |= c << (8 * i); else hi |= c << (8 * (i - 4));
  }
  uint8_t* dst = tile + (size_t)o0 * d + lane * vpl;
  if (vpl == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
  else if (vpl == 4) *reinterpret_cast<uint32_t*>(dst) = lo;
  else *reinterpret_cast<uint16_t*>(dst) = (uint16_t)lo;
  if (set_scale && lane == 0) *scale_ptr = s;
}

// INT4 asymmetric side of a one-token group at offset o0.
__device__ __forceinline__ void append_asym4(const float x[8], int vpl, uint8_t* tile, float* scale_ptr, uint8_t* zp_ptr,
                                             float s_old, int zp_old, int o0, int d, uint8_t* tbl, int lane) {
  float lo = 0.0f, hi = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i >= vpl) continue;
    lo = fminf(lo, x[i]);
    hi = fmaxf(hi, x[i]);
  }
  lo = warp_min(lo);
  hi = warp_max(hi);
  float s;
  int zp;
  bool set_scale = true;
  if (o0 == 0) {
    derive_asym(lo, hi, s, zp);
  } else if (fits_asym(lo, hi, s_old, zp_old)) {
    s = s_old;
    zp = zp_old;
    set_scale = false;
  } else {
    rebuild_asym4(tile, d, o0, s_old, zp_old, lo, hi, tbl, lane, s, zp);
  }
  uint32_t packed = 0;  // vpl / 2 bytes: byte j = code[2j] | code[2j+1] << 4
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    if (i >= vpl) continue;
    const uint32_t b = (uint32_t)(quant_asym(x[i], s, zp) | (quant_asym(x[i + 1], s, zp) << 4));
    packed |= b << (4 * i);
  }
  uint8_t* dst = tile + (size_t)o0 * (d / 2) + lane * (vpl / 2);
  if (vpl == 8) *reinterpret_cast<uint32_t*>(dst) = packed;
  else if (vpl == 4) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
  else *dst = (uint8_t)packed;
  if (set_scale && lane == 0) {
    *scale_ptr = s;
    *zp_ptr = (uint8_t)zp;
  }
}

__device__ __forceinline__ void append_fp16(const uint32_t raw[4], int vpl, __half* tile, int o0, int d, int lane) {
  __half* dst = tile + (size_t)o0 * d + lane * vpl;
  if (vpl == 8) *reinterpret_cast<uint4*>(dst) = make_uint4(raw[0], raw[1], raw[2], raw[3]);
  else if (vpl == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(raw[0], raw[1]);
  else *reinterpret_cast<uint32_t*>(dst) = raw[0];
}

// One (token t, KV head h) of a store: the warp of the first token of a group (the run of tokens
// bound for one block) stores the whole group for head h; the warps of the other tokens return.
// tbl: 256 bytes of shared memory owned by this warp (a rebuild's code table).
template <int KT, int VT>
__device__ __forceinline__ void store_job(const StoreParams& p, const int t, const int h, const int lane, uint8_t* tbl) {
  if (h >= p.num_kv_heads) return;
  const int bs = p.block_size;
  const int d = p.head_dim;
  const int vpl = d / 32;
  const int64_t num_slots = (int64_t)p.num_blocks * bs;
  const int64_t row_stride = (int64_t)p.num_kv_heads * d;

  // ---- one round of independent loads: the slots of tokens t-1 .. t+30 (lane i holds token
  // t-1+i) and this token's own K and V values for this head ----
  const int idx = t - 1 + lane;
  int64_t sl = INT64_MIN;  // "no token"
  if (idx >= 0 && idx < p.T) sl = p.slot_mapping[idx];
  uint32_t kraw[4], vraw[4];
  load_halves(p.k_new + (size_t)t * row_stride + (size_t)h * d + lane * vpl, vpl, kraw);
  load_halves(p.v_new + (size_t)t * row_stride + (size_t)h * d + lane * vpl, vpl, vraw);

  const int64_t slot = __shfl_sync(kFull, sl, 1);
  const int64_t prev = __shfl_sync(kFull, sl, 0);
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (h == 0 && lane == 0) record_error(p.dev_error, PKV_DEVERR_SLOT);
    return;
  }
  const int64_t block = slot / bs;
  if (prev >= 0 && prev < num_slots && prev / bs == block) return;  // not the group's first token

  // the group: following tokens with a valid slot in the same block; offsets must be consecutive
  int n = 1;
  bool consecutive = true;
  {
    const bool same = lane >= 2 && sl >= 0 && sl < num_slots && sl / bs == block;
    const bool step_ok = sl == slot + (lane - 1);
    const uint32_t m = __ballot_sync(kFull, same) >> 2;  // bit k: token t+1+k
    const int run = (m == 0x3FFFFFFFu) ? 30 : (__ffs(~m) - 1);
    if (__ballot_sync(kFull, same && !step_ok && lane - 2 < run)) consecutive = false;
    n += run;
  }
  if (n == 31) {  // the group may go on beyond token t+30
    while (true) {
      const int i2 = t + n + lane;
      bool same = false, step_ok = true;
      if (i2 < p.T) {
        const int64_t s2 = p.slot_mapping[i2];
        same = s2 >= 0 && s2 < num_slots && s2 / bs == block;
        step_ok = s2 == slot + n + lane;
      }
      const uint32_t run_mask = __ballot_sync(kFull, same);
      const int run = (run_mask == kFull) ? 32 : (__ffs(~run_mask) - 1);
      if (__ballot_sync(kFull, same && !step_ok && lane < run)) consecutive = false;
      n += run;
      if (run < 32 || n > bs) break;
    }
  }
  if (!consecutive || n > bs) {
    if (h == 0 && lane == 0) record_error(p.dev_error, PKV_DEVERR_SLOT_GROUP);
    return;
  }
  const int o0 = (int)(slot % bs);
  const size_t tile_idx = (size_t)block * p.num_kv_heads + h;
  int8_t* k_tile8 = static_cast<int8_t*>(p.k_codes) + tile_idx * bs * d;
  __half* k_tile16 = static_cast<__half*>(p.k_codes) + tile_idx * bs * d;
  int8_t* v_tile8 = static_cast<int8_t*>(p.v_codes) + tile_idx * bs * d;
  uint8_t* v_tile4 = static_cast<uint8_t*>(p.v_codes) + tile_idx * bs * (d / 2);
  __half* v_tile16 = static_cast<__half*>(p.v_codes) + tile_idx * bs * d;

  if (n == 1) {
    // the stored scale / zero point matter only when appending into a partly filled tile
    float ks_old = 0.f, vs_old = 0.f;
    int vzp_old = 0;
    if (o0 > 0) {
      if constexpr (KT != PKV_FP16) ks_old = p.k_scale[tile_idx];
      if constexpr (VT != PKV_FP16) vs_old = p.v_scale[tile_idx];
      if constexpr (VT == PKV_INT4_ASYM) vzp_old = p.v_zp[tile_idx];
    }
    float kx[8], vx[8];
    halves_to_float(kraw, kx);
    halves_to_float(vraw, vx);
    if constexpr (KT == PKV_INT8_SYM) {
      append_sym(kx, vpl, k_tile8, p.k_scale + tile_idx, ks_old, o0, d, tbl, lane);
    } else if constexpr (KT == PKV_FP8_E4M3) {
      append_fp8(kx, vpl, reinterpret_cast<uint8_t*>(k_tile8), p.k_scale + tile_idx, ks_old, o0, d, tbl, lane);
    } else {
      append_fp16(kraw, vpl, k_tile16, o0, d, lane);
    }
    if constexpr (VT == PKV_INT8_SYM) {
      append_sym(vx, vpl, v_tile8, p.v_scale + tile_idx, vs_old, o0, d, tbl, lane);
    } else if constexpr (VT == PKV_FP8_E4M3) {
      append_fp8(vx, vpl, reinterpret_cast<uint8_t*>(v_tile8), p.v_scale + tile_idx, vs_old, o0, d, tbl, lane);
    } else if constexpr (VT == PKV_INT4_ASYM) {
      append_asym4(vx, vpl, v_tile4, p.v_scale + tile_idx, p.v_zp + tile_idx, vs_old, vzp_old, o0, d, tbl, lane);
    } else {
      append_fp16(vraw, vpl, v_tile16, o0, d, lane);
    }
    return;
  }

  // groups of several tokens
  GroupSrc src;
  src.row_stride = row_stride;
  src.n = n;
  src.d = d;
  src.base = p.k_new + (size_t)t * src.row_stride + (size_t)h * d;
  if constexpr (KT == PKV_INT8_SYM) {
    store_sym(src, k_tile8, p.k_scale + tile_idx, o0, tbl, lane);
  } else if constexpr (KT == PKV_FP8_E4M3) {
    store_fp8(src, reinterpret_cast<uint8_t*>(k_tile8), p.k_scale + tile_idx, o0, tbl, lane);
  } else {
    store_fp16(src, k_tile16, o0, lane);
  }
  src.base = p.v_new + (size_t)t * src.row_stride + (size_t)h * d;
  if constexpr (VT == PKV_INT8_SYM) {
    store_sym(src, v_tile8, p.v_scale + tile_idx, o0, tbl, lane);
  } else if constexpr (VT == PKV_FP8_E4M3) {
    store_fp8(src, reinterpret_cast<uint8_t*>(v_tile8), p.v_scale + tile_idx, o0, tbl, lane);
  } else if constexpr (VT == PKV_INT4_ASYM) {
    store_asym4(src, v_tile4, p.v_scale + tile_idx, p.v_zp + tile_idx, o0, tbl, lane);
  } else {
    store_fp16(src, v_tile16, o0, lane);
  }
}

}  // namespace
}  // namespace store_detail
}  // namespace pkv
