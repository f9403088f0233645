// store.cu -- quantize new K/V tokens and scatter them into pool blocks (sm_100a).
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
// __float2int_rn rounds half to even. Maxima and minima are order independent.
//
// Work split: one warp per (token, KV head). The warp of the first token of a group (the run of
// tokens bound for one block) does the whole group; the others return at once.
#include "common.cuh"
#include "internal.h"

namespace pkv {

namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kWarpsPerCta = 4;

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

// Values of the group for one head: element e of token i at src + i * row_stride + e.
struct GroupSrc {
  const __half* base;  // token 0 of the group, this head
  int64_t row_stride;  // elements between tokens (num_kv_heads * head_dim)
  int n;               // tokens in the group
  int d;               // head_dim
};

// ---- INT8 symmetric side of one (block, head) tile ----
__device__ void store_sym(const GroupSrc& src, int8_t* tile, float* scale_ptr, int o0, int lane) {
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
    bool fits = true;
    for (int e = lane; e < quads; e += 32) {
      const int i = (4 * e) / d, j = (4 * e) % d;
      float f[4];
      load4(src.base + i * src.row_stride + j, f);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (s_old == 0.0f) {
          fits = fits && (f[u] == 0.0f);
        } else {
          const int r = __float2int_rn(__fdiv_rn(f[u], s_old));
          fits = fits && (r <= 127 && r >= -127);
        }
      }
    }
    fits = __all_sync(kFull, fits);
    if (fits) {
      s = s_old;
    } else {
      // rebuild: old codes -> binary32 x_hat = code * s_old; scale from old and new together
      const int old_quads = o0 * d / 4;
      float m_old = 0.0f;
      for (int e = lane; e < old_quads; e += 32) {
        const uint32_t w = reinterpret_cast<const uint32_t*>(tile)[e];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = (int)(int8_t)((w >> (8 * u)) & 0xff);
          m_old = fmaxf(m_old, fabsf(__fmul_rn((float)q, s_old)));
        }
      }
      m_old = warp_max(m_old);
      s = __fdiv_rn(fmaxf(m_old, m_new), 127.0f);
      for (int e = lane; e < old_quads; e += 32) {
        uint32_t w = reinterpret_cast<const uint32_t*>(tile)[e];
        uint32_t out = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = (int)(int8_t)((w >> (8 * u)) & 0xff);
          const int r = quant_sym(__fmul_rn((float)q, s_old), s);
          out |= ((uint32_t)(r & 0xff)) << (8 * u);
        }
        reinterpret_cast<uint32_t*>(tile)[e] = out;
      }
    }
  }
  // new codes
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

// ---- INT4 asymmetric side: tile is [bs][d/2] bytes, byte j = code[2j] | code[2j+1] << 4 ----
__device__ void store_asym4(const GroupSrc& src, uint8_t* tile, float* scale_ptr, uint8_t* zp_ptr, int o0,
                            int lane) {
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
    bool fits = true;
    for (int e = lane; e < quads; e += 32) {
      const int i = (4 * e) / d, j = (4 * e) % d;
      float f[4];
      load4(src.base + i * src.row_stride + j, f);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (s_old == 0.0f) {
          fits = fits && (f[u] == 0.0f);
        } else {
          const int r = __float2int_rn(__fadd_rn(__fdiv_rn(f[u], s_old), (float)zp_old));
          fits = fits && (r >= 0 && r <= 15);
        }
      }
    }
    fits = __all_sync(kFull, fits);
    if (fits) {
      s = s_old;
      zp = zp_old;
    } else {
      // rebuild: x_hat = (code - zp_old) * s_old in binary32; range over old and new values
      const int old_bytes = o0 * d / 2;
      for (int e = lane; e < old_bytes; e += 32) {
        const uint8_t byte = tile[e];
        const float a = __fmul_rn((float)((int)(byte & 0xF) - zp_old), s_old);
        const float b = __fmul_rn((float)((int)(byte >> 4) - zp_old), s_old);
        lo = fminf(lo, fminf(a, b));
        hi = fmaxf(hi, fmaxf(a, b));
      }
      lo = warp_min(lo);
      hi = warp_max(hi);
      derive_asym(lo, hi, s, zp);
      for (int e = lane; e < old_bytes; e += 32) {
        const uint8_t byte = tile[e];
        const float a = __fmul_rn((float)((int)(byte & 0xF) - zp_old), s_old);
        const float b = __fmul_rn((float)((int)(byte >> 4) - zp_old), s_old);
        tile[e] = (uint8_t)(quant_asym(a, s, zp) | (quant_asym(b, s, zp) << 4));
      }
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
__device__ void store_fp16(const GroupSrc& src, __half* tile, int o0, int lane) {
  const int d = src.d, n = src.n;
  const int vecs = n * d / 8;  // 16-byte vectors
  __half* dst = tile + (size_t)o0 * d;
  for (int e = lane; e < vecs; e += 32) {
    const int i = (8 * e) / d, j = (8 * e) % d;
    reinterpret_cast<uint4*>(dst + (size_t)i * d)[j / 8] =
        *reinterpret_cast<const uint4*>(src.base + i * src.row_stride + j);
  }
}

// ---- single-token groups (the decode-step append): everything in registers ----
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

// INT8 symmetric side of a one-token group at offset o0. Returns false (nothing written) when the
// token does not fit the stored scale: the caller then takes the general path (rebuild).
__device__ bool fast_sym(const float x[8], int vpl, int8_t* tile, float* scale_ptr, float s_old, int o0, int d,
                         int lane) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < vpl) m = fmaxf(m, fabsf(x[i]));
  m = warp_max(m);
  float s;
  if (o0 == 0) {
    s = __fdiv_rn(m, 127.0f);
  } else {
    bool fits = true;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= vpl) continue;
      if (s_old == 0.0f) {
        fits = fits && (x[i] == 0.0f);
      } else {
        const int r = __float2int_rn(__fdiv_rn(x[i], s_old));
        fits = fits && (r <= 127 && r >= -127);
      }
    }
    if (!__all_sync(kFull, fits)) {
      if (vpl > 4) return false;  // head_dim 256: the general path rebuilds
      // rebuild in registers: the lane's codes of every old row in one batch of loads, then
      // x_hat = code * s_old in binary32, a scale covering old and new values, requantize
      uint32_t oldw[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        oldw[r] = 0;
        if (r < o0) {
          const int8_t* src = tile + (size_t)r * d + lane * vpl;
          oldw[r] = (vpl == 4) ? *reinterpret_cast<const uint32_t*>(src) : *reinterpret_cast<const uint16_t*>(src);
        }
      }
      float m_old = 0.0f;
#pragma unroll
      for (int r = 0; r < 32; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (r < o0 && i < vpl) {
            const int q = (int)(int8_t)((oldw[r] >> (8 * i)) & 0xff);
            m_old = fmaxf(m_old, fabsf(__fmul_rn((float)q, s_old)));
          }
      m_old = warp_max(m_old);
      s = __fdiv_rn(fmaxf(m_old, m), 127.0f);
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        if (r >= o0) continue;
        uint32_t out = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i < vpl) {
            const int q = (int)(int8_t)((oldw[r] >> (8 * i)) & 0xff);
            out |= ((uint32_t)(quant_sym(__fmul_rn((float)q, s_old), s) & 0xff)) << (8 * i);
          }
        int8_t* dst = tile + (size_t)r * d + lane * vpl;
        if (vpl == 4) *reinterpret_cast<uint32_t*>(dst) = out;
        else *reinterpret_cast<uint16_t*>(dst) = (uint16_t)out;
      }
      if (lane == 0) *scale_ptr = s;  // the new token's codes below use the rebuilt scale
    } else {
      s = s_old;
    }
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
  if (o0 == 0 && lane == 0) *scale_ptr = s;
  return true;
}

// INT4 asymmetric side of a one-token group; false when the token does not fit (rebuild needed).
__device__ bool fast_asym4(const float x[8], int vpl, uint8_t* tile, float* scale_ptr, uint8_t* zp_ptr, float s_old,
                           int zp_old, int o0, int d, int lane) {
  float s;
  int zp;
  if (o0 == 0) {
    float lo = 0.0f, hi = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= vpl) continue;
      lo = fminf(lo, x[i]);
      hi = fmaxf(hi, x[i]);
    }
    lo = warp_min(lo);
    hi = warp_max(hi);
    derive_asym(lo, hi, s, zp);
  } else {
    bool fits = true;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= vpl) continue;
      if (s_old == 0.0f) {
        fits = fits && (x[i] == 0.0f);
      } else {
        const int r = __float2int_rn(__fadd_rn(__fdiv_rn(x[i], s_old), (float)zp_old));
        fits = fits && (r >= 0 && r <= 15);
      }
    }
    if (!__all_sync(kFull, fits)) {
      if (vpl > 4) return false;  // head_dim 256: the general path rebuilds
      // rebuild in registers: old nibbles of every row in one batch of loads; range over
      // x_hat = (code - zp_old) * s_old (binary32) and the new values; requantize everything
      uint32_t oldw[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        oldw[r] = 0;
        if (r < o0) {
          const uint8_t* src = tile + (size_t)r * (d / 2) + lane * (vpl / 2);
          oldw[r] = (vpl == 4) ? *reinterpret_cast<const uint16_t*>(src) : *src;
        }
      }
      float lo = 0.0f, hi = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i >= vpl) continue;
        lo = fminf(lo, x[i]);
        hi = fmaxf(hi, x[i]);
      }
#pragma unroll
      for (int r = 0; r < 32; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (r < o0 && i < vpl) {
            const int q = (int)((oldw[r] >> (4 * i)) & 0xF);
            const float v = __fmul_rn((float)(q - zp_old), s_old);
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
          }
      lo = warp_min(lo);
      hi = warp_max(hi);
      derive_asym(lo, hi, s, zp);
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        if (r >= o0) continue;
        uint32_t out = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i < vpl) {
            const int q = (int)((oldw[r] >> (4 * i)) & 0xF);
            out |= (uint32_t)quant_asym(__fmul_rn((float)(q - zp_old), s_old), s, zp) << (4 * i);
          }
        uint8_t* dst = tile + (size_t)r * (d / 2) + lane * (vpl / 2);
        if (vpl == 4) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)out;
        else *dst = (uint8_t)out;
      }
      if (lane == 0) {
        *scale_ptr = s;
        *zp_ptr = (uint8_t)zp;
      }
    } else {
      s = s_old;
      zp = zp_old;
    }
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
  if (o0 == 0 && lane == 0) {
    *scale_ptr = s;
    *zp_ptr = (uint8_t)zp;
  }
  return true;
}

__device__ __forceinline__ void fast_fp16(const uint32_t raw[4], int vpl, __half* tile, int o0, int d, int lane) {
  __half* dst = tile + (size_t)o0 * d + lane * vpl;
  if (vpl == 8) *reinterpret_cast<uint4*>(dst) = make_uint4(raw[0], raw[1], raw[2], raw[3]);
  else if (vpl == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(raw[0], raw[1]);
  else *reinterpret_cast<uint32_t*>(dst) = raw[0];
}

__global__ void __launch_bounds__(32 * kWarpsPerCta) store_quantized_kernel(const StoreParams p) {
  // a kernel launched after this one with programmatic serialization (the decode) may begin its
  // set-up now; it waits for this grid to complete before it reads the pool
  asm volatile("griddepcontrol.launch_dependents;");
  const int t = blockIdx.x;
  const int h = blockIdx.y * kWarpsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
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

  bool k_done = false, v_done = false;
  if (n == 1) {
    // the stored scale / zero point matter only when appending into a partly filled tile
    float ks_old = 0.f, vs_old = 0.f;
    int vzp_old = 0;
    if (o0 > 0) {
      if (p.k_dtype == PKV_INT8_SYM) ks_old = p.k_scale[tile_idx];
      if (p.v_dtype != PKV_FP16) vs_old = p.v_scale[tile_idx];
      if (p.v_dtype == PKV_INT4_ASYM) vzp_old = p.v_zp[tile_idx];
    }
    float kx[8], vx[8];
    halves_to_float(kraw, kx);
    halves_to_float(vraw, vx);
    if (p.k_dtype == PKV_INT8_SYM) {
      k_done = fast_sym(kx, vpl, k_tile8, p.k_scale + tile_idx, ks_old, o0, d, lane);
    } else {
      fast_fp16(kraw, vpl, k_tile16, o0, d, lane);
      k_done = true;
    }
    if (p.v_dtype == PKV_INT8_SYM) {
      v_done = fast_sym(vx, vpl, v_tile8, p.v_scale + tile_idx, vs_old, o0, d, lane);
    } else if (p.v_dtype == PKV_INT4_ASYM) {
      v_done = fast_asym4(vx, vpl, v_tile4, p.v_scale + tile_idx, p.v_zp + tile_idx, vs_old, vzp_old, o0, d, lane);
    } else {
      fast_fp16(vraw, vpl, v_tile16, o0, d, lane);
      v_done = true;
    }
  }

  // general path: groups of several tokens, and appends that must rebuild the tile
  GroupSrc src;
  src.row_stride = row_stride;
  src.n = n;
  src.d = d;
  if (!k_done) {
    src.base = p.k_new + (size_t)t * src.row_stride + (size_t)h * d;
    if (p.k_dtype == PKV_INT8_SYM) {
      store_sym(src, k_tile8, p.k_scale + tile_idx, o0, lane);
    } else {
      store_fp16(src, k_tile16, o0, lane);
    }
  }
  if (!v_done) {
    src.base = p.v_new + (size_t)t * src.row_stride + (size_t)h * d;
    if (p.v_dtype == PKV_INT8_SYM) {
      store_sym(src, v_tile8, p.v_scale + tile_idx, o0, lane);
    } else if (p.v_dtype == PKV_INT4_ASYM) {
      store_asym4(src, v_tile4, p.v_scale + tile_idx, p.v_zp + tile_idx, o0, lane);
    } else {
      store_fp16(src, v_tile16, o0, lane);
    }
  }
}

}  // namespace

cudaError_t launch_store(const StoreParams& p, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  dim3 grid(p.T, (p.num_kv_heads + kWarpsPerCta - 1) / kWarpsPerCta);
  store_quantized_kernel<<<grid, 32 * kWarpsPerCta, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
