// decode_kernel.cuh -- decode-phase paged attention over the block-quantized KV cache (sm_100a):
// the kernel and its launch, instantiated per (K dtype, V dtype) in decode_<dtypes>.cu.
//
// What it computes (for sequence s, query head h, KV head g = h / group):
//   token t < L_s lives in physical block b = block_tables[s][t / bs] at offset t % bs
//     (yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section
//      "PagedAttention分页注意力机制与vLLM实现": block_table maps logical to physical blocks;
//      tbr8.org "如何通过 PagedAttention 与分块量化结合..." §2);
//   k_hat = code * k_scale[b][g], v_hat = (code - zp) * v_scale[b][g]
//     (yunthe.com, same page, section "KV Cache量化技术原理": x_hat = (Q(x) - zero_point) * scale);
//   out[s][h] = sum_t softmax_t(softmax_scale * q . k_hat_t) * v_hat_t.
// The dequantization happens in registers right after the codes leave shared memory; no
// dequantized copy of the cache exists anywhere (tbr8.org page, §5 item 2: dequantize inside the
// attention operator so no intermediate product occupies memory).
//
// How (B200 design, not taken from the pages): a persistent, stream-K kernel.
//   * A "unit" is (sequence s, head group hg): GT query heads sharing one KV head. Every unit
//     contributes ceil(L_s / bs) blocks to one global stream, ordered (s, hg, block). The grid
//     is a fixed set of worker warps (one CTA per SM, each warp independent); warp w owns
//     the contiguous stream range [w*T/W, (w+1)*T/W), so every warp gets the same number of
//     blocks whatever the length mix.
//   * Each warp streams its range through its own ring of NS shared-memory stages: lane 0
//     issues two bulk asynchronous copies per block (the contiguous bs x D K tile and V tile of
//     this head, 1-4 KiB each; 1-D copies for the CUDA-core engine, tiled copies with 128-byte
//     swizzle for the tensor-core engine) that complete on the stage's mbarrier, up to NS blocks
//     ahead and straight across unit boundaries; the warp reads tiles with 16-byte shared loads.
//   * Block ids are read 32 at a time ("windows", one id per lane) one window ahead; per-block
//     scales are fetched when the window's first copy is issued, NS blocks before use.
//   * q . k for INT8 K is exact integer arithmetic: q on a 22-bit fixed-point grid split into
//     three signed byte planes, three dp4a per 4 codes. V codes become exact floats through the
//     float bit layout (PRMT + paired FADD, no I2F); p . v accumulates with paired FFMA.
//   * Online softmax in the log2 domain (ex2.approx), rescaling only when the running max grows.
//   * A unit processed entirely by one warp is written out directly. A unit split across warps
//     gets one partial (max, sum, acc) per warp in the workspace; the last warp to finish (a
//     self-resetting atomicInc ticket after a release fence) merges them, lanes in parallel over
//     partials and dims. No CTA barrier, no second kernel.
//   * Optionally (FUSED) the same launch first does a step's copy-on-write copies and stores with
//     every warp, behind grid barriers (cooperative launch).
#pragma once

#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "copy_impl.cuh"
#include "store_impl.cuh"

namespace pkv {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr float kNegBig = -1.0e30f;  // finite "minus infinity" for running maxima

// One CTA per SM, with as many warps as the engine's registers allow (measured best): 16 for
// one INT8-K query head per warp, 12 for two, 8 for four on the CUDA cores or for FP16 K, 12 for
// the tensor-core engine (8 with head_dim 256). Warps of one CTA share the SM without the
// launch-order priority that the scheduler gives warps of earlier CTAs, which made warps of the
// last CTA on an SM run up to a third slower than those of the first and finish last. The
// copy rings take PKV_DECODE_SMEM_SM bytes of the SM's shared memory. (Both overridable at
// build time for tuning sweeps.)
#ifndef PKV_DECODE_SMEM_SM
#define PKV_DECODE_SMEM_SM 131072
#endif
#ifndef PKV_DECODE_WARPS_SM
#define PKV_DECODE_WARPS_SM 0  // 0: by engine, as above
#endif
// INT8 K with one or two query heads per KV head (MHA) on the tensor-core engine (1) or on the
// CUDA-core engine's dp4a planes (0, measured faster: 62.8 vs 81.9 us on the Llama-2-7B-shaped
// batch; the warp-level MMA pipe, not memory, limits the former at one useful column in eight).
#ifndef PKV_DECODE_MMA_MHA
#define PKV_DECODE_MMA_MHA 0
#endif
// INT8 K in the tensor-core engine: q.k on the integer tensor cores against three exact byte
// planes of q (1), or the codes turned into fp16 and multiplied with fp16 q (0, measured faster:
// 74.8 vs 78.4 us on the GQA shared-prefix batch; the integer MMAs triple the tensor-pipe work).
#ifndef PKV_DECODE_IMMA_QK
#define PKV_DECODE_IMMA_QK 0
#endif
// 1: the CUDA-core engine walks a 16-token-block pool two blocks per stream position (one 32-token
// tile, each half with its own scales), when the warps per CTA stay the same; 0: one block each.
// Measured on one B200: 239.7 vs 244.8 us on the lognormal-length INT8 K / INT4 V batch (fewer
// waits, walk steps and softmax passes per token). INT8 V with head_dim 128 keeps one block per
// position: its paired tile would leave room for 12 warps per CTA instead of 16.
#ifndef PKV_DECODE_PAIR
#define PKV_DECODE_PAIR 1
#endif
// INT8 K with one query head per KV head and 32-row tiles: q.k on the integer tensor cores, the
// three byte planes of q as three columns of one mma (1), or in dp4a planes on the CUDA cores (0);
// p.v stays on the CUDA cores either way. Measured on one B200: 157.8 vs 163.9 us on 8 sequences
// of 8K-32K tokens in 32-token blocks (two 16-row slices per tile: two independent mma chains),
// 223.3 vs 233.4 us on the lognormal-length batch in paired 16-token blocks (once q's planes cost
// about four instructions per value at a unit's start: warps whose range crosses many short
// sequences had lagged behind the rest). Tiles of 16 rows (one chain each) keep the dp4a planes.
#ifndef PKV_DECODE_HYB
#define PKV_DECODE_HYB 1
#endif
// Tuning switches (defaults: as described above): PKV_DECODE_HYB_ALL 1 takes the tensor-core q.k
// for 16-row tiles too; PKV_DECODE_KCOPY 0 / 1 forces the CUDA-core engine's K tile to a 1-D bulk
// copy / a swizzled tiled copy (-1: tiled exactly when q.k runs on the tensor cores).
#ifndef PKV_DECODE_HYB_ALL
#define PKV_DECODE_HYB_ALL 0
#endif
#ifndef PKV_DECODE_KCOPY
#define PKV_DECODE_KCOPY -1
#endif
// 1: a tile that lies wholly inside the sequence and whose blocks are valid skips the per-row
// masking of its scores (a warp-uniform branch); 0: every tile is masked row by row
#ifndef PKV_DECODE_FULLTILE
#define PKV_DECODE_FULLTILE 1
#endif
#ifndef PKV_DECODE_MAX_STAGES
#define PKV_DECODE_MAX_STAGES 6
#endif

template <int KT, int VT, int BS, int D, int GT>
struct Cfg {
  static constexpr int K_ROW = (KT == PKV_FP16) ? 2 * D : D;
  static constexpr int V_ROW = (VT == PKV_FP16) ? 2 * D : (VT == PKV_INT4_ASYM ? D / 2 : D);
  static constexpr int K_TILE = BS * K_ROW;
  static constexpr int V_TILE = BS * V_ROW;
  static constexpr int STAGE = K_TILE + V_TILE;
  // tensor-core engine: INT8 K (q.k on the integer tensor cores) with INT8 or INT4 V and E4M3 codes
  // (one conversion per pair) for every group size with D >= 128 (MHA INT8 K only with
  // PKV_DECODE_MMA_MHA); FP16/FP16 for groups of 4 or 8 query heads
  static constexpr bool FP8 = KT == PKV_FP8_E4M3 && VT == PKV_FP8_E4M3;
  static constexpr bool I8K = KT == PKV_INT8_SYM && (VT == PKV_INT8_SYM || VT == PKV_INT4_ASYM);
  static constexpr bool MMA = (D >= 128 && I8K && (GT >= 4 || PKV_DECODE_MMA_MHA)) ||
                              (GT >= 4 && KT == PKV_FP16 && VT == PKV_FP16) || (FP8 && D >= 128);
  // CUDA-core engine with INT8 K, one query head per KV head and 32-row tiles (a pool of 32-token
  // blocks, or the paired walk of 16-token blocks): q.k on the integer tensor cores (mma m16n8k32
  // with q's byte planes as columns), p.v on the CUDA cores
  static constexpr bool HYB =
      !MMA && KT == PKV_INT8_SYM && GT == 1 && K_ROW % 128 == 0 && (BS == 32 || PKV_DECODE_HYB_ALL) && PKV_DECODE_HYB;
  // the K tile arrives by a tiled copy with 128-byte swizzle (tensor-core fragments of it), or by a
  // 1-D bulk copy (rows as they are)
  static constexpr bool TILED_K =
      MMA || (KT == PKV_INT8_SYM && K_ROW % 128 == 0 &&
              (PKV_DECODE_KCOPY == 1 || (PKV_DECODE_KCOPY == -1 && HYB)));
  // the tensor-core engine's V tile arrives swizzled (tiled copy) when its rows are whole 128-byte
  // units; INT4 V, and V for the CUDA cores, by a 1-D bulk copy (unswizzled rows)
  static constexpr bool V_SWZ = MMA && V_ROW % 128 == 0 && VT != PKV_INT4_ASYM;
  static constexpr int WARPS_AUTO =
      MMA ? (D >= 256 ? 8 : 12) : (KT == PKV_FP16 ? 8 : (GT == 1 ? 16 : (GT == 2 ? 12 : 8)));
  static constexpr int WARPS_WANT = PKV_DECODE_WARPS_SM > 0 ? PKV_DECODE_WARPS_SM : WARPS_AUTO;
  static constexpr int WARPS_FIT = (200 * 1024) / (2 * STAGE);  // two stages per warp at least
  static constexpr int NW = WARPS_WANT < WARPS_FIT ? WARPS_WANT : WARPS_FIT;  // warps per CTA
  static constexpr int NS_RAW = PKV_DECODE_SMEM_SM / (NW * STAGE);             // stages per warp
  static constexpr int NS = NS_RAW < 2 ? 2 : (NS_RAW > PKV_DECODE_MAX_STAGES ? PKV_DECODE_MAX_STAGES : NS_RAW);
  static constexpr int THREADS = 32 * NW;
  static constexpr int SMEM_STAGES = NW * NS * STAGE;
  static constexpr int SMEM_BAR_FLAG = SMEM_STAGES + NW * NS * 8;  // one int: a grid barrier's outcome
  // The tensor-core engine's tiles arrive by tiled copies with 128-byte swizzle, whose shared
  // destinations must be 1024-byte aligned: the stages start on the next 1024-byte boundary.
  static constexpr int SMEM_ALIGN = TILED_K ? 1024 : 0;
  static constexpr int SMEM = SMEM_BAR_FLAG + 16 + SMEM_ALIGN;
  static constexpr int CTAS_PER_SM = 1;
  static_assert(D % 16 == 0 && D / 16 <= 32, "head_dim");
  static_assert(K_TILE % 16 == 0 && V_TILE % 16 == 0 && STAGE % 16 == 0, "bulk copy granularity");
  static_assert(!TILED_K || (K_ROW % 128 == 0 && K_TILE % 1024 == 0 && STAGE % 1024 == 0 &&
                          (!V_SWZ || V_TILE % 1024 == 0)),
                "swizzled tiles: 128-byte row units, 1024-byte aligned tiles");
  static_assert(NW >= 1 && SMEM <= 227 * 1024, "shared memory per CTA");
};

// 16 fp16 values of one token row (8 at pa, 8 at pb) -> 8 float2 (pa's dims first)
__device__ __forceinline__ void load_h16(const uint8_t* pa, const uint8_t* pb, float2 f[8]) {
  const uint4 w0 = *reinterpret_cast<const uint4*>(pa);
  const uint4 w1 = *reinterpret_cast<const uint4*>(pb);
  const uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
}

// 16 consecutive V values of one token row (lane chunk) -> 8 float2 of (code - zp);
// neg_bias = -(2^23 + zp) in both lanes (INT4 only)
template <int VT>
__device__ __forceinline__ void load_v16(const uint8_t* p, float2 neg_bias, float2 f[8]) {
  if constexpr (VT == PKV_INT8_SYM) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    s8x4_to_f32x2(w.x, f[0], f[1]);
    s8x4_to_f32x2(w.y, f[2], f[3]);
    s8x4_to_f32x2(w.z, f[4], f[5]);
    s8x4_to_f32x2(w.w, f[6], f[7]);
  } else if constexpr (VT == PKV_INT4_ASYM) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    u4x8_to_f32x2(w.x, neg_bias, f);
    u4x8_to_f32x2(w.y, neg_bias, f + 4);
  } else {
    load_h16(p, p + 16, f);
  }
}

// 8 unsigned 4-bit codes (nibble k = dim k) -> 4 float2 of 0.5 + code / 256, dims in order: the
// nibble becomes mantissa bits 16..19 under the exponent of 0.5 (bit pattern 0x3F0c0000), exact
// and linear in the code, so a p.v over these values needs no per-code subtraction; the offset
// 0.5 and the zero point are removed from the sums instead.
__device__ __forceinline__ void u4x8_to_half_offset_f32x2(uint32_t w, float2 f[4]) {
  const uint32_t even = w & 0x0F0F0F0Fu;        // nibbles 0,2,4,6 in bytes 0..3
  const uint32_t odd = (w >> 4) & 0x0F0F0F0Fu;  // nibbles 1,3,5,7
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // result bytes: [0x00, 0x00, nibble, 0x3F] taken from {x, 0x3F000000}
    const uint32_t sel = 0x7054u | ((uint32_t)i << 8);
    f[i] = make_float2(__uint_as_float(__byte_perm(even, 0x3F000000u, sel)),
                       __uint_as_float(__byte_perm(odd, 0x3F000000u, sel)));
  }
}

__device__ __forceinline__ int clamp_len(const DecodeParams& p, int L, int bs) {
  const int cap = min(p.max_context_len, p.max_blocks_per_seq * bs);
  return max(0, min(L, cap));
}

// The worker warp whose stream range contains position g (start_w = floor(w*T/W) <= g).
__device__ __forceinline__ int owner_of(long long g, long long T, int W) {
  return (int)(((g + 1) * (long long)W - 1) / T);
}

// A window: up to 32 consecutive blocks of one unit (warp-uniform description; lane k holds
// block j0 + k in the per-lane registers of the window).
struct Win {
  int s, hg, j0, n;     // walk position of the sequence, head group, first block, blocks in the window (0 = none)
  int sa;               // the sequence itself (its index in q, out, tables): seq_order[s], or s
  int g;                // KV head of the head group
  int L, nblk;          // clamped length of the sequence and its private block count (after sb)
  int sb;               // its leading blocks attended by the shared-prefix pass (0 without one)
  int r0;               // position of block j0 relative to the warp's first position
  long long seq_p0;     // stream position of the sequence's first block (head group 0)
};

// A window lane's stream position: one physical block, or two consecutive ones of the unit (the
// paired walk: a 32-token tile of two 16-token blocks).
// Before the scales are fetched, b holds the ids as read from the table; after, the physical block
// to copy (0 stands in for an invalid id; -1 where a paired position holds no second block), the
// K scale in the log2 domain, the V scale, and the V zero point (0 without one), or -1 where the
// block is not valid (its tokens are masked).
template <int VB>
struct WinLanes {
  int b[VB];
  bool meta;  // scales fetched (warp-uniform)
  float ks[VB], vs[VB], zv[VB];
};

// ============================================================================================
// Per-block arithmetic. Both engines see one (block, KV head) tile in shared memory at a time
// and keep the running softmax state of GT query heads for the current unit.
// ============================================================================================

// Byte offset of (row r, byte x) in a tile of R-byte rows stored by a tiled copy with 128-byte
// swizzle: rows are cut into 128-byte units (unit u = r * R/128 + x/128), and within unit u the
// 16-byte chunk j sits at chunk j ^ (u mod 8). Rows of 128 or 256 bytes otherwise all start on
// bank 0, and the fragment loads below (the same column of several rows at once) would conflict.
template <int R>
__device__ __forceinline__ int swz(int r, int x) {
  const int u = r * (R / 128) + (x >> 7);
  return (u << 7) | ((((x >> 4) & 7) ^ (u & 7)) << 4) | (x & 15);
}

// ---- tensor-core helpers (mma.sync m16n8k16, fp16 operands, fp32 accumulators) ----
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// integer tensor cores: m16n8k32, signed 8-bit operands, int32 accumulators
__device__ __forceinline__ void imma_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                           uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2_pack(float lo, float hi) {
  const __half2 r = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&r);
}
// fp16 1024 + 128 in both halves: a byte b placed under exponent 0x64 reads 1024 + b, and
// (c ^ 0x80) = c + 128 for a signed code c, so subtracting this leaves c exactly
constexpr uint32_t kH2Bias = 0x64806480u;
// two E4M3 codes (low byte first) -> two exact fp16 values (low half first)
__device__ __forceinline__ uint32_t fp8x2_to_h2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// CUDA-core engine (1, 2 or 4 query heads per KV head): a lane owns 16 consecutive dims of
// bs/(32*16/D) token rows; q.k in exact integer dp4a planes (INT8 K) or paired FFMA (FP16 K);
// p.v with paired FFMA on codes made exact floats through the float bit layout.
//
// With INT8 K and one query head (C::HYB), q.k runs on the integer tensor cores instead: per
// 16-row slice one mma m16n8k32 per 32 dims, A = the slice's K codes (rows = tokens) straight from
// the swizzled tile, B = q on its 22-bit fixed-point grid, whose three signed byte planes fill
// columns 0, 1, 2 (and again 4, 5, 6; columns 3 and 7 are zero). Lane (gq, tq) then holds planes
// 0 and 1 of tokens gq and gq + 8 when tq is even, plane 2 in its odd neighbour: one exchange
// completes a score, and the scores move to the p.v layout by index shuffles.
template <int KT, int VT, int BS, int D, int GT>
struct CoreEngine {
  using C = Cfg<KT, VT, BS, D, GT>;
  static constexpr int CH = D / 16, TG = 32 / CH, TPL = BS / TG;
  static_assert(BS % TG == 0, "block_size must cover the token rows of a warp pass");
  static constexpr bool HYB = C::HYB;
  static constexpr int KQ = D / 32;  // k32-steps of one slice's q.k (HYB)
  static_assert(!HYB || (GT == 1 && BS % 16 == 0 && 16 % TG == 0), "tensor-core q.k");
  // A lane owns 16 dims: [a, a + 8) and [b, b + 8). With byte codes they are contiguous
  // (a = 16c, b = a + 8: a lane's 16 codes are one 16-byte load). With fp16 rows (2D bytes),
  // 16 contiguous dims would put lanes c and c + 4 of a load on the same banks; a = 8c and
  // b = D/2 + 8c instead make the 8 lanes of each load read 128 contiguous bytes.
  static constexpr bool SPLIT = (KT == PKV_FP16);
  int c, tg;
  __device__ __forceinline__ int dim_a() const { return SPLIT ? 8 * c : 16 * c; }
  __device__ __forceinline__ int dim_b() const { return SPLIT ? D / 2 + 8 * c : 16 * c + 8; }
  float2 qf[GT][8];
  uint32_t qplane[GT][HYB ? 1 : 3][4];
  uint32_t qbf[HYB ? KQ : 1][2];  // HYB: B fragments, k32-step kk, (b0, b1)
  int lid;
  float qinv[GT];
  float m_run[GT], l_run[GT];
  float2 acc[GT][8];
  // INT4 V (OFS): the p.v sums run over 0.5 + code/256 (no per-code subtraction); after every tile
  // the offset part (0.5 x the tile's sum of p * v_scale) is taken out of acc, so acc holds
  // sum(p * vs * code) / 256, and zsum collects sum(p * vs * zp); finish() forms 256 acc - zsum.
  // (Measured on one B200 with the dp4a q.k: 233.5 vs 237.7 us on the lognormal-length INT8 K /
  // INT4 V batch; with q.k on the tensor cores, whose tiles wait on the mma chain, it measured
  // slower, 164.6 vs 157.8 us on the 32-token-block batch, so there the per-code subtraction
  // stays. The paired 16-token INT4 pools now take the tensor-core q.k, so the offset form serves
  // the remaining dp4a tiles: INT4 V with 2 or 4 query heads per warp, or where pairing is off.)
  static constexpr bool OFS = VT == PKV_INT4_ASYM && !HYB;
  float zsum[OFS ? GT : 1];

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      m_run[hh] = kNegBig;
      l_run[hh] = 0.f;
      if constexpr (OFS) zsum[hh] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[hh][j] = make_float2(0.f, 0.f);
    }
  }

  __device__ __forceinline__ void begin(const DecodeParams& p, int s, int hg, int lane) {
    c = lane % CH;
    tg = lane / CH;
    lid = lane;
    if constexpr (HYB) begin_hyb(p, s, hg, lane);
    else begin_core(p, s, hg);
  }

  __device__ __forceinline__ void begin_core(const DecodeParams& p, int s, int hg) {
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      const __half* qp = p.q + ((size_t)s * p.num_q_heads + (size_t)hg * GT + hh) * D;
      const uint4 w0 = *reinterpret_cast<const uint4*>(qp + dim_a());
      const uint4 w1 = *reinterpret_cast<const uint4*>(qp + dim_b());
      const uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) qf[hh][i] = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
    }
    reset();
    // INT8 K: q . k is computed exactly in integers. Each head's q is put on a fixed-point grid
    // of 2^-shift (22 bits below its largest magnitude; fp16 q loses nothing above 2^-22 of its
    // max) and split into three signed byte planes, q_fixed = 2^16 b2 + 2^8 b1 + b0, so a
    // 4-code word costs three dp4a with int32 accumulation and no code is converted to float.
    if constexpr (KT == PKV_INT8_SYM) {
#pragma unroll
      for (int hh = 0; hh < GT; ++hh) {
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fmaxf(fabsf(qf[hh][i].x), fabsf(qf[hh][i].y)));
#pragma unroll
        for (int off = 1; off < CH; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
        int e = 0;
        (void)frexpf(amax, &e);                    // amax < 2^e
        const int shift = amax > 0.f ? 22 - e : 0;  // |q| * 2^shift < 2^22
        const float up = __int_as_float((127 + shift) << 23);
        qinv[hh] = __int_as_float((127 - shift) << 23);
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          uint32_t p0 = 0, p1 = 0, p2 = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 pr = qf[hh][(4 * wd + k) / 2];
            const int qi = __float2int_rn((((4 * wd + k) & 1) ? pr.y : pr.x) * up);
            const int b0 = ((qi + 128) & 0xFF) - 128;
            const int r1 = (qi - b0) >> 8;
            const int b1 = ((r1 + 128) & 0xFF) - 128;
            const int b2 = (r1 - b1) >> 8;
            p0 |= (uint32_t)(b0 & 0xFF) << (8 * k);
            p1 |= (uint32_t)(b1 & 0xFF) << (8 * k);
            p2 |= (uint32_t)(b2 & 0xFF) << (8 * k);
          }
          qplane[hh][0][wd] = p0;
          qplane[hh][1][wd] = p1;
          qplane[hh][2][wd] = p2;
        }
      }
    } else {
#pragma unroll
      for (int hh = 0; hh < GT; ++hh) qinv[hh] = 1.f;
    }
  }

  // q on the fixed-point grid of the dp4a planes (same shift, same planes), as B fragments: lane
  // (gq, tq) gives column gq, i.e. byte plane gq % 4 (3: zero), over dims tq * D/4 + [0, D/4);
  // k32-step kk holds dims tq * D/4 + 8kk + [0, 4) in b0 and + [4, 8) in b1, the dims of the A
  // fragments read in block().
  __device__ __forceinline__ void begin_hyb(const DecodeParams& p, int s, int hg, int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    const uint4* qp = reinterpret_cast<const uint4*>(p.q + ((size_t)s * p.num_q_heads + hg) * D + tq * (D / 4));
    float x[D / 4];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const uint4 w = qp[i];
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[k]));
        x[8 * i + 2 * k] = f.x;
        x[8 * i + 2 * k + 1] = f.y;
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < D / 4; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    int e = 0;
    (void)frexpf(amax, &e);                    // amax < 2^e
    const int shift = amax > 0.f ? 22 - e : 0;  // |q| * 2^shift < 2^22
    const float up = __int_as_float((127 + shift) << 23);
    qinv[0] = __int_as_float((127 - shift) << 23);
    // byte of plane pl of qi (qi = b0 + 2^8 b1 + 2^16 b2, signed bytes): ((qi + off) >> 8pl) & 0xFF
    // with off = 0, 2^7, 2^7 + 2^15; qi itself from the binary32 sum x * up + 1.5 * 2^23 (exact
    // product, one round-to-nearest-even into the low mantissa bits)
    const int pl = gq & 3;
    const int off = (pl == 0 ? 0 : (pl == 1 ? 128 : 32896)) - 0x4B400000;
    const int sh = 8 * (pl & 3);
    const uint32_t keep = pl == 3 ? 0u : 0xFFFFFFFFu;
#pragma unroll
    for (int kk = 0; kk < KQ; ++kk) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t b[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float r = __fmaf_rn(x[8 * kk + 4 * h + k], up, 12582912.0f);
          b[k] = (uint32_t)((__float_as_int(r) + off) >> sh);
        }
        const uint32_t lo = __byte_perm(b[0], b[1], 0x0040), hi = __byte_perm(b[2], b[3], 0x0040);
        qbf[kk][h] = __byte_perm(lo, hi, 0x5410) & keep;
      }
    }
    reset();
  }

  // One tile of BS token rows made of BS / HB physical blocks of HB rows (1 or 2): per physical
  // block ks = K scale in the log2 domain (INT8 K), vs = V scale, nzb = -(2^23+zp), valid. A row's
  // block is known at compile time: a lane's rows are tg + TG*i and HB is a multiple of TG.
  template <int HB>
  __device__ __forceinline__ void block(const uint8_t* kt, const uint8_t* vt, const float (&ks)[2], const float (&vs)[2],
                                        const float (&nzb)[2], const bool (&valid)[2], int tok0, int L,
                                        float scale_log2) {
    static_assert(BS % HB == 0 && BS / HB <= 2 && HB % TG == 0, "physical blocks of a tile");
    float z[TPL][GT];
    if constexpr (HYB) {
      scores_hyb(kt, z);
    } else {
      scores_core(kt, z);
    }
    block_softmax_pv<HB>(vt, z, ks, vs, nzb, valid, tok0, L, scale_log2);
  }

  // byte offset of (row r, byte x) in the K tile as its copy left it
  __device__ __forceinline__ static int koff(int r, int x) { return C::TILED_K ? swz<C::K_ROW>(r, x) : r * C::K_ROW + x; }

  // q.k of the tile's rows tg + TG*i on the integer tensor cores (C::HYB; see above)
  __device__ __forceinline__ void scores_hyb(const uint8_t* kt, float (&z)[TPL][GT]) const {
    constexpr int NSL = BS / 16;
    const int gq = lid >> 2, tq = lid & 3;
    float sA[NSL], sB[NSL];  // tokens 16h2 + gq and 16h2 + gq + 8 (complete where tq is even)
#pragma unroll
    for (int h2 = 0; h2 < NSL; ++h2) {
      int cc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < D / 64; ++i) {  // 16 codes = 2 k32-steps per 16-byte load
        const int x = tq * (D / 4) + 16 * i;
        const uint4 r0 = *reinterpret_cast<const uint4*>(kt + koff(16 * h2 + gq, x));
        const uint4 r1 = *reinterpret_cast<const uint4*>(kt + koff(16 * h2 + gq + 8, x));
        imma_16832(cc, r0.x, r1.x, r0.y, r1.y, qbf[2 * i][0], qbf[2 * i][1]);
        imma_16832(cc, r0.z, r1.z, r0.w, r1.w, qbf[2 * i + 1][0], qbf[2 * i + 1][1]);
      }
      // |plane sums| < 2^21: planes 0 and 1 combine exactly in int32, plane 2 in fp32
      const int u0 = __shfl_xor_sync(kFull, cc[0], 1);
      const int u2 = __shfl_xor_sync(kFull, cc[2], 1);
      sA[h2] = __fmaf_rn((float)u0, 65536.f, (float)(cc[1] * 256 + cc[0]));
      sB[h2] = __fmaf_rn((float)u2, 65536.f, (float)(cc[3] * 256 + cc[2]));
    }
    // row tg + TG*i: slice (TG*i)/16, token (tg + TG*i) % 16 of it, held by lane 4 * (token % 8)
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int h2 = (TG * i) / 16;
      const bool upper = (TG * i) % 16 >= 8;
      z[i][0] = __shfl_sync(kFull, upper ? sB[h2] : sA[h2], 4 * ((tg + TG * i) % 8));
    }
  }

  // q.k of the tile's rows tg + TG*i on the CUDA cores: a lane's 16 dims, then summed over the
  // CH lanes of a row
  __device__ __forceinline__ void scores_core(const uint8_t* kt, float (&z)[TPL][GT]) const {
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int row = tg + TG * i;
      if constexpr (KT == PKV_INT8_SYM) {
        const uint4 wv = *reinterpret_cast<const uint4*>(kt + koff(row, c * (C::K_ROW / CH)));
        const int kw[4] = {(int)wv.x, (int)wv.y, (int)wv.z, (int)wv.w};
#pragma unroll
        for (int hh = 0; hh < GT; ++hh) {
          int acc_p[3];
#pragma unroll
          for (int pl = 0; pl < 3; ++pl) {
            int a = __dp4a((int)qplane[hh][pl][0], kw[0], 0);
            a = __dp4a((int)qplane[hh][pl][1], kw[1], a);
            a = __dp4a((int)qplane[hh][pl][2], kw[2], a);
            acc_p[pl] = __dp4a((int)qplane[hh][pl][3], kw[3], a);
          }
          // |acc_p| < 2^18: the low two planes combine exactly in int32, the top one in fp32
          z[i][hh] = __fmaf_rn((float)acc_p[2], 65536.f, (float)(acc_p[1] * 256 + acc_p[0]));
        }
      } else {
        float2 kf[8];
        load_h16(kt + row * C::K_ROW + 2 * dim_a(), kt + row * C::K_ROW + 2 * dim_b(), kf);
#pragma unroll
        for (int hh = 0; hh < GT; ++hh) {
          float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < 8; j += 2) {
            a0 = __ffma2_rn(qf[hh][j], kf[j], a0);
            a1 = __ffma2_rn(qf[hh][j + 1], kf[j + 1], a1);
          }
          z[i][hh] = (a0.x + a0.y) + (a1.x + a1.y);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < TPL; ++i)
#pragma unroll
      for (int hh = 0; hh < GT; ++hh)
#pragma unroll
        for (int off = 1; off < CH; off <<= 1) z[i][hh] += __shfl_xor_sync(kFull, z[i][hh], off);
  }

  // online softmax of the tile's scores z (unscaled) and p.v into the running state
  template <int HB>
  __device__ __forceinline__ void block_softmax_pv(const uint8_t* vt, float (&z)[TPL][GT], const float (&ks)[2],
                                                   const float (&vs)[2], const float (&nzb)[2], const bool (&valid)[2],
                                                   int tok0, int L, float scale_log2) {
    float pv[TPL][GT];
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      const float zs0 = (KT == PKV_FP16) ? scale_log2 : ks[0] * qinv[hh];
      const float zs1 = (KT == PKV_FP16) ? scale_log2 : ks[1] * qinv[hh];
      float mloc = -INFINITY;
      // the tile's blocks valid and its last row inside the sequence: no row is masked
      const bool full = PKV_DECODE_FULLTILE && valid[0] && valid[BS / HB - 1] && tok0 + BS <= L;
      if (full) {
#pragma unroll
        for (int i = 0; i < TPL; ++i) {
          const float zz = z[i][hh] * (((TG * i) / HB) ? zs1 : zs0);
          z[i][hh] = zz;
          mloc = fmaxf(mloc, zz);
        }
      } else {
#pragma unroll
        for (int i = 0; i < TPL; ++i) {
          const int t = tok0 + tg + TG * i;
          const int hb = (TG * i) / HB;  // the row's physical block (compile time)
          float zz = z[i][hh] * (hb ? zs1 : zs0);
          zz = (valid[hb] && t < L) ? zz : -INFINITY;
          z[i][hh] = zz;
          mloc = fmaxf(mloc, zz);
        }
      }
#pragma unroll
      for (int off = CH; off < 32; off <<= 1) mloc = fmaxf(mloc, __shfl_xor_sync(kFull, mloc, off));
      // the running max is warp-uniform; rescale only when it grows (rare after the first blocks)
      if (mloc > m_run[hh]) {
        const float alpha = ex2(m_run[hh] - mloc);
        m_run[hh] = mloc;
        l_run[hh] *= alpha;
        if constexpr (OFS) zsum[hh] *= alpha;
        const float2 alpha2 = make_float2(alpha, alpha);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[hh][j] = __fmul2_rn(acc[hh][j], alpha2);
      }
      const float m_new = m_run[hh];
      float lsum = 0.f;
#pragma unroll
      for (int i = 0; i < TPL; ++i) {
        const float pr = ex2(z[i][hh] - m_new);
        lsum += pr;
        pv[i][hh] = (VT == PKV_FP16) ? pr : pr * vs[(TG * i) / HB];
      }
      l_run[hh] += lsum;
    }
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int row = tg + TG * i;
      const int hb = (TG * i) / HB;
      const float2 neg_zp_bias = make_float2(nzb[hb], nzb[hb]);
      float2 vf[8];
      if constexpr (VT == PKV_FP16) {
        load_h16(vt + row * C::V_ROW + 2 * dim_a(), vt + row * C::V_ROW + 2 * dim_b(), vf);
      } else if constexpr (OFS) {
        const uint2 w = *reinterpret_cast<const uint2*>(vt + row * C::V_ROW + c * (C::V_ROW / CH));
        u4x8_to_half_offset_f32x2(w.x, vf);
        u4x8_to_half_offset_f32x2(w.y, vf + 4);
      } else {
        load_v16<VT>(vt + row * C::V_ROW + c * (C::V_ROW / CH), neg_zp_bias, vf);
      }
#pragma unroll
      for (int hh = 0; hh < GT; ++hh) {
        const float2 pv2 = make_float2(pv[i][hh], pv[i][hh]);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[hh][j] = __ffma2_rn(pv2, vf[j], acc[hh][j]);
      }
    }
    if constexpr (OFS) {
      // take the tile's offset part out of acc now (it stays about the size of the result, which
      // bounds the rounding of later sums), and collect the zero-point part
#pragma unroll
      for (int hh = 0; hh < GT; ++hh) {
        float s1[2] = {0.f, 0.f};  // sum of p * vs over this lane's rows of each physical block
#pragma unroll
        for (int i = 0; i < TPL; ++i) s1[(TG * i) / HB] += pv[i][hh];
        const float half_s = -0.5f * (s1[0] + s1[1]);
        const float2 d = make_float2(half_s, half_s);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[hh][j] = __fadd2_rn(acc[hh][j], d);
        // zero points: -(nzb + 2^23) = zp
        zsum[hh] = __fmaf_rn(-(nzb[0] + kMagic), s1[0], zsum[hh]);
        if constexpr (BS / HB > 1) zsum[hh] = __fmaf_rn(-(nzb[1] + kMagic), s1[1], zsum[hh]);
      }
    }
  }

  // end of a segment: sum the lanes' partial states over the token-row groups
  __device__ __forceinline__ void finish() {
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      if constexpr (OFS) {  // sum(p * vs * (code - zp)) = 256 acc - zsum
        const float2 k256 = make_float2(256.f, 256.f), nz = make_float2(-zsum[hh], -zsum[hh]);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[hh][j] = __ffma2_rn(acc[hh][j], k256, nz);
      }
#pragma unroll
      for (int off = CH; off < 32; off <<= 1) l_run[hh] += __shfl_xor_sync(kFull, l_run[hh], off);
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int off = CH; off < 32; off <<= 1) {
          acc[hh][j].x += __shfl_xor_sync(kFull, acc[hh][j].x, off);
          acc[hh][j].y += __shfl_xor_sync(kFull, acc[hh][j].y, off);
        }
    }
  }

  __device__ __forceinline__ void write_out(const DecodeParams& p, int s, int hg) {
    if (tg != 0) return;
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      const float inv = l_run[hh] > 0.f ? 1.f / l_run[hh] : 0.f;
      __half* ob = p.out + ((size_t)s * p.num_q_heads + (size_t)hg * GT + hh) * D;
      __half2* oa = reinterpret_cast<__half2*>(ob + dim_a());
      __half2* obb = reinterpret_cast<__half2*>(ob + dim_b());
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        oa[j] = __floats2half2_rn(acc[hh][j].x * inv, acc[hh][j].y * inv);
        obb[j] = __floats2half2_rn(acc[hh][4 + j].x * inv, acc[hh][4 + j].y * inv);
      }
    }
  }

  __device__ __forceinline__ void write_partial(const DecodeParams& p, long long slot, int lane) {
    if (tg == 0) {
#pragma unroll
      for (int hh = 0; hh < GT; ++hh) {
        float* base = p.ws_acc + ((size_t)slot * GT + hh) * D;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          reinterpret_cast<float4*>(base + (j < 2 ? dim_a() + 4 * j : dim_b() + 4 * (j - 2)))[0] =
              make_float4(acc[hh][2 * j].x, acc[hh][2 * j].y, acc[hh][2 * j + 1].x, acc[hh][2 * j + 1].y);
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int hh = 0; hh < GT; ++hh) {
        p.ws_ml[((size_t)slot * GT + hh) * 2 + 0] = m_run[hh];
        p.ws_ml[((size_t)slot * GT + hh) * 2 + 1] = l_run[hh];
      }
    }
  }
};

// Tensor-core engine (4 or 8 query heads per KV head): per 16-token slice of a block,
//   S = K . q^T  as mma m16n8k16 with M = 16 tokens, N = 8 heads, K = 16 dims per step, and
//   O^T += V^T . P^T  with M = 16 dims per tile, N = 8 heads, K = 16 tokens,
// the int8 codes turned into exact fp16 integers in registers on the way into the A operands.
// Dim order inside an mma step is a fixed permutation, the same for both operands of a product.
// Lane (g = lane/4, c = lane%4): q.k reads token rows g, g+8 at dims [c*D/4, (c+1)*D/4); p.v reads
// token rows 2c, 2c+1, 2c+8, 2c+9 at dims [g*D/8, (g+1)*D/8) and owns the outputs of heads 2c,
// 2c+1 at those dims. P goes through movmatrix.trans from accumulator to operand layout, split
// into an fp16 high and low part so p.v keeps about 22 bits of each weight.
template <int KT, int VT, int BS, int D, int GT>
struct MmaEngine {
  using C = Cfg<KT, VT, BS, D, GT>;
  static constexpr int KS = D / 16;  // q.k steps and p.v dim tiles
  static_assert(BS % 16 == 0, "16-token slices");
  // INT8 K: q.k on the integer tensor cores, the codes as they sit in shared memory against q on a
  // 22-bit fixed-point grid per head split into three signed byte planes (exact, as in the
  // CUDA-core engine); otherwise K is turned into fp16 and multiplied with fp16 q.
  static constexpr bool IMMA = KT == PKV_INT8_SYM && PKV_DECODE_IMMA_QK;
  int g, c;
  uint32_t qb[IMMA ? 1 : KS][2];
  uint32_t qp8[IMMA ? 3 : 1][IMMA ? KS / 2 : 1][2];  // planes, k32-steps, (b0, b1)
  float qz[2];                                       // 2^-shift of heads 2c, 2c+1
  float acc[KS][4];
  float m_run[2], l_run[2];

  __device__ __forceinline__ void reset() {
    m_run[0] = m_run[1] = kNegBig;
    l_run[0] = l_run[1] = 0.f;
#pragma unroll
    for (int j = 0; j < KS; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  }

  __device__ __forceinline__ void begin(const DecodeParams& p, int s, int hg, int lane) {
    g = lane >> 2;
    c = lane & 3;
    if constexpr (IMMA) {
      // head g of the group, dims [c*D/4, (c+1)*D/4); k32-step kk holds dims c*D/4 + 8kk + [0,4) (b0)
      // and + [4,8) (b1), the same dims as the A fragments of the K rows below
      float x[D / 4];
      if (g < GT) {
        const uint4* qp = reinterpret_cast<const uint4*>(p.q + ((size_t)s * p.num_q_heads + (size_t)hg * GT + g) * D +
                                                         c * (D / 4));
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
          const uint4 wv = qp[i];
          const uint32_t u[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[k]));
            x[8 * i + 2 * k] = f.x;
            x[8 * i + 2 * k + 1] = f.y;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < D / 4; ++i) x[i] = 0.f;
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < D / 4; ++i) amax = fmaxf(amax, fabsf(x[i]));
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
      int ex = 0;
      (void)frexpf(amax, &ex);                    // amax < 2^ex
      const int shift = amax > 0.f ? 22 - ex : 0;  // |q| * 2^shift < 2^22
      const float up = __int_as_float((127 + shift) << 23);
      const float qinv = __int_as_float((127 - shift) << 23);
      qz[0] = __shfl_sync(kFull, qinv, 8 * c);      // head 2c lives on lanes 4 (2c) + ..
      qz[1] = __shfl_sync(kFull, qinv, 8 * c + 4);  // head 2c + 1
#pragma unroll
      for (int kk = 0; kk < KS / 2; ++kk) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t p0 = 0, p1 = 0, p2 = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int qi = __float2int_rn(x[8 * kk + 4 * h + k] * up);
            const int b0 = ((qi + 128) & 0xFF) - 128;
            const int r1 = (qi - b0) >> 8;
            const int b1 = ((r1 + 128) & 0xFF) - 128;
            const int b2 = (r1 - b1) >> 8;
            p0 |= (uint32_t)(b0 & 0xFF) << (8 * k);
            p1 |= (uint32_t)(b1 & 0xFF) << (8 * k);
            p2 |= (uint32_t)(b2 & 0xFF) << (8 * k);
          }
          qp8[0][kk][h] = p0;
          qp8[1][kk][h] = p1;
          qp8[2][kk][h] = p2;
        }
      }
    } else {
      load_q16(p, s, hg);
    }
    reset();
  }

  // q^T fragments (fp16 K): head g of the group, dims [c*D/4, (c+1)*D/4) as 2*KS half2 words
  __device__ __forceinline__ void load_q16(const DecodeParams& p, int s, int hg) {
#pragma unroll
    for (int j = 0; j < KS; ++j) qb[j][0] = qb[j][1] = 0u;
    if (g < GT) {
      const uint4* qp = reinterpret_cast<const uint4*>(p.q + ((size_t)s * p.num_q_heads + (size_t)hg * GT + g) * D +
                                                       c * (D / 4));
#pragma unroll
      for (int i = 0; i < KS / 2; ++i) {
        const uint4 w = qp[i];
        qb[2 * i][0] = w.x;
        qb[2 * i][1] = w.y;
        qb[2 * i + 1][0] = w.z;
        qb[2 * i + 1][1] = w.w;
      }
    }
  }

  // one (block, KV head) tile (HB == BS: the tensor-core engine takes one physical block per tile)
  template <int HB>
  __device__ __forceinline__ void block(const uint8_t* kt, const uint8_t* vt, const float (&ksa)[2],
                                        const float (&vsa)[2], const float (&nzba)[2], const bool (&valida)[2],
                                        int tok0, int L, float scale_log2) {
    static_assert(HB == BS, "one physical block per tile");
    const float ks = ksa[0], vs = vsa[0], nzb = nzba[0];
    const bool valid = valida[0];
    const float zscale = (KT == PKV_FP16) ? scale_log2 : ks;
#pragma unroll
    for (int h2 = 0; h2 < BS / 16; ++h2) {
      // ---- S = K . q^T over this 16-token slice ----
      float sacc[4] = {0.f, 0.f, 0.f, 0.f};
      const int kr0 = 16 * h2 + g, kx = c * (C::K_ROW / 4);  // rows kr0, kr0 + 8 from byte kx
      if constexpr (KT == PKV_INT8_SYM && IMMA) {
        int ia[3][4];
#pragma unroll
        for (int pl = 0; pl < 3; ++pl) ia[pl][0] = ia[pl][1] = ia[pl][2] = ia[pl][3] = 0;
#pragma unroll
        for (int i = 0; i < KS / 4; ++i) {  // 16 codes = 2 k32-steps per 16-byte load
          const uint4 r0 = *reinterpret_cast<const uint4*>(kt + swz<C::K_ROW>(kr0, kx + 16 * i));
          const uint4 r1 = *reinterpret_cast<const uint4*>(kt + swz<C::K_ROW>(kr0 + 8, kx + 16 * i));
#pragma unroll
          for (int pl = 0; pl < 3; ++pl) {
            imma_16832(ia[pl], r0.x, r1.x, r0.y, r1.y, qp8[pl][2 * i][0], qp8[pl][2 * i][1]);
            imma_16832(ia[pl], r0.z, r1.z, r0.w, r1.w, qp8[pl][2 * i + 1][0], qp8[pl][2 * i + 1][1]);
          }
        }
        // |plane sums| < 2^18: the low two combine exactly in int32, the top one in fp32; then
        // the head's 2^-shift (columns 2c, 2c+1)
#pragma unroll
        for (int r = 0; r < 4; ++r)
          sacc[r] = __fmaf_rn((float)ia[2][r], 65536.f, (float)(ia[1][r] * 256 + ia[0][r])) * qz[r & 1];
      } else if constexpr (KT == PKV_INT8_SYM) {
#pragma unroll
        for (int i = 0; i < KS / 4; ++i) {  // 16 codes = 4 steps per 16-byte load
          const uint4 r0 = *reinterpret_cast<const uint4*>(kt + swz<C::K_ROW>(kr0, kx + 16 * i));
          const uint4 r1 = *reinterpret_cast<const uint4*>(kt + swz<C::K_ROW>(kr0 + 8, kx + 16 * i));
          const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w};
          const uint32_t w1[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint32_t u0 = w0[q4] ^ 0x80808080u, u1 = w1[q4] ^ 0x80808080u;
            uint32_t a[4];
            a[0] = h2_sub(__byte_perm(u0, 0x64646464u, 0x4140), kH2Bias);  // row g, dims +0,+1
            a[1] = h2_sub(__byte_perm(u1, 0x64646464u, 0x4140), kH2Bias);  // row g+8
            a[2] = h2_sub(__byte_perm(u0, 0x64646464u, 0x4342), kH2Bias);  // row g, dims +2,+3
            a[3] = h2_sub(__byte_perm(u1, 0x64646464u, 0x4342), kH2Bias);  // row g+8
            const int kk = 4 * i + q4;
            mma_16816(sacc, a, qb[kk][0], qb[kk][1]);
          }
        }
      } else if constexpr (KT == PKV_FP8_E4M3) {
#pragma unroll
        for (int i = 0; i < KS / 4; ++i) {  // 16 codes = 4 steps per 16-byte load
          const uint4 r0 = *reinterpret_cast<const uint4*>(kt + swz<C::K_ROW>(kr0, kx + 16 * i));
          const uint4 r1 = *reinterpret_cast<const uint4*>(kt + swz<C::K_ROW>(kr0 + 8, kx + 16 * i));
          const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w};
          const uint32_t w1[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t a[4];
            a[0] = fp8x2_to_h2(w0[q4]);        // row g, dims +0,+1
            a[1] = fp8x2_to_h2(w1[q4]);        // row g+8
            a[2] = fp8x2_to_h2(w0[q4] >> 16);  // row g, dims +2,+3
            a[3] = fp8x2_to_h2(w1[q4] >> 16);  // row g+8
            const int kk = 4 * i + q4;
            mma_16816(sacc, a, qb[kk][0], qb[kk][1]);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < KS / 2; ++i) {  // 8 halves = 2 steps per 16-byte load
          const uint4 r0 = *reinterpret_cast<const uint4*>(kt + swz<C::K_ROW>(kr0, kx + 16 * i));
          const uint4 r1 = *reinterpret_cast<const uint4*>(kt + swz<C::K_ROW>(kr0 + 8, kx + 16 * i));
          uint32_t a[4] = {r0.x, r1.x, r0.y, r1.y};
          mma_16816(sacc, a, qb[2 * i][0], qb[2 * i][1]);
          uint32_t b[4] = {r0.z, r1.z, r0.w, r1.w};
          mma_16816(sacc, b, qb[2 * i + 1][0], qb[2 * i + 1][1]);
        }
      }
      // ---- online softmax on the accumulator layout: rows = tokens g, g+8; cols = heads 2c, 2c+1 ----
      const int t0 = tok0 + 16 * h2 + g, t1 = t0 + 8;
      float z[4];
      z[0] = (valid && t0 < L) ? sacc[0] * zscale : -INFINITY;
      z[1] = (valid && t0 < L) ? sacc[1] * zscale : -INFINITY;
      z[2] = (valid && t1 < L) ? sacc[2] * zscale : -INFINITY;
      z[3] = (valid && t1 < L) ? sacc[3] * zscale : -INFINITY;
      float mx0 = fmaxf(z[0], z[2]), mx1 = fmaxf(z[1], z[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
      }
      const bool grow0 = mx0 > m_run[0], grow1 = mx1 > m_run[1];
      if (__any_sync(kFull, grow0 || grow1)) {
        const float al0 = grow0 ? ex2(m_run[0] - mx0) : 1.f;
        const float al1 = grow1 ? ex2(m_run[1] - mx1) : 1.f;
        if (grow0) m_run[0] = mx0;
        if (grow1) m_run[1] = mx1;
        l_run[0] *= al0;
        l_run[1] *= al1;
#pragma unroll
        for (int j = 0; j < KS; ++j) {
          acc[j][0] *= al0;
          acc[j][2] *= al0;
          acc[j][1] *= al1;
          acc[j][3] *= al1;
        }
      }
      const float p0 = ex2(z[0] - m_run[0]), p1 = ex2(z[1] - m_run[1]);
      const float p2 = ex2(z[2] - m_run[0]), p3 = ex2(z[3] - m_run[1]);
      l_run[0] += p0 + p2;
      l_run[1] += p1 + p3;
      // weights for p.v (V scale folded in), fp16 high + low parts, transposed to operand layout
      const float w0 = (VT == PKV_FP16) ? p0 : p0 * vs, w1 = (VT == PKV_FP16) ? p1 : p1 * vs;
      const float w2 = (VT == PKV_FP16) ? p2 : p2 * vs, w3 = (VT == PKV_FP16) ? p3 : p3 * vs;
      const uint32_t hi0 = h2_pack(w0, w1), hi1 = h2_pack(w2, w3);
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&hi0));
      const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&hi1));
      const uint32_t lo0 = h2_pack(w0 - f0.x, w1 - f0.y), lo1 = h2_pack(w2 - f1.x, w3 - f1.y);
      const uint32_t bh0 = movmatrix_trans(hi0), bh1 = movmatrix_trans(hi1);
      const uint32_t bl0 = movmatrix_trans(lo0), bl1 = movmatrix_trans(lo1);
      // ---- O^T += V^T . P^T: token rows 2c, 2c+1, 2c+8, 2c+9 at dims [g*D/8, (g+1)*D/8) ----
      const int vr = 16 * h2 + 2 * c, vx = g * (C::V_ROW / 8);  // rows vr, +1, +8, +9 from byte vx
      if constexpr (VT == PKV_INT8_SYM) {
#pragma unroll
        for (int i = 0; i < KS / 8; ++i) {  // 16 bytes per row = 8 dim tiles
          const uint4 ra = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr, vx + 16 * i));
          const uint4 rb = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr + 1, vx + 16 * i));
          const uint4 rc = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr + 8, vx + 16 * i));
          const uint4 rd = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr + 9, vx + 16 * i));
          const uint32_t xa[4] = {ra.x, ra.y, ra.z, ra.w}, xb[4] = {rb.x, rb.y, rb.z, rb.w};
          const uint32_t xc[4] = {rc.x, rc.y, rc.z, rc.w}, xd[4] = {rd.x, rd.y, rd.z, rd.w};
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {  // dim tile: bytes 2jj (row r) and 2jj+1 (row r+8)
            const int wd = jj / 2, k = 2 * (jj % 2);
            const uint32_t sel0 = k | (k << 4) | ((4 + k) << 8) | ((4 + k) << 12);
            const uint32_t sel1 = (k + 1) | ((k + 1) << 4) | ((5 + k) << 8) | ((5 + k) << 12);
            uint32_t a[4];
            a[0] = h2_sub((__byte_perm(xa[wd], xb[wd], sel0) & 0x00FF00FFu) ^ kH2Bias, kH2Bias);
            a[1] = h2_sub((__byte_perm(xa[wd], xb[wd], sel1) & 0x00FF00FFu) ^ kH2Bias, kH2Bias);
            a[2] = h2_sub((__byte_perm(xc[wd], xd[wd], sel0) & 0x00FF00FFu) ^ kH2Bias, kH2Bias);
            a[3] = h2_sub((__byte_perm(xc[wd], xd[wd], sel1) & 0x00FF00FFu) ^ kH2Bias, kH2Bias);
            const int j = 8 * i + jj;
            mma_16816(acc[j], a, bh0, bh1);
            mma_16816(acc[j], a, bl0, bl1);
          }
        }
      } else if constexpr (VT == PKV_INT4_ASYM) {
        // unswizzled rows of D/2 bytes: dims [g*D/8, (g+1)*D/8) of a row are D/16 bytes, byte jj
        // holding dims 2jj (low nibble, M row g) and 2jj+1 (high nibble, M row g+8) of a dim tile;
        // (1024 + nibble) as fp16 minus (1024 + zp) is the exact (code - zp)
        const float zp = -(nzb + kMagic);
        const uint32_t bias = h2_pack(1024.f + zp, 1024.f + zp);
        const int vb = g * (D / 16);
#pragma unroll
        for (int i = 0; i < KS / 8; ++i) {  // 8 bytes per row = 8 dim tiles
          const uint2 ra = *reinterpret_cast<const uint2*>(vt + vr * C::V_ROW + vb + 8 * i);
          const uint2 rb = *reinterpret_cast<const uint2*>(vt + (vr + 1) * C::V_ROW + vb + 8 * i);
          const uint2 rc = *reinterpret_cast<const uint2*>(vt + (vr + 8) * C::V_ROW + vb + 8 * i);
          const uint2 rd = *reinterpret_cast<const uint2*>(vt + (vr + 9) * C::V_ROW + vb + 8 * i);
          const uint32_t xa[2] = {ra.x, ra.y}, xb[2] = {rb.x, rb.y}, xc[2] = {rc.x, rc.y}, xd[2] = {rd.x, rd.y};
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int wd = jj / 4, k = jj % 4;
            const uint32_t sel = k | ((4 + k) << 8);  // {first.b_k, -, second.b_k, -}
            const uint32_t pab = __byte_perm(xa[wd], xb[wd], sel), pcd = __byte_perm(xc[wd], xd[wd], sel);
            uint32_t a[4];
            a[0] = h2_sub((pab & 0x000F000Fu) | 0x64006400u, bias);
            a[1] = h2_sub(((pab >> 4) & 0x000F000Fu) | 0x64006400u, bias);
            a[2] = h2_sub((pcd & 0x000F000Fu) | 0x64006400u, bias);
            a[3] = h2_sub(((pcd >> 4) & 0x000F000Fu) | 0x64006400u, bias);
            const int j = 8 * i + jj;
            mma_16816(acc[j], a, bh0, bh1);
            mma_16816(acc[j], a, bl0, bl1);
          }
        }
      } else if constexpr (VT == PKV_FP8_E4M3) {
#pragma unroll
        for (int i = 0; i < KS / 8; ++i) {  // 16 codes per row = 8 dim tiles
          const uint4 ra = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr, vx + 16 * i));
          const uint4 rb = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr + 1, vx + 16 * i));
          const uint4 rc = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr + 8, vx + 16 * i));
          const uint4 rd = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr + 9, vx + 16 * i));
          const uint32_t xa[4] = {ra.x, ra.y, ra.z, ra.w}, xb[4] = {rb.x, rb.y, rb.z, rb.w};
          const uint32_t xc[4] = {rc.x, rc.y, rc.z, rc.w}, xd[4] = {rd.x, rd.y, rd.z, rd.w};
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {  // dim tile: bytes 2jj (M row g) and 2jj+1 (M row g+8)
            const int wd = jj / 2, k = 2 * (jj % 2);
            // {row r byte k, row r+1 byte k, row r byte k+1, row r+1 byte k+1}
            const uint32_t sel = k | ((4 + k) << 4) | ((k + 1) << 8) | ((5 + k) << 12);
            const uint32_t pab = __byte_perm(xa[wd], xb[wd], sel), pcd = __byte_perm(xc[wd], xd[wd], sel);
            uint32_t a[4];
            a[0] = fp8x2_to_h2(pab);
            a[1] = fp8x2_to_h2(pab >> 16);
            a[2] = fp8x2_to_h2(pcd);
            a[3] = fp8x2_to_h2(pcd >> 16);
            const int j = 8 * i + jj;
            mma_16816(acc[j], a, bh0, bh1);
            mma_16816(acc[j], a, bl0, bl1);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < KS / 4; ++i) {  // 16 bytes per row = 8 halves = 4 dim tiles
          const uint4 ra = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr, vx + 16 * i));
          const uint4 rb = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr + 1, vx + 16 * i));
          const uint4 rc = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr + 8, vx + 16 * i));
          const uint4 rd = *reinterpret_cast<const uint4*>(vt + swz<C::V_ROW>(vr + 9, vx + 16 * i));
          const uint32_t xa[4] = {ra.x, ra.y, ra.z, ra.w}, xb[4] = {rb.x, rb.y, rb.z, rb.w};
          const uint32_t xc[4] = {rc.x, rc.y, rc.z, rc.w}, xd[4] = {rd.x, rd.y, rd.z, rd.w};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {  // dim tile: half 0 of the word (row r), half 1 (row r+8)
            uint32_t a[4];
            a[0] = __byte_perm(xa[jj], xb[jj], 0x5410);
            a[1] = __byte_perm(xa[jj], xb[jj], 0x7632);
            a[2] = __byte_perm(xc[jj], xd[jj], 0x5410);
            a[3] = __byte_perm(xc[jj], xd[jj], 0x7632);
            const int j = 4 * i + jj;
            mma_16816(acc[j], a, bh0, bh1);
            mma_16816(acc[j], a, bl0, bl1);
          }
        }
      }
    }
  }

  // end of a segment: sum the lanes' partial softmax denominators over the token rows
  __device__ __forceinline__ void finish() {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l_run[0] += __shfl_xor_sync(kFull, l_run[0], off);
      l_run[1] += __shfl_xor_sync(kFull, l_run[1], off);
    }
  }

  // this lane's outputs: heads 2c (acc[.][0], acc[.][2]) and 2c+1 (acc[.][1], acc[.][3]) at
  // dims g*D/8 + 2j (+1)
  __device__ __forceinline__ void write_out(const DecodeParams& p, int s, int hg) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int hh = 2 * c + e;
      if (hh >= GT) continue;
      const float inv = l_run[e] > 0.f ? 1.f / l_run[e] : 0.f;
      __half2* o = reinterpret_cast<__half2*>(p.out + ((size_t)s * p.num_q_heads + (size_t)hg * GT + hh) * D + g * (D / 8));
#pragma unroll
      for (int j = 0; j < KS; ++j) o[j] = __floats2half2_rn(acc[j][e] * inv, acc[j][e + 2] * inv);
    }
  }

  __device__ __forceinline__ void write_partial(const DecodeParams& p, long long slot, int lane) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int hh = 2 * c + e;
      if (hh >= GT) continue;
      float2* dst = reinterpret_cast<float2*>(p.ws_acc + ((size_t)slot * GT + hh) * D + g * (D / 8));
#pragma unroll
      for (int j = 0; j < KS; ++j) dst[j] = make_float2(acc[j][e], acc[j][e + 2]);
      if (g == 0) {
        p.ws_ml[((size_t)slot * GT + hh) * 2 + 0] = m_run[e];
        p.ws_ml[((size_t)slot * GT + hh) * 2 + 1] = l_run[e];
      }
    }
  }
};

template <int KT, int VT, int BS, int D, int GT>
using EngineFor = typename std::conditional<Cfg<KT, VT, BS, D, GT>::MMA, MmaEngine<KT, VT, BS, D, GT>,
                                            CoreEngine<KT, VT, BS, D, GT>>::type;

// ---- merge of a split unit ----
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}
__device__ __forceinline__ float warp_maxf(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
  return v;
}

// Merge the n_seg partials of one unit (slots slot0 .. slot0 + n_seg - 1) and write its outputs:
// out = sum_i 2^(m_i - M) acc_i / sum_i 2^(m_i - M) l_i. Lane i fetches the (max, sum) of partial
// i (32 at a time); each lane owns D / 32 consecutive dims of every head and fetches them from
// four partials at once.
template <int GT, int D>
__device__ __forceinline__ void merge_partials(const DecodeParams& p, long long slot0, int n_seg, long long pslot0,
                                               int n_pref, int s, int hg, int lane) {
  constexpr int DL = D / 32;
  static_assert(DL == 2 || DL == 4 || DL == 8, "head_dim");
  float M[GT], Ls[GT], A[GT][DL];
#pragma unroll
  for (int hh = 0; hh < GT; ++hh) {
    M[hh] = kNegBig;
    Ls[hh] = 0.f;
#pragma unroll
    for (int d = 0; d < DL; ++d) A[hh][d] = 0.f;
  }
  // the warps' partials of the unit, then (shared-prefix decode) the prefix pass's partials
#pragma unroll 1
  for (int range = 0; range < 2; ++range) {
    const float* mlb = range == 0 ? p.ws_ml : p.ws_pml;
    const float* accb = range == 0 ? p.ws_acc : p.ws_pacc;
    const long long base = range == 0 ? slot0 : pslot0;
    const int n = range == 0 ? n_seg : n_pref;
    for (int i0 = 0; i0 < n; i0 += 32) {
      const bool has = i0 + lane < n;
      float e[GT];
#pragma unroll
      for (int hh = 0; hh < GT; ++hh) {
        float2 ml = make_float2(kNegBig, 0.f);
        if (has) ml = __ldcg(reinterpret_cast<const float2*>(mlb) + (base + i0 + lane) * GT + hh);
        const float mn = fmaxf(M[hh], warp_maxf(ml.x));
        const float f = ex2(M[hh] - mn);
        Ls[hh] *= f;
#pragma unroll
        for (int d = 0; d < DL; ++d) A[hh][d] *= f;
        M[hh] = mn;
        e[hh] = has ? ex2(ml.x - mn) : 0.f;
        Ls[hh] += warp_sum(ml.y * e[hh]);
      }
      const int nj = min(32, n - i0);
      for (int j = 0; j < nj; j += 4) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          if (j + jj >= nj) break;
          const long long sl = base + i0 + j + jj;
#pragma unroll
          for (int hh = 0; hh < GT; ++hh) {
            const float ej = __shfl_sync(kFull, e[hh], j + jj);
            const float* src = accb + (sl * GT + hh) * D + lane * DL;
#pragma unroll
            for (int d = 0; d < DL; d += 2) {
              const float2 a = __ldcg(reinterpret_cast<const float2*>(src + d));
              A[hh][d] = fmaf(a.x, ej, A[hh][d]);
              A[hh][d + 1] = fmaf(a.y, ej, A[hh][d + 1]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int hh = 0; hh < GT; ++hh) {
    const float inv = Ls[hh] > 0.f ? 1.f / Ls[hh] : 0.f;
    __half2* o = reinterpret_cast<__half2*>(p.out + ((size_t)s * p.num_q_heads + (size_t)hg * GT + hh) * D + lane * DL);
#pragma unroll
    for (int d = 0; d < DL; d += 2) o[d / 2] = __floats2half2_rn(A[hh][d] * inv, A[hh][d + 1] * inv);
  }
}

// Pull the q rows of unit (s, hg) toward the SM ahead of the engine's begin(): the GT * D fp16
// values are contiguous; one lane per 128-byte line.
template <int GT, int D>
__device__ __forceinline__ void prefetch_q(const DecodeParams& p, int s, int hg, int lane) {
  constexpr int LINES = (GT * D * 2 + 127) / 128;
  const char* base = reinterpret_cast<const char*>(p.q + ((size_t)s * p.num_q_heads + (size_t)hg * GT) * D);
  if (lane < LINES) asm volatile("prefetch.global.L1 [%0];" ::"l"(base + 128 * lane));
}

// ---- fused step: grid-wide phases before the decode ----
// Bound on the polls of one grid barrier (each sleeps ~0.25 us): well under a second.
constexpr int kBarrierPolls = 1 << 21;

// CTA-wide rendezvous on named barrier 1 (every thread of the CTA, from any call site).
__device__ __forceinline__ void cta_sync1() { asm volatile("barrier.sync 1;" ::: "memory"); }

// Grid-wide barrier: the CTA's threads meet, then one thread per CTA arrives and polls until
// `target` CTAs have arrived in total; the rest of the CTA waits at the second rendezvous. The
// cooperative launch keeps every CTA resident, so the wait ends; the poll bound turns a broken
// launch into an error code. `flag`: one int of shared memory for the outcome.
__device__ __forceinline__ bool grid_barrier(uint32_t* ctr, uint32_t target, int32_t* dev_error, int* flag) {
  __threadfence();
  cta_sync1();
  if (threadIdx.x == 0) {
    int ok = 1;
    atomicAdd(ctr, 1u);
    int polls = 0;
    while (*reinterpret_cast<volatile uint32_t*>(ctr) < target) {
      if (++polls > kBarrierPolls) {
        record_error(dev_error, PKV_DEVERR_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(256);
    }
    __threadfence();
    *flag = ok;
  }
  cta_sync1();
  return *flag != 0;
}

// After the CTA's warps are all done, the last CTA to leave clears the barrier counters for the
// next call.
__device__ __forceinline__ void grid_exit(uint32_t* bar, uint32_t ctas) {
  cta_sync1();
  if (threadIdx.x == 0 && atomicAdd(&bar[1], 1u) == ctas - 1) {
    bar[0] = 0;
    bar[1] = 0;
  }
}

// The store phase: (token, KV head) jobs spread over the grid's warps in job order.
template <int KT, int VT>
__device__ __noinline__ void step_store(const StoreParams& sp, int w, int W, int lane, uint8_t* tbl) {
  const int jobs = sp.T * sp.num_kv_heads;
  for (int job = w; job < jobs; job += W)
    store_detail::store_job<KT, VT>(sp, job / sp.num_kv_heads, job % sp.num_kv_heads, lane, tbl);
}

// BS: the pool's block size; VB: physical blocks per stream position (1, or 2 for the paired walk
// of the CUDA-core engine: the tile holds two consecutive blocks of the unit, which halves the
// per-position work of the copy ring and the walk).
template <int KT, int VT, int BS, int D, int GT, bool FUSED, int VB>
__global__ void __launch_bounds__(Cfg<KT, VT, BS * VB, D, GT>::THREADS, Cfg<KT, VT, BS * VB, D, GT>::CTAS_PER_SM)
    paged_decode_kernel(const DecodeParams p, const StepParams sp, const __grid_constant__ TileMaps tm) {
  using C = Cfg<KT, VT, BS * VB, D, GT>;
  static_assert(VB == 1 || (VB == 2 && !C::MMA), "paired blocks: CUDA-core engine only");
  // stream positions of a unit with nphys private blocks
  auto npos = [](int nphys) -> int { return (nphys + VB - 1) / VB; };
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  constexpr uint32_t kAlign = C::SMEM_ALIGN ? C::SMEM_ALIGN : 1;
  uint8_t* const smem = smem_raw + ((kAlign - (smem_addr(smem_raw) & (kAlign - 1))) & (kAlign - 1));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int W = gridDim.x * C::NW;
  const int w = blockIdx.x * C::NW + warp;
  const int HG = p.num_q_heads / GT;
  const int S = p.num_seqs;
  // Sequences are walked in the caller's order when one is given (sequences that share blocks
  // placed next to each other read them while they are still in L2); an entry outside [0, S)
  // makes that walk position empty and is reported.
  auto sid = [&](int k) -> int {
    if (p.seq_order == nullptr) return k;
    const int a = __ldg(p.seq_order + k);
    if (a < 0 || a >= S) {
      record_error(p.dev_error, PKV_DEVERR_SEQ_ORDER);
      return -1;
    }
    return a;
  };
  auto len_at = [&](int k) -> int {  // clamped length of the sequence at walk position k < S
    const int a = sid(k);
    return a < 0 ? 0 : clamp_len(p, p.context_lens[a], BS);
  };
  // Shared-prefix decode: leading blocks of the sequence at walk position k (length L) that the
  // prefix pass attended; at least its last block stays with the decode (a count beyond that is
  // clamped and reported).
  auto sb_at = [&](int k, int L) -> int {
    if (p.shared_blocks == nullptr || L == 0) return 0;
    const int a = p.seq_order == nullptr ? k : __ldg(p.seq_order + k);  // valid: L > 0
    const int v = p.shared_blocks[a];
    const int sb = max(0, min(v, min((L + BS - 1) / BS - 1, p.max_shared_blocks)));
    if (sb != v && w == 0) record_error(p.dev_error, PKV_DEVERR_SHARED);
    return sb;
  };

  uint8_t* my_stages = smem + (size_t)warp * C::NS * C::STAGE;
  uint64_t* my_bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_STAGES) + warp * C::NS;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < C::NS; ++st) mbar_init(&my_bars[st], 1);
    fence_mbar_init();
  }

  // ---- fused step: the copy-on-write copies, then the stores, by every warp of the grid ----
  uint32_t phases = 0;  // grid barriers passed (each counts every CTA once)
  int* bar_flag = reinterpret_cast<int*>(smem + C::SMEM_BAR_FLAG);
  if constexpr (FUSED) {
    if (sp.copy.n_pairs > 0) {
      copy_detail::copy_all(sp.copy, (int64_t)blockIdx.x * C::THREADS + threadIdx.x, (int64_t)gridDim.x * C::THREADS);
      grid_barrier(sp.bar, gridDim.x * ++phases, p.dev_error, bar_flag);
    }
    step_store<KT, VT>(sp.store, w, W, lane, my_stages);  // a rebuild's table borrows the ring
    __syncwarp();
  }

  // ---- pass 1: total stream length T; zero the outputs of empty sequences ----
  long long T = 0;
  for (int base = 0; base < S; base += 32) {
    const int s = base + lane;
    int L = 0;
    if (s < S) {
      const int raw = p.context_lens[s];
      L = clamp_len(p, raw, BS);
      if (raw != L && w == 0) record_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN);
    }
    // the stream counts the sequences in walk order (the same as index order without one)
    const int Lw = p.seq_order == nullptr ? L : (s < S ? len_at(s) : 0);
    int sum = npos((Lw + BS - 1) / BS - (s < S ? sb_at(s, Lw) : 0));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
    T += sum;
    uint32_t empty = __ballot_sync(kFull, s < S && L == 0);
    while (empty) {  // outputs of sequences with nothing to attend over are 0
      const int e = __ffs(empty) - 1;
      empty &= empty - 1;
      const int se = base + e;
      for (int hg = 0; hg < HG; ++hg) {
        if ((int)(((long long)se * HG + hg) % W) != w) continue;
        __half2* o = reinterpret_cast<__half2*>(p.out + ((size_t)se * p.num_q_heads + (size_t)hg * GT) * D);
        for (int i = lane; i < GT * D / 2; i += 32) o[i] = __floats2half2_rn(0.f, 0.f);
      }
    }
  }
  T *= HG;
  __syncwarp();
  // With fewer blocks than warps only the first T warps work, so that every working warp owns
  // at least one block and the warps sharing a unit are consecutive (the merge relies on it).
  const int We = (int)min((long long)W, T);
  if (w >= We) {  // nothing to decode; in a fused step still a party to the barrier
    if constexpr (FUSED) {
      grid_barrier(sp.bar, gridDim.x * ++phases, p.dev_error, bar_flag);
      grid_exit(sp.bar, gridDim.x);
    }
    return;
  }
  const long long start = (long long)w * T / We;
  const long long end = (long long)(w + 1) * T / We;

  // ---- pass 2: the unit and block of `start` ----
  Win cur;
  int Lchunk = 0, SBchunk = 0, chunk_base = 0;  // lane: length and shared blocks at walk position chunk_base + lane
  {
    long long acc0 = 0;
    cur.s = cur.sa = 0;
    cur.L = cur.nblk = 1;
    cur.sb = 0;
    cur.seq_p0 = 0;
    for (int base = 0; base < S; base += 32) {  // found before base reaches S: start < T
      const int s = base + lane;
      const int L = s < S ? len_at(s) : 0;
      const int sb = s < S ? sb_at(s, L) : 0;
      const long long cnt = (long long)npos((L + BS - 1) / BS - sb) * HG;
      long long incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long o = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += o;
      }
      const long long total = __shfl_sync(kFull, incl, 31);
      if (acc0 + total > start) {
        const uint32_t m = __ballot_sync(kFull, acc0 + incl > start);
        const int f = __ffs(m) - 1;
        cur.s = base + f;
        cur.sa = p.seq_order == nullptr ? cur.s : __ldg(p.seq_order + cur.s);  // valid: it has blocks
        cur.L = __shfl_sync(kFull, L, f);
        cur.sb = __shfl_sync(kFull, sb, f);
        cur.nblk = npos((cur.L + BS - 1) / BS - cur.sb);
        cur.seq_p0 = acc0 + __shfl_sync(kFull, incl - cnt, f);
        Lchunk = L;
        SBchunk = sb;
        chunk_base = base;
        break;
      }
      acc0 += total;
    }
    const long long o = start - cur.seq_p0;
    cur.hg = (int)(o / cur.nblk);
    cur.j0 = (int)(o % cur.nblk);
    cur.g = (cur.hg * GT) / p.group;
    cur.r0 = 0;
    cur.n = (int)min((long long)min(32, cur.nblk - cur.j0), end - start);
  }
  const int n_total = (int)(end - start);  // positions of this warp

  // clamped length of sequence s, from the lane-held chunk when possible
  auto seq_len = [&](int s) -> int {
    if (s < chunk_base || s >= chunk_base + 32) {
      chunk_base = s;
      Lchunk = (s + lane < S) ? len_at(s + lane) : 0;
      SBchunk = (s + lane < S) ? sb_at(s + lane, Lchunk) : 0;
    }
    return __shfl_sync(kFull, Lchunk, s - chunk_base);
  };
  auto seq_sb = [&](int s) -> int { return __shfl_sync(kFull, SBchunk, s - chunk_base); };  // after seq_len(s)

  // the window after `a`, within [.., end); n = 0 if none
  auto next_win = [&](const Win& a) -> Win {
    Win b = a;
    b.r0 = a.r0 + a.n;
    b.n = 0;
    if (a.n == 0 || b.r0 >= n_total) return b;
    b.j0 = a.j0 + a.n;
    if (b.j0 >= a.nblk) {
      b.j0 = 0;
      b.hg = a.hg + 1;
      if (b.hg >= HG) {
        b.hg = 0;
        b.seq_p0 = a.seq_p0 + (long long)HG * a.nblk;
        int s = a.s, L = 0;
        do {  // sequences without blocks contribute no stream positions
          ++s;
          L = s < S ? seq_len(s) : 0;
        } while (L == 0 && s < S);
        b.s = s;
        b.sa = (s < S && p.seq_order != nullptr) ? __ldg(p.seq_order + s) : s;  // valid when L > 0
        b.L = L;
        b.sb = s < S ? seq_sb(s) : 0;
        b.nblk = npos((L + BS - 1) / BS - b.sb);
      }
      b.g = (b.hg * GT) / p.group;
    }
    b.n = min(min(32, b.nblk - b.j0), n_total - b.r0);
    return b;
  };

  // phase A of a window: block ids (one per lane); phase B (at its first copy): scales
  auto load_ids = [&](const Win& a, WinLanes<VB>& r) {
    r.meta = false;
    const int nphys = (a.L + BS - 1) / BS - a.sb;  // the unit's private blocks
#pragma unroll
    for (int h = 0; h < VB; ++h) {
      r.b[h] = -1;
      if (lane < a.n && VB * (a.j0 + lane) + h < nphys)
        r.b[h] = p.block_tables[(size_t)a.sa * p.max_blocks_per_seq + a.sb + VB * (a.j0 + lane) + h];
    }
  };
  auto load_meta = [&](const Win& a, WinLanes<VB>& r) {
    const int nphys = (a.L + BS - 1) / BS - a.sb;
#pragma unroll
    for (int h = 0; h < VB; ++h) {
      const bool has = lane < a.n && VB * (a.j0 + lane) + h < nphys;
      const bool valid = has && r.b[h] >= 0 && r.b[h] < p.num_blocks;
      if (has && !valid) record_error(p.dev_error, PKV_DEVERR_BLOCK_ID);
      r.b[h] = valid ? r.b[h] : (has ? 0 : -1);
      r.ks[h] = r.vs[h] = 0.f;
      r.zv[h] = valid ? 0.f : -1.f;
      if (has) {
        const size_t meta = (size_t)r.b[h] * p.num_kv_heads + a.g;
        if constexpr (KT != PKV_FP16) r.ks[h] = p.k_scale[meta] * p.scale_log2;  // log2 domain
        if constexpr (VT != PKV_FP16) r.vs[h] = p.v_scale[meta];
        if constexpr (VT == PKV_INT4_ASYM) if (valid) r.zv[h] = (float)p.v_zp[meta];
      }
    }
    r.meta = true;
  };

  prefetch_q<GT, D>(p, cur.sa, cur.hg, lane);
  WinLanes<VB> rc, rn;
  load_ids(cur, rc);
  Win nxt = next_win(cur);
  load_ids(nxt, rn);
  if (nxt.n > 0 && (nxt.s != cur.s || nxt.hg != cur.hg)) prefetch_q<GT, D>(p, nxt.sa, nxt.hg, lane);
  // Everything above reads only what the host wrote before the preceding kernel (lengths,
  // tables). From here on the pool is read, which the preceding kernel (the store of the new
  // tokens) may still be writing: wait for it to complete (no-op without a programmatic launch).
  // In a fused step, wait instead for every warp's stores, and order them (written through the
  // generic proxy) before this warp's bulk copies (the async proxy).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if constexpr (FUSED) {
    grid_barrier(sp.bar, gridDim.x * ++phases, p.dev_error, bar_flag);
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  load_meta(cur, rc);
  __syncwarp();  // barrier initialisation by lane 0 is visible to the warp


  // ---- the copy ring ----
  // one physical (block, KV head) tile: its K rows to kd, its V rows to vd. A tiled copy takes the
  // tile's BS rows from row tile * BS, swizzled; a 1-D bulk copy takes them as they are.
  auto copy_tile = [&](uint8_t* kd, uint8_t* vd, int b, int g, uint64_t* bar) {
    constexpr uint32_t PK = BS * C::K_ROW, PV = BS * C::V_ROW;
    const size_t tile = (size_t)b * p.num_kv_heads + g;
    const int row = (int)(tile * BS);
    if constexpr (!C::TILED_K) bulk_g2s(kd, static_cast<const uint8_t*>(p.k_codes) + tile * PK, PK, bar);
    else if constexpr (C::K_ROW == 128) tma_load_2d(kd, &tm.k, 0, row, bar);
    else tma_load_3d(kd, &tm.k, 0, 0, row, bar);
    if constexpr (!C::V_SWZ) bulk_g2s(vd, static_cast<const uint8_t*>(p.v_codes) + tile * PV, PV, bar);
    else if constexpr (C::V_ROW == 128) tma_load_2d(vd, &tm.v, 0, row, bar);
    else tma_load_3d(vd, &tm.v, 0, 0, row, bar);
  };
  // a stream position: one tile, or two (paired walk) whose rows follow each other
  auto issue = [&](int st, int b, int b1, bool has1, int g) {
    constexpr uint32_t PK = BS * C::K_ROW, PV = BS * C::V_ROW;
    uint8_t* dst = my_stages + (size_t)st * C::STAGE;
    mbar_arrive_expect_tx(&my_bars[st], (has1 ? 2u : 1u) * (PK + PV));
    copy_tile(dst, dst + C::K_TILE, b, g, &my_bars[st]);
    if (has1) copy_tile(dst + PK, dst + C::K_TILE + PV, b1, g, &my_bars[st]);
  };
  // positions relative to `start`: consumed (cpos) and issued (ipos); stage / parity of each
  int cpos = 0, ipos = 0, cst = 0, ist = 0;
  uint32_t cpar = 0;
  // issue every position below min(cpos + NS, n_total) whose window is known (cur or nxt); a
  // stage is reused only after the position NS before it has been consumed
  auto issue_ahead = [&]() {
    const int lim = min(cpos + C::NS, n_total);
    while (ipos < lim) {
      int b, b1 = -1, g;
      if (ipos < cur.r0 + cur.n) {
        b = __shfl_sync(kFull, rc.b[0], ipos - cur.r0);
        if constexpr (VB == 2) b1 = __shfl_sync(kFull, rc.b[VB - 1], ipos - cur.r0);
        g = cur.g;
      } else if (nxt.n > 0 && ipos < nxt.r0 + nxt.n) {
        if (!rn.meta) load_meta(nxt, rn);
        b = __shfl_sync(kFull, rn.b[0], ipos - nxt.r0);
        if constexpr (VB == 2) b1 = __shfl_sync(kFull, rn.b[VB - 1], ipos - nxt.r0);
        g = nxt.g;
      } else {
        break;
      }
      if (lane == 0) issue(ist, b, b1, b1 >= 0, g);
      ist = (ist + 1 == C::NS) ? 0 : ist + 1;
      ++ipos;
    }
  };

  // A split unit's ticket. The warp that writes a partial must make it visible before its ticket
  // counts (a release fence, then a relaxed increment); only the warp that gets the last ticket
  // needs the partials of the others (an acquire fence, then the merge). The release fence waits
  // for the warp's outstanding writes, so with one query head per warp (registers to spare) the
  // ticket is taken two blocks later, when the partial's writes have long completed, and read at
  // the next split-unit end (or after the last block). Otherwise all of it happens at once.
  constexpr bool kDeferTicket = GT == 1;
  int pend = 0;              // 0: none; 1: partial written, ticket not taken; 2: ticket taken
  int pend_since = 0;        // cpos when the partial was written
  uint32_t pend_ticket = 0;  // lane 0: the increment's result
  uint32_t pend_nseg = 0;
  long long pend_slot0 = 0, pend_u = 0, pend_pslot0 = 0;
  int pend_s = 0, pend_hg = 0, pend_np = 0;
  auto take_ticket = [&]() {
    if (lane == 0) {
      fence_acq_rel_gpu();
      pend_ticket = atomic_inc_relaxed_gpu(&p.ws_count[pend_u], pend_nseg - 1);
    }
    pend = 2;
  };
  auto resolve_pending = [&]() {
    if (pend == 0) return;
    if (pend == 1) take_ticket();
    const uint32_t t = __shfl_sync(kFull, pend_ticket, 0);
    if (t == pend_nseg - 1) {
      // Lane 0 read the last ticket: its acquire fence orders the other warps' partials (released
      // before their increments) before its later reads; the warp barrier then extends that
      // order to every lane of the warp before any of them reads a partial.
      if (lane == 0) fence_acq_rel_gpu();
      __syncwarp();
      merge_partials<GT, D>(p, pend_slot0, (int)pend_nseg, pend_pslot0, pend_np, pend_s, pend_hg, lane);
    }
    pend = 0;
  };

  // the first copies go out before the engine's set-up (which waits for q)
  issue_ahead();
  // ---- per-unit state: the arithmetic engine for GT query heads ----
  EngineFor<KT, VT, BS * VB, D, GT> eng;
  int seg_j0 = cur.j0;  // first block of the current segment within its unit
  eng.begin(p, cur.sa, cur.hg, lane);

  bool aborted = false;
  while (cpos < n_total) {
    if (cpos == cur.r0 + cur.n) {  // step into the next window
      const bool new_unit = (nxt.s != cur.s) || (nxt.hg != cur.hg);
      cur = nxt;
      rc = rn;
      if (!rc.meta) load_meta(cur, rc);
      nxt = next_win(cur);
      load_ids(nxt, rn);
      if (nxt.n > 0 && (nxt.s != cur.s || nxt.hg != cur.hg)) prefetch_q<GT, D>(p, nxt.sa, nxt.hg, lane);
      if (new_unit) {
        eng.begin(p, cur.sa, cur.hg, lane);
        seg_j0 = cur.j0;
      }
    }
    issue_ahead();
    const int st = cst;
    if (!__all_sync(kFull, mbar_wait_bounded(&my_bars[st], cpar))) {
      if (lane == 0) record_error(p.dev_error, PKV_DEVERR_TIMEOUT);
      aborted = true;
      break;
    }

    // ---- one block: q . k, online softmax, p . v ----
    const int kw_i = cpos - cur.r0;
    float ks[2], vs[2], nzb[2];
    bool valid[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // per physical block of the position (the second only when paired)
      if (h < VB) {
        const int hv = h < VB ? h : 0;
        ks[h] = __shfl_sync(kFull, rc.ks[hv], kw_i);  // K scale, log2 domain
        vs[h] = __shfl_sync(kFull, rc.vs[hv], kw_i);
        const float zv = __shfl_sync(kFull, rc.zv[hv], kw_i);
        nzb[h] = -(kMagic + zv);
        valid[h] = zv >= 0.f;
      } else {
        ks[h] = ks[0];
        vs[h] = vs[0];
        nzb[h] = nzb[0];
        valid[h] = valid[0];
      }
    }
    const uint8_t* kt = my_stages + (size_t)st * C::STAGE;
    eng.template block<BS>(kt, kt + C::K_TILE, ks, vs, nzb, valid, (cur.sb + VB * (cur.j0 + kw_i)) * BS, cur.L,
                           p.scale_log2);
    __syncwarp();  // the stage's reads are complete (their values were consumed above)
    if constexpr (kDeferTicket) {
      if (pend == 1 && cpos >= pend_since + 2) take_ticket();
    }
    ++cpos;
    if (++cst == C::NS) {
      cst = 0;
      cpar ^= 1u;
    }

    // ---- end of a segment: the unit's last block, or the end of this warp's range ----
    const int j_end = cur.j0 + kw_i + 1;
    if (j_end == cur.nblk || cpos == n_total) {
      eng.finish();
      const long long u = (long long)cur.s * HG + cur.hg;
      if (seg_j0 == 0 && j_end == cur.nblk && cur.sb == 0) {
        eng.write_out(p, cur.sa, cur.hg);  // the whole unit was processed by this warp
      } else {
        // one segment of a split unit: publish the partial; the last warp to finish merges
        eng.write_partial(p, u + w, lane);
        const long long unit_p0 = cur.seq_p0 + (long long)cur.hg * cur.nblk;
        const int w_first = owner_of(unit_p0, T, We);
        const int w_last = owner_of(unit_p0 + cur.nblk - 1, T, We);
        const uint32_t n_seg = (uint32_t)(w_last - w_first + 1);
        __syncwarp();  // the warp's partial writes precede lane 0's release fence
        if constexpr (kDeferTicket) resolve_pending();
        pend = 1;
        pend_since = cpos;
        pend_nseg = n_seg;
        pend_u = u;
        pend_slot0 = u + w_first;
        pend_s = cur.sa;
        pend_hg = cur.hg;
        // a unit with a shared prefix also folds in the prefix pass's partials
        pend_np = cur.sb > 0 ? p.prefix_splits : 0;
        pend_pslot0 = ((long long)cur.sa * HG + cur.hg) * p.prefix_splits;
        if constexpr (!kDeferTicket) resolve_pending();
      }
      eng.reset();
      seg_j0 = j_end;  // (a new unit restarts it at its first block)
    }
  }

  if constexpr (kDeferTicket) resolve_pending();
  if (aborted && lane == 0) {
    // A copy never completed (outputs touched by this warp are unspecified; dev_error says so).
    // Wait, again bounded, for the copies this warp issued and did not consume, so that no bulk
    // copy is still writing this CTA's shared memory when it exits.
    for (int k = cpos; k < ipos; ++k) (void)mbar_wait_bounded(&my_bars[k % C::NS], (uint32_t)((k / C::NS) & 1));
  }
  if constexpr (FUSED) grid_exit(sp.bar, gridDim.x);
}

template <int KT, int VT, int BS, int D, int GT, int VB>
cudaError_t launch_vb(const DecodeParams& p, const StepParams& sp, const DecodeShape& sh, cudaStream_t stream) {
  using C = Cfg<KT, VT, BS * VB, D, GT>;
  auto kern = sp.fused ? paged_decode_kernel<KT, VT, BS, D, GT, true, VB>
                       : paged_decode_kernel<KT, VT, BS, D, GT, false, VB>;
  static unsigned long long configured[2] = {0, 0};  // one bit per device and variant; benign race
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured[sp.fused ? 1 : 0] & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured[sp.fused ? 1 : 0] |= bit;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sh.grid_ctas);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (sp.fused) {
    // the grid barriers need every CTA resident at once: a cooperative launch guarantees it
    // (or fails to launch)
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    // programmatic dependent launch: the kernel may start while the previous kernel in the
    // stream finishes; it waits for it (griddepcontrol.wait) before reading the pool
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  TileMaps tm;
  memset(&tm, 0, sizeof(tm));
  if constexpr (C::TILED_K) {
    const uint64_t rows = (uint64_t)p.num_blocks * p.num_kv_heads * BS;
    if (!encode_tile_map(&tm.k, p.k_codes, rows, C::K_ROW, BS)) return cudaErrorInvalidValue;
    if (C::V_SWZ && !encode_tile_map(&tm.v, p.v_codes, rows, C::V_ROW, BS)) return cudaErrorInvalidValue;
  }
  return cudaLaunchKernelEx(&cfg, kern, p, sp, tm);
}

// The paired walk (two 16-token blocks per stream position) for the CUDA-core engine with INT8 K
// and INT8 / INT4 V, unless the decode starts units after shared-prefix blocks (whose count need
// not be even). (At a unit's end a paired position may hold one block; the other half of its tile
// keeps stale bytes, masked by the length: codes of any bytes are finite numbers, which fp16 bytes
// are not.)
template <int KT, int VT, int BS, int D, int GT>
cudaError_t launch_one(const DecodeParams& p, const StepParams& sp, const DecodeShape& sh, cudaStream_t stream) {
  if constexpr (PKV_DECODE_PAIR && BS == 16 && KT == PKV_INT8_SYM && VT != PKV_FP16 && !Cfg<KT, VT, BS, D, GT>::MMA &&
                Cfg<KT, VT, 2 * BS, D, GT>::NW == Cfg<KT, VT, BS, D, GT>::NW) {
    if (p.shared_blocks == nullptr) return launch_vb<KT, VT, BS, D, GT, 2>(p, sp, sh, stream);
  }
  return launch_vb<KT, VT, BS, D, GT, 1>(p, sp, sh, stream);
}

template <int KT, int VT, int BS, int D, int GT>
bool info_one(DecodeKernelInfo* info) {
  using C = Cfg<KT, VT, BS, D, GT>;
  info->warps_per_cta = C::NW;
  info->ctas_per_sm = C::CTAS_PER_SM;
  info->smem_bytes = C::SMEM;
  info->stages = C::NS;
  return true;
}

// 8 heads per warp exist only with the tensor-core engine
template <int KT, int VT, int BS, int D>
cudaError_t launch_one8(const DecodeParams& p, const StepParams& sp, const DecodeShape& sh, cudaStream_t stream) {
  if constexpr (Cfg<KT, VT, BS, D, 8>::MMA) return launch_one<KT, VT, BS, D, 8>(p, sp, sh, stream);
  else return cudaErrorInvalidValue;
}
template <int KT, int VT, int BS, int D>
bool info_one8(DecodeKernelInfo* info) {
  if constexpr (Cfg<KT, VT, BS, D, 8>::MMA) return info_one<KT, VT, BS, D, 8>(info);
  else return false;
}

// FN<KT, VT, BS, D, GT>(args...) for the instantiation matching `sh`
#define PKV_DISPATCH_GT(KT, VT, BS, D, FN, ...)       \
  switch (sh.heads_per_warp) {                        \
    case 1: return FN<KT, VT, BS, D, 1>(__VA_ARGS__); \
    case 2: return FN<KT, VT, BS, D, 2>(__VA_ARGS__); \
    case 4: return FN<KT, VT, BS, D, 4>(__VA_ARGS__); \
    case 8: return FN##8<KT, VT, BS, D>(__VA_ARGS__); \
    default: break;                                   \
  }
#define PKV_DISPATCH_D(KT, VT, BS, FN, ...)                   \
  switch (sh.head_dim) {                                      \
    case 64: PKV_DISPATCH_GT(KT, VT, BS, 64, FN, __VA_ARGS__) break;   \
    case 128: PKV_DISPATCH_GT(KT, VT, BS, 128, FN, __VA_ARGS__) break; \
    case 256: PKV_DISPATCH_GT(KT, VT, BS, 256, FN, __VA_ARGS__) break; \
    default: break;                                           \
  }
#define PKV_DISPATCH_BS(KT, VT, FN, ...)                      \
  switch (sh.block_size) {                                    \
    case 16: PKV_DISPATCH_D(KT, VT, 16, FN, __VA_ARGS__) break; \
    case 32: PKV_DISPATCH_D(KT, VT, 32, FN, __VA_ARGS__) break; \
    default: break;                                           \
  }
}  // namespace
}  // namespace pkv
