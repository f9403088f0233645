// prefill_kernel.cuh -- chunked-prefill attention over the paged, block-quantized KV cache (sm_100a).
//
// What it computes: sequence s holds q_len = cu_q_lens[s+1] - cu_q_lens[s] new query tokens, the
// last q_len of its context_lens[s] tokens (their K/V already stored by pkv_store_quantized); the
// query at position p attends causally to tokens 0 .. p of the sequence:
//   out[row][h] = sum_{t <= p} softmax_t(softmax_scale * q[row][h] . k_hat_t) * v_hat_t
// with k_hat = code * k_scale, v_hat = (code - zp) * v_scale dequantized inside the kernel
// (yunthe.com "LLM推理显存优化KV Cache量化与PagedAttention实现详解", section "Prefix Caching与多轮对话场景
// 优化实践": only the new tokens are computed, over the cached prefix; section "KV Cache量化技术原理":
// x_hat = (Q - zero_point) * scale; tbr8.org "如何通过 PagedAttention 与分块量化结合..." §5 item 2:
// dequantization inside the attention operator, no dequantized copy of the cache).
//
// How (B200 design, not taken from the pages). A CTA of 8 warps takes 128 query columns (a column
// is one (query token, query head) pair of one KV head) and streams the blocks they need through a
// ring of K/V tile stages filled by bulk tensor copies (one thread issues them, an mbarrier per
// stage). Per block:
//   * S^T = Q . K^T on the integer tensor cores (mma m16n8k32 s8 x s8 -> s32): each warp owns 16
//     columns; q is put on a 22-bit fixed-point grid per column and split into three signed byte
//     planes (exact, as in the decode), so the int8 K codes are multiplied as they sit in shared
//     memory, with no conversion at all;
//   * online softmax per column (log2 domain); the running maximum is moved only when a block's
//     maximum exceeds it by more than 2^8, so the accumulators are rescaled rarely; weights (with
//     the block's V scale folded in) are split into an fp16 high and low part and written to
//     shared memory;
//   * one CTA barrier; then O^T += V^T . P^T on the fp16 tensor cores (mma m16n8k16): each warp
//     owns 16 of the 128 dims for all 128 columns, so every V code is converted to fp16 exactly
//     once per CTA (byte permutes plus one fp16 subtraction per pair), and the weights arrive by
//     ldmatrix.
// At the end each column is normalised by its sum and written as fp16.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace pkv {
namespace prefill_detail {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kCols = 128;        // query columns per CTA
constexpr int kD = 128;           // head_dim
constexpr float kGrowLog2 = 8.f;  // the running maximum moves when exceeded by more than this

template <int VT, int BS>
struct Cfg {
  static constexpr int K_ROW = kD;                                   // int8 codes
  static constexpr int V_ROW = VT == PKV_INT4_ASYM ? kD / 2 : kD;    // int8 or packed nibbles
  static constexpr int K_TILE = BS * K_ROW, V_TILE = BS * V_ROW;
  static constexpr bool V_SWZ = V_ROW % 128 == 0;                    // V by a swizzled tiled copy
  static constexpr int STAGE = ((K_TILE + V_TILE) + 1023) / 1024 * 1024;
  static constexpr int NS = 4;                                       // ring depth (blocks)
  static constexpr int P_ROW = 2 * BS + 16;                          // bytes per column (padded: no bank conflicts)
  static constexpr int P_BUF = kCols * P_ROW;                        // one of (high, low) of one parity
  static constexpr int OFF_P = NS * STAGE;
  static constexpr int OFF_ALPHA = OFF_P + 4 * P_BUF;                // [2 parity][kCols] f32
  static constexpr int OFF_FLAG = OFF_ALPHA + 2 * kCols * 4;         // [2 parity][kWarps] int
  static constexpr int OFF_L = OFF_FLAG + 2 * kWarps * 4;            // [kCols] f32 final sums
  static constexpr int OFF_META = OFF_L + kCols * 4;                 // [NS] per-stage block facts
  static constexpr int OFF_BAR = OFF_META + NS * 16;                 // [NS] mbarriers
  static constexpr int SMEM = OFF_BAR + NS * 8 + 1024;               // + alignment slack
  static_assert(P_ROW % 16 == 0, "ldmatrix rows are 16-byte aligned");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void imma_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void hmma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2_pack(float lo, float hi) {
  const __half2 r = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&r);
}
// Byte offset of (row r, byte x) in a tile of 128-byte rows stored with 128-byte swizzle: the
// 16-byte chunk j of row r sits at chunk j ^ (r mod 8).
__device__ __forceinline__ int swz128(int r, int x) { return (r << 7) | ((((x >> 4) & 7) ^ (r & 7)) << 4) | (x & 15); }

// What the consumer of a stage needs to know about its block (written by the thread that issues
// the block's copies, read after a CTA barrier).
struct StageMeta {
  int valid;  // the table held a block id inside the pool
  float ks, vs, zp;
};

// fp16 1024 + 128 in both halves: (b ^ 0x80) under exponent 0x64 reads 1024 + 128 + c for a signed
// byte c, so subtracting this leaves c exactly
constexpr uint32_t kH2Bias8 = 0x64806480u;

}  // namespace

template <int VT, int BS, bool PREFIX>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ TileMaps tm) {
  using C = Cfg<VT, BS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* const smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int kvh = blockIdx.y;
  const int G = p.group;
  const int col0 = blockIdx.x * kCols;  // first column of this CTA
  const int cap_tab = p.max_blocks_per_seq * BS;

  // ---- the work of this CTA: its columns, the blocks they see, where the results go ----
  // Prefill: columns of sequence s = blockIdx.z are (chunk token i, head hh) = (c / G, c % G);
  //   blocks [0, the last column's causal limit); the output rows are normalised.
  // Prefix (shared-prefix decode): columns of group gi = blockIdx.z / splits are (member m, head
  //   hh) = (c / G, c % G) with the members' one decode query each; blocks [split * per_split,
  //   ...) of the group's shared blocks, all visible; the results are partials for the decode.
  int ncols, jb, je, s_tab, pos0 = 0, q0 = 0, gstart = 0, split = 0;
  if constexpr (!PREFIX) {
    const int s = blockIdx.z;
    q0 = p.cu_q_lens[s];
    const int qlen = p.cu_q_lens[s + 1] - q0;
    if (q0 < 0 || qlen < 0 || qlen > p.max_q_len || q0 + qlen > p.total_q) {  // rows outside q / out
      if (threadIdx.x == 0 && blockIdx.x == 0 && kvh == 0) record_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN);
      return;
    }
    if (qlen == 0 || col0 >= qlen * G) return;
    ncols = min(kCols, qlen * G - col0);
    int ctx = p.context_lens[s];
    const int cap = min(p.max_context_len, cap_tab);
    if (qlen > ctx || ctx > cap) {
      // a chunk longer than its context, or a context beyond the table / the host bound: the
      // rows are zeroed (the first CTA of the sequence and head reports it)
      if (threadIdx.x == 0 && blockIdx.x == 0 && kvh == 0) record_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN);
      if (qlen > ctx) {
        for (int col = threadIdx.x; col < ncols; col += kThreads) {
          const int gc = col0 + col;
          __half2* o = reinterpret_cast<__half2*>(p.out + ((size_t)(q0 + gc / G) * p.num_q_heads +
                                                           (size_t)kvh * G + gc % G) * kD);
          for (int d = 0; d < kD / 2; ++d) o[d] = __floats2half2_rn(0.f, 0.f);
        }
        return;
      }
      ctx = cap;
    }
    pos0 = ctx - qlen;  // position of the first query token
    const int lim_last = min(pos0 + (col0 + ncols - 1) / G + 1, cap);  // the last column sees the most
    jb = 0;
    je = (lim_last + BS - 1) / BS;
    s_tab = s;
  } else {
    const int gi = blockIdx.z / p.splits;
    split = blockIdx.z % p.splits;
    gstart = p.group_start[gi];
    const int gsize = p.group_start[gi + 1] - gstart;
    if (gstart < 0 || gsize < 0 || gsize > p.max_group_size || gstart + gsize > p.n_members) {
      if (threadIdx.x == 0 && blockIdx.x == 0 && kvh == 0 && split == 0) record_error(p.dev_error, PKV_DEVERR_SHARED);
      return;
    }
    if (gsize == 0 || col0 >= gsize * G) return;
    ncols = min(kCols, gsize * G - col0);
    s_tab = p.members[gstart];
    if (s_tab < 0 || s_tab >= p.num_seqs) return;  // reported by the decode, which skips it too
    // the group's shared blocks, as the decode counts them for its first member
    const int L = max(0, min(p.context_lens[s_tab], min(p.max_context_len, cap_tab)));
    const int nb = (L + BS - 1) / BS;
    const int sb = max(0, min(p.shared_blocks[s_tab], min(nb - 1, p.max_shared_blocks)));
    jb = min(split * p.per_split, sb);
    je = min(jb + p.per_split, sb);
  }
  const int nblk = je - jb;

  uint8_t* const stages = smem;
  uint8_t* const pbuf = smem + C::OFF_P;
  float* const alpha_s = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
  int* const flag_s = reinterpret_cast<int*>(smem + C::OFF_FLAG);
  float* const lsum_s = reinterpret_cast<float*>(smem + C::OFF_L);
  uint64_t* const bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  StageMeta* const meta = reinterpret_cast<StageMeta*>(smem + C::OFF_META);

  const int32_t* table = p.block_tables + (size_t)s_tab * p.max_blocks_per_seq + jb;
  int issued = 0;            // thread 0: blocks whose copies have been issued
  auto issue = [&](int j) {  // thread 0: copies of the CTA's block j into stage j % NS, and its facts
    const int raw = table[j];
    const bool valid = raw >= 0 && raw < p.num_blocks;  // an invalid id reads block 0, masked, reported
    const int b = valid ? raw : 0;
    if (!valid) record_error(p.dev_error, PKV_DEVERR_BLOCK_ID);
    const int st = j % C::NS;
    const size_t mi = (size_t)b * p.num_kv_heads + kvh;
    StageMeta m;
    m.valid = valid ? 1 : 0;
    m.ks = p.k_scale[mi];
    m.vs = p.v_scale[mi];
    m.zp = VT == PKV_INT4_ASYM ? (float)p.v_zp[mi] : 0.f;
    meta[st] = m;
    ++issued;
    uint8_t* dst = stages + st * C::STAGE;
    mbar_arrive_expect_tx(&bars[st], (uint32_t)(C::K_TILE + C::V_TILE));
    const int row = (int)(((size_t)b * p.num_kv_heads + kvh) * BS);
    tma_load_2d(dst, &tm.k, 0, row, &bars[st]);
    if constexpr (C::V_SWZ) {
      tma_load_2d(dst + C::K_TILE, &tm.v, 0, row, &bars[st]);
    } else {
      bulk_g2s(dst + C::K_TILE,
               static_cast<const uint8_t*>(p.v_codes) + ((size_t)b * p.num_kv_heads + kvh) * C::V_TILE,
               (uint32_t)C::V_TILE, &bars[st]);
    }
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    for (int j = 0; j < min(C::NS, nblk); ++j) issue(j);
  }
  __syncthreads();  // barriers initialised, first stages' facts visible

  // ---- this warp's 16 columns: q on a 22-bit grid in three signed byte planes (A operands) ----
  // Lane (g, c) holds columns cA = 16 warp + g and cB = cA + 8 at dims [32c, 32c + 32); within an
  // mma k-step kk the logical k range [4c, 4c+4) is dims 32c + 8kk + [0, 4) and [16+4c, 16+4c+4)
  // is dims 32c + 8kk + [4, 8), for both operands.
  uint32_t qa[3][4][4];
  float zsc[2];  // per column: 2^-shift * softmax_scale * log2(e)
  int lim[2];    // per column: tokens t < lim are visible
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int col = 16 * warp + g + 8 * e;
    const int gc = col0 + col;
    const int tok = gc / G;
    bool valid = col < ncols;
    size_t qrow = 0;  // (row, head) of q
    if constexpr (!PREFIX) {
      qrow = (size_t)(q0 + tok) * p.num_q_heads + (size_t)kvh * G + gc % G;
    } else {
      const int sm = valid ? p.members[gstart + tok] : -1;
      valid = valid && sm >= 0 && sm < p.num_seqs;
      qrow = (size_t)max(sm, 0) * p.num_q_heads + (size_t)kvh * G + gc % G;
    }
    float x[32];
    if (valid) {
      const uint4* qp = reinterpret_cast<const uint4*>(p.q + qrow * kD + 32 * c);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
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
      for (int i = 0; i < 32; ++i) x[i] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    int ex = 0;
    (void)frexpf(amax, &ex);                    // amax < 2^ex
    const int shift = amax > 0.f ? 22 - ex : 0;  // |q| * 2^shift < 2^22
    const float up = __int_as_float((127 + shift) << 23);
    zsc[e] = __int_as_float((127 - shift) << 23) * p.scale_log2;
    lim[e] = !valid ? 0 : (PREFIX ? INT_MAX : pos0 + tok + 1);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
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
        const int reg = e + 2 * h;  // a0: cA low k, a1: cB low k, a2: cA high k, a3: cB high k
        qa[0][kk][reg] = p0;
        qa[1][kk][reg] = p1;
        qa[2][kk][reg] = p2;
      }
    }
  }

  float m_used[2] = {-INFINITY, -INFINITY};  // per column (uniform over the 4 lanes of a column)
  float l_part[2] = {0.f, 0.f};              // this lane's share of each column's sum
  float acc[16][4];                          // O^T: dims of this warp x all 128 columns
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

  const uint32_t p_base = smem_addr(pbuf);
  bool aborted = false;
  int abort_at = 0;
  for (int j = 0; j < nblk; ++j) {
    const int st = j % C::NS;
    const int par = j & 1;
    const bool ok = mbar_wait_bounded(&bars[st], (uint32_t)((j / C::NS) & 1));
    const uint8_t* kt = stages + st * C::STAGE;
    const uint8_t* vt = kt + C::K_TILE;
    const StageMeta bm_ = meta[st];
    const bool bvalid = bm_.valid != 0;
    const float ks = bm_.ks, vs = bm_.vs;
    const int tok0 = (jb + j) * BS;

    // ---- S^T = Q K^T for this warp's 16 columns and the block's BS tokens ----
    float z[BS / 8][4];
#pragma unroll
    for (int nt = 0; nt < BS / 8; ++nt) {
      const int row = 8 * nt + g;
      const uint4 r0 = *reinterpret_cast<const uint4*>(kt + swz128(row, 32 * c));
      const uint4 r1 = *reinterpret_cast<const uint4*>(kt + swz128(row, 32 * c + 16));
      const uint32_t bw[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
      int a[3][4];
#pragma unroll
      for (int pl = 0; pl < 3; ++pl) {
        a[pl][0] = a[pl][1] = a[pl][2] = a[pl][3] = 0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) imma_16832(a[pl], qa[pl][kk], bw[2 * kk], bw[2 * kk + 1]);
      }
      // d0: (cA, token 2c), d1: (cA, 2c+1), d2: (cB, 2c), d3: (cB, 2c+1) of this n-tile
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float raw = __fmaf_rn((float)a[2][r], 65536.f, (float)(a[1][r] * 256 + a[0][r]));
        const int e = r >> 1;
        const int t = tok0 + 8 * nt + 2 * c + (r & 1);
        z[nt][r] = (bvalid && t < lim[e]) ? raw * (zsc[e] * ks) : -INFINITY;
      }
    }
    // ---- online softmax per column ----
    float bm[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < BS / 8; ++nt) {
      bm[0] = fmaxf(bm[0], fmaxf(z[nt][0], z[nt][1]));
      bm[1] = fmaxf(bm[1], fmaxf(z[nt][2], z[nt][3]));
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      bm[e] = fmaxf(bm[e], __shfl_xor_sync(kFull, bm[e], 1));
      bm[e] = fmaxf(bm[e], __shfl_xor_sync(kFull, bm[e], 2));
    }
    float al[2] = {1.f, 1.f};
    bool grew = false;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (bm[e] > m_used[e] + kGrowLog2) {  // (-inf + 8 is -inf: the first visible block sets it)
        al[e] = m_used[e] == -INFINITY ? 0.f : ex2(m_used[e] - bm[e]);
        m_used[e] = bm[e];
        l_part[e] *= al[e];
        grew = true;
      }
    }
    grew = __any_sync(kFull, grew);
    if (c == 0) {
      alpha_s[par * kCols + 16 * warp + g] = al[0];
      alpha_s[par * kCols + 16 * warp + g + 8] = al[1];
    }
    if (lane == 0) flag_s[par * kWarps + warp] = grew ? 1 : 0;
    // weights (V scale folded in) as fp16 high + low parts, rows [column][token]
    uint8_t* phi = pbuf + (2 * par) * C::P_BUF;
    uint8_t* plo = phi + C::P_BUF;
#pragma unroll
    for (int nt = 0; nt < BS / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        // (a column with nothing visible yet keeps m_used = -inf: its weights are 0)
        const bool live = m_used[e] != -INFINITY;
        const float w0 = live ? ex2(z[nt][2 * e] - m_used[e]) : 0.f;
        const float w1 = live ? ex2(z[nt][2 * e + 1] - m_used[e]) : 0.f;
        l_part[e] += w0 + w1;
        const float v0 = w0 * vs, v1 = w1 * vs;
        const uint32_t hi = h2_pack(v0, v1);
        const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi));
        const uint32_t lo = h2_pack(v0 - hf.x, v1 - hf.y);
        const int off = (16 * warp + g + 8 * e) * C::P_ROW + 2 * (8 * nt + 2 * c);
        *reinterpret_cast<uint32_t*>(phi + off) = hi;
        *reinterpret_cast<uint32_t*>(plo + off) = lo;
      }
    }
    // every warp's weights are written and every warp is done with the previous block's stage
    aborted = __syncthreads_or(!ok) != 0;
    if (aborted) {
      abort_at = j;
      break;
    }
    if (threadIdx.x == 0 && j + C::NS - 1 < nblk && j >= 1) issue(j + C::NS - 1);

    // ---- O^T += V^T P^T: this warp's 16 dims (M rows g and g+8 are dims 16g + 2w and + 1) ----
    const int* flags = flag_s + par * kWarps;
#pragma unroll
    for (int w2 = 0; w2 < kWarps; ++w2) {
      if (flags[w2]) {  // columns of warp w2 moved their maximum: n-tiles 2 w2 and 2 w2 + 1
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 a2 = *reinterpret_cast<const float2*>(alpha_s + par * kCols + 8 * (2 * w2 + h) + 2 * c);
          float* ac = acc[2 * w2 + h];
          ac[0] *= a2.x;
          ac[1] *= a2.y;
          ac[2] *= a2.x;
          ac[3] *= a2.y;
        }
      }
    }
    const float zp = bm_.zp;
#pragma unroll
    for (int ks16 = 0; ks16 < BS / 16; ++ks16) {
      // A = V^T (16 dims x 16 tokens): a0 (dim row g, tokens 2c, 2c+1), a1 (row g+8, same
      // tokens), a2 (row g, tokens 2c+8, 2c+9), a3 (row g+8, tokens 2c+8, 2c+9)
      uint32_t av[4];
      const int t0 = 16 * ks16 + 2 * c;
      if constexpr (VT == PKV_INT4_ASYM) {
        const int x = 8 * g + warp;  // byte of dims 16g + 2w (low nibble) and 16g + 2w + 1 (high)
        const uint32_t y0 = vt[(t0)*C::V_ROW + x], y1 = vt[(t0 + 1) * C::V_ROW + x];
        const uint32_t y2 = vt[(t0 + 8) * C::V_ROW + x], y3 = vt[(t0 + 9) * C::V_ROW + x];
        const uint32_t pa = y0 | (y1 << 16), pb = y2 | (y3 << 16);
        const uint32_t bias = h2_pack(1024.f + zp, 1024.f + zp);  // 1024 + zp exact in fp16
        av[0] = h2_sub((pa & 0x000F000Fu) | 0x64006400u, bias);
        av[1] = h2_sub(((pa >> 4) & 0x000F000Fu) | 0x64006400u, bias);
        av[2] = h2_sub((pb & 0x000F000Fu) | 0x64006400u, bias);
        av[3] = h2_sub(((pb >> 4) & 0x000F000Fu) | 0x64006400u, bias);
      } else {
        const int x = 16 * g + 2 * warp;  // bytes of dims 16g + 2w and 16g + 2w + 1
        auto ld2 = [&](int t) -> uint32_t {
          return (uint32_t)*reinterpret_cast<const uint16_t*>(vt + swz128(t, x));
        };
        const uint32_t y0 = ld2(t0), y1 = ld2(t0 + 1), y2 = ld2(t0 + 8), y3 = ld2(t0 + 9);
        // {dim 2w of token t, dim 2w of token t+1} and the same for dim 2w+1, biased bytes
        // result bytes {first.b0, -, second.b0, -} (selector 0x0400) or the b1 bytes (0x0501)
        av[0] = h2_sub((__byte_perm(y0, y1, 0x0400) & 0x00FF00FFu) ^ kH2Bias8, kH2Bias8);
        av[1] = h2_sub((__byte_perm(y0, y1, 0x0501) & 0x00FF00FFu) ^ kH2Bias8, kH2Bias8);
        av[2] = h2_sub((__byte_perm(y2, y3, 0x0400) & 0x00FF00FFu) ^ kH2Bias8, kH2Bias8);
        av[3] = h2_sub((__byte_perm(y2, y3, 0x0501) & 0x00FF00FFu) ^ kH2Bias8, kH2Bias8);
      }
      // B = P^T (16 tokens x 8 columns) per n-tile, high and low parts by one ldmatrix.x4:
      // matrices (high, tokens 0-7), (high, 8-15), (low, 0-7), (low, 8-15) of the k-step
      const int mi = lane >> 3, mr = lane & 7;
      const uint32_t lrow = p_base + (uint32_t)((2 * par + (mi >> 1)) * C::P_BUF + mr * C::P_ROW +
                                                 2 * (16 * ks16 + 8 * (mi & 1)));
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        uint32_t bfr[4];
        ldsm_x4(bfr, lrow + (uint32_t)(8 * n * C::P_ROW));
        hmma_16816(acc[n], av, bfr[0], bfr[1]);
        hmma_16816(acc[n], av, bfr[2], bfr[3]);
      }
    }
  }

  if (aborted) {
    if (threadIdx.x == 0) {
      record_error(p.dev_error, PKV_DEVERR_TIMEOUT);
      // let every copy still in flight land before the CTA's shared memory is released: the
      // blocks from the one whose wait gave up to the last one issued (bounded waits again)
      for (int k = abort_at; k < issued; ++k) (void)mbar_wait_bounded(&bars[k % C::NS], (uint32_t)((k / C::NS) & 1));
    }
    return;
  }

  // ---- column sums ----
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    l_part[e] += __shfl_xor_sync(kFull, l_part[e], 1);
    l_part[e] += __shfl_xor_sync(kFull, l_part[e], 2);
  }
  if constexpr (PREFIX) {
    // partials for the decode: slot (sequence, decode head group, split), head within the group;
    // (max, sum) from the lanes that own each column, accumulators from every warp
    const int GT = p.gt, HGd = p.num_q_heads / p.gt;
    auto slot_of = [&](int col, int& hh) -> long long {
      const int gc = col0 + col;
      const int sm = p.members[gstart + gc / G];
      if (sm < 0 || sm >= p.num_seqs) return -1;
      const int h = kvh * G + gc % G;
      hh = h % GT;
      return ((long long)sm * HGd + h / GT) * p.splits + split;
    };
    if (c == 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = 16 * warp + g + 8 * e;
        if (col >= ncols) continue;
        int hh;
        const long long sl = slot_of(col, hh);
        if (sl < 0) continue;
        float* ml = p.pml + (sl * GT + hh) * 2;
        ml[0] = m_used[e] == -INFINITY ? -1.0e30f : m_used[e];
        ml[1] = l_part[e];
      }
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = 8 * n + 2 * c + e;
        if (col >= ncols) continue;
        int hh;
        const long long sl = slot_of(col, hh);
        if (sl < 0) continue;
        *reinterpret_cast<float2*>(p.pacc + (sl * GT + hh) * kD + 16 * g + 2 * warp) =
            make_float2(acc[n][e], acc[n][e + 2]);
      }
    }
    return;
  }
  // ---- normalise and write ----
  if (c == 0) {
    lsum_s[16 * warp + g] = l_part[0];
    lsum_s[16 * warp + g + 8] = l_part[1];
  }
  __syncthreads();
#pragma unroll
  for (int n = 0; n < 16; ++n) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int col = 8 * n + 2 * c + e;
      if (col >= ncols) continue;
      const float l = lsum_s[col];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int gc = col0 + col;
      __half* o = p.out + ((size_t)(q0 + gc / G) * p.num_q_heads + (size_t)kvh * G + gc % G) * kD + 16 * g + 2 * warp;
      *reinterpret_cast<__half2*>(o) = __floats2half2_rn(acc[n][e] * inv, acc[n][e + 2] * inv);
    }
  }
}

}  // namespace prefill_detail
}  // namespace pkv
