// prefill_tc.cuh -- multi-query paged attention on the fifth-generation tensor cores (tcgen05):
// chunked prefill and the shared-prefix pass of the decode (sm_100a).
//
// What it computes is what prefill_kernel.cuh states (the same work split per CTA: 128 query
// columns of one KV head, a range of blocks of one block table, causal limits for a prefill,
// partial softmax states for the shared-prefix pass). How:
//   * the CTA's 128 columns are the M = 128 rows of the MMAs; a thread owns one column, which is
//     one lane of tensor memory, so its softmax needs no shuffles;
//   * S = Q K^T per block: tcgen05.mma kind::i8 with A = q in three exact signed byte planes
//     (written once to shared memory in the 128-byte-swizzled K-major layout) and B = the block's
//     int8 K codes exactly as the tiled copy left them (K-major, 128-byte swizzle); int32
//     accumulators in tensor memory, three planes combined per thread;
//   * O += P V per block: tcgen05.mma kind::f16 with A = the weights (fp16 high and low parts,
//     K-major) and B = the V codes turned into exact fp16 integers once per block by the CTA's
//     threads (MN-major, 128-byte swizzle); the accumulator stays in tensor memory for the whole
//     block range and is rescaled in place only when a column's maximum grows by more than 2^8.
// One thread issues the MMAs; completion is tracked with tcgen05.commit on an mbarrier.
#pragma once

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace pkv {
namespace prefill_tc {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kThreads = 128;  // one thread per column
constexpr int kCols = 128;
constexpr int kD = 128;
constexpr float kGrowLog2 = 8.f;
constexpr uint32_t kTmemCols = 256;  // S planes at columns [0, 3 BS), O at [128, 256)
constexpr uint32_t kOCol = 128;

template <int VT, int BS>
struct Cfg {
  static constexpr int K_ROW = kD;
  static constexpr int V_ROW = VT == PKV_INT4_ASYM ? kD / 2 : kD;
  static constexpr int K_TILE = BS * K_ROW, V_TILE = BS * V_ROW;
  static constexpr bool V_SWZ = V_ROW % 128 == 0;
  static constexpr int STAGE = (K_TILE + V_TILE + 1023) / 1024 * 1024;
  static constexpr int NS = 4;
  static constexpr int QPL = kCols * kD;        // one q byte plane (A of S), 128-byte swizzled
  static constexpr int VH = BS * kD * 2;        // fp16 V of one block (B of PV)
  static constexpr int P_SBO = (BS / 8) * 128;  // weights: 8-row groups of (BS/8) 8x16-byte cores
  static constexpr int PB = kCols / 8 * P_SBO;  // one of (high, low)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_ST = OFF_Q + 3 * QPL;
  static constexpr int OFF_V = OFF_ST + NS * STAGE;
  static constexpr int OFF_P = OFF_V + 2 * VH;
  static constexpr int OFF_META = OFF_P + 2 * PB;
  static constexpr int OFF_BAR = OFF_META + NS * 16;
  static constexpr int OFF_TMEM = OFF_BAR + (NS + 1) * 8;
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;  // + alignment slack
  // S: M = 128 columns x N = BS tokens, s8 x s8 -> s32, both K-major
  static constexpr uint32_t ID_S = tc::idesc(2, 1, 1, 0, 0, 128, BS);
  // PV: M = 128 columns x N = 128 dims, f16 x f16 -> f32, A K-major, B MN-major
  static constexpr uint32_t ID_PV = tc::idesc(1, 0, 0, 0, 1, 128, kD);
  static_assert(OFF_ST % 1024 == 0 && OFF_V % 1024 == 0 && STAGE % 1024 == 0 && VH % 1024 == 0, "atoms");
  static_assert(3 * BS <= (int)kOCol, "tensor memory columns");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct StageMeta {
  int valid;
  float ks, vs, zp;
};

__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2_pack(float lo, float hi) {
  const __half2 r = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ int swz128(int r, int x) { return (r << 7) | ((((x >> 4) & 7) ^ (r & 7)) << 4) | (x & 15); }
constexpr uint32_t kH2Bias8 = 0x64806480u;

}  // namespace

template <int VT, int BS, bool PREFIX>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_tc_kernel(const PrefillParams p, const __grid_constant__ TileMaps tm) {
  using C = Cfg<VT, BS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* const smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int kvh = blockIdx.y;
  const int G = p.group;
  const int col0 = blockIdx.x * kCols;
  const int cap_tab = p.max_blocks_per_seq * BS;

  // ---- the work of this CTA (as in prefill_kernel.cuh) ----
  int ncols, jb, je, s_tab, pos0 = 0, q0 = 0, gstart = 0, split = 0;
  if constexpr (!PREFIX) {
    const int s = blockIdx.z;
    q0 = p.cu_q_lens[s];
    const int qlen = p.cu_q_lens[s + 1] - q0;
    if (q0 < 0 || qlen < 0 || qlen > p.max_q_len || q0 + qlen > p.total_q) {
      if (tid == 0 && blockIdx.x == 0 && kvh == 0) record_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN);
      return;
    }
    if (qlen == 0 || col0 >= qlen * G) return;
    ncols = min(kCols, qlen * G - col0);
    int ctx = p.context_lens[s];
    const int cap = min(p.max_context_len, cap_tab);
    if (qlen > ctx || ctx > cap) {
      if (tid == 0 && blockIdx.x == 0 && kvh == 0) record_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN);
      if (qlen > ctx) {
        if (tid < ncols) {
          const int gc = col0 + tid;
          uint4* o = reinterpret_cast<uint4*>(p.out + ((size_t)(q0 + gc / G) * p.num_q_heads + (size_t)kvh * G + gc % G) * kD);
          for (int d = 0; d < kD / 8; ++d) o[d] = make_uint4(0u, 0u, 0u, 0u);
        }
        return;
      }
      ctx = cap;
    }
    pos0 = ctx - qlen;
    const int lim_last = min(pos0 + (col0 + ncols - 1) / G + 1, cap);
    jb = 0;
    je = (lim_last + BS - 1) / BS;
    s_tab = s;
  } else {
    const int gi = blockIdx.z / p.splits;
    split = blockIdx.z % p.splits;
    gstart = p.group_start[gi];
    const int gsize = p.group_start[gi + 1] - gstart;
    if (gstart < 0 || gsize < 0 || gsize > p.max_group_size || gstart + gsize > p.n_members) {
      if (tid == 0 && blockIdx.x == 0 && kvh == 0 && split == 0) record_error(p.dev_error, PKV_DEVERR_SHARED);
      return;
    }
    if (gsize == 0 || col0 >= gsize * G) return;
    ncols = min(kCols, gsize * G - col0);
    s_tab = p.members[gstart];
    if (s_tab < 0 || s_tab >= p.num_seqs) return;
    const int L = max(0, min(p.context_lens[s_tab], min(p.max_context_len, cap_tab)));
    const int nb = (L + BS - 1) / BS;
    const int sb = max(0, min(p.shared_blocks[s_tab], min(nb - 1, p.max_shared_blocks)));
    jb = min(split * p.per_split, sb);
    je = min(jb + p.per_split, sb);
  }
  const int nblk = je - jb;

  uint8_t* const qsm = smem + C::OFF_Q;
  uint8_t* const stages = smem + C::OFF_ST;
  uint8_t* const vsm = smem + C::OFF_V;
  uint8_t* const psm = smem + C::OFF_P;
  StageMeta* const meta = reinterpret_cast<StageMeta*>(smem + C::OFF_META);
  uint64_t* const bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* const mma_bar = bars + C::NS;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);

  const int32_t* table = p.block_tables + (size_t)s_tab * p.max_blocks_per_seq + jb;
  int issued = 0;
  auto issue = [&](int j) {  // thread 0: block j's copies into stage j % NS, and its facts
    const int raw = table[j];
    const bool valid = raw >= 0 && raw < p.num_blocks;
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
      bulk_g2s(dst + C::K_TILE, static_cast<const uint8_t*>(p.v_codes) + mi * C::V_TILE, (uint32_t)C::V_TILE,
               &bars[st]);
    }
  };

  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i <= C::NS; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    for (int j = 0; j < min(C::NS, nblk); ++j) issue(j);
  }

  // ---- this thread's column: q on a 22-bit grid in three signed byte planes (A of S) ----
  const int col = tid;
  const int gc = col0 + col;
  const int tok = gc / G;
  bool cvalid = col < ncols;
  size_t qrow = 0;
  if constexpr (!PREFIX) {
    qrow = (size_t)(q0 + tok) * p.num_q_heads + (size_t)kvh * G + gc % G;
  } else {
    const int sm = cvalid ? p.members[gstart + tok] : -1;
    cvalid = cvalid && sm >= 0 && sm < p.num_seqs;
    qrow = (size_t)max(sm, 0) * p.num_q_heads + (size_t)kvh * G + gc % G;
  }
  const uint4* qp = reinterpret_cast<const uint4*>(p.q + qrow * kD);
  float amax = 0.f;
  if (cvalid) {
    for (int i = 0; i < kD / 8; ++i) {
      const uint4 wv = qp[i];
      const uint32_t u[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[k]));
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
  int ex = 0;
  (void)frexpf(amax, &ex);
  const int shift = amax > 0.f ? 22 - ex : 0;
  const float up = __int_as_float((127 + shift) << 23);
  const float zsc = __int_as_float((127 - shift) << 23) * p.scale_log2;
  const int lim = !cvalid ? 0 : (PREFIX ? INT_MAX : pos0 + tok + 1);
  {
    const int r8 = col & 7;
    uint8_t* rowp = qsm + (col >> 3) * 1024 + r8 * 128;
    for (int j = 0; j < kD / 16; ++j) {  // 16 dims = one 16-byte chunk of each plane
      uint32_t w[3][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint4 wv = make_uint4(0u, 0u, 0u, 0u);
        if (cvalid) wv = qp[2 * j + h];
        const uint32_t u[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int wd = 0; wd < 2; ++wd) {
          uint32_t pl0 = 0, pl1 = 0, pl2 = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[2 * wd + (k >> 1)]));
            const int qi = __float2int_rn(((k & 1) ? f.y : f.x) * up);
            const int b0 = ((qi + 128) & 0xFF) - 128;
            const int r1 = (qi - b0) >> 8;
            const int b1 = ((r1 + 128) & 0xFF) - 128;
            const int b2 = (r1 - b1) >> 8;
            pl0 |= (uint32_t)(b0 & 0xFF) << (8 * k);
            pl1 |= (uint32_t)(b1 & 0xFF) << (8 * k);
            pl2 |= (uint32_t)(b2 & 0xFF) << (8 * k);
          }
          w[0][2 * h + wd] = pl0;
          w[1][2 * h + wd] = pl1;
          w[2][2 * h + wd] = pl2;
        }
      }
#pragma unroll
      for (int pl = 0; pl < 3; ++pl)
        *reinterpret_cast<uint4*>(rowp + pl * C::QPL + ((j ^ r8) << 4)) = make_uint4(w[pl][0], w[pl][1], w[pl][2], w[pl][3]);
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's lanes

  const uint32_t q_base = smem_addr(qsm), st_base = smem_addr(stages), v_base = smem_addr(vsm), p_base = smem_addr(psm);
  float m_used = -INFINITY, lsum = 0.f;
  uint32_t mma_phase = 0;
  bool aborted = false;
  int abort_at = 0;
  for (int j = 0; j < nblk; ++j) {
    const int st = j % C::NS;
    const int par = j & 1;
    bool ok = mbar_wait_bounded(&bars[st], (uint32_t)((j / C::NS) & 1));
    const uint32_t k_addr = st_base + st * C::STAGE;
    if (tid == 0 && ok) {
      tc::fence_after_sync();
#pragma unroll
      for (int pl = 0; pl < 3; ++pl)
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk)
          tc::mma_i8(tmem + pl * BS, tc::smem_desc(q_base + pl * C::QPL + kk * 32, 16, 1024, tc::kLayoutSw128),
                     tc::smem_desc(k_addr + kk * 32, 16, 1024, tc::kLayoutSw128), C::ID_S, kk > 0 ? 1u : 0u);
      tc::commit(mma_bar);
    }
    const StageMeta bm = meta[st];
    // ---- V codes of the block -> exact fp16 (code - zp), MN-major 128-byte-swizzled atoms of
    // 8 tokens x 64 dims; the V scale goes into the weights ----
    if (ok) {
      const uint8_t* vt = stages + st * C::STAGE + C::K_TILE;
      uint8_t* vdst = vsm + par * C::VH;
      const uint32_t zbias = h2_pack(1024.f + bm.zp, 1024.f + bm.zp);
#pragma unroll
      for (int k = 0; k < BS / 8; ++k) {
        const int ci = tid + kThreads * k;
        const int tk = ci >> 4, dc = ci & 15;  // token, 8-dim chunk
        uint32_t h[4];
        if constexpr (VT == PKV_INT4_ASYM) {
          const uint32_t x = *reinterpret_cast<const uint32_t*>(vt + tk * C::V_ROW + 4 * dc);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t t = x >> (8 * b);
            h[b] = h2_sub((t & 0xFu) | ((t << 12) & 0xF0000u) | 0x64006400u, zbias);
          }
        } else {
          const uint2 x = *reinterpret_cast<const uint2*>(vt + swz128(tk, 8 * dc));
          const uint32_t u0 = x.x ^ 0x80808080u, u1 = x.y ^ 0x80808080u;
          h[0] = h2_sub(__byte_perm(u0, 0x64646464u, 0x5140), kH2Bias8);
          h[1] = h2_sub(__byte_perm(u0, 0x64646464u, 0x5342), kH2Bias8);
          h[2] = h2_sub(__byte_perm(u1, 0x64646464u, 0x5140), kH2Bias8);
          h[3] = h2_sub(__byte_perm(u1, 0x64646464u, 0x5342), kH2Bias8);
        }
        const int r8 = tk & 7, c8 = dc & 7;
        *reinterpret_cast<uint4*>(vdst + (tk >> 3) * 2048 + (dc >> 3) * 1024 + r8 * 128 + ((c8 ^ r8) << 4)) =
            make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
    tc::fence_proxy_async_smem();
    // ---- S of this block: this thread's column, three planes ----
    ok = ok && mbar_wait_bounded(mma_bar, mma_phase & 1u);
    ++mma_phase;
    tc::fence_after_sync();
    float z[BS];
    {
#pragma unroll
      for (int h16 = 0; h16 < BS / 16; ++h16) {
        uint32_t r0[16], r1[16], r2[16];
        tc::ld_x16(t_lane + 0 * BS + 16 * h16, r0);
        tc::ld_x16(t_lane + 1 * BS + 16 * h16, r1);
        tc::ld_x16(t_lane + 2 * BS + 16 * h16, r2);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = (jb + j) * BS + 16 * h16 + i;
          const float raw = __fmaf_rn((float)(int)r2[i], 65536.f, (float)((int)r1[i] * 256 + (int)r0[i]));
          z[16 * h16 + i] = (bm.valid && t < lim) ? raw * (zsc * bm.ks) : -INFINITY;
        }
      }
    }
    float bmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < BS; ++i) bmax = fmaxf(bmax, z[i]);
    // (-inf + 8 is -inf: the first visible block sets the maximum)
    const bool grow = bmax > m_used + kGrowLog2;
    float al = 1.f;
    if (grow) {
      al = m_used == -INFINITY ? 0.f : ex2(m_used - bmax);
      lsum *= al;
    }
    // a column whose O holds earlier blocks is rescaled in place (the warp's lanes load and store
    // together; the others multiply by 1)
    const bool rescale = grow && j > 0 && m_used != -INFINITY;
    if (grow) m_used = bmax;
    if (__any_sync(kFull, rescale)) {
      const float f = rescale ? al : 1.f;
#pragma unroll 1
      for (int c16 = 0; c16 < kD / 16; ++c16) {
        uint32_t r[16];
        tc::ld_x16(t_lane + kOCol + 16 * c16, r);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
        tc::st_x16(t_lane + kOCol + 16 * c16, r);
      }
      tc::wait_st();
    }
    // weights, V scale folded in, fp16 high + low parts: this column's row of the A operand
    {
      const bool live = m_used != -INFINITY;
      uint32_t hi[BS / 2], lo[BS / 2];
#pragma unroll
      for (int i = 0; i < BS; i += 2) {
        const float w0 = live ? ex2(z[i] - m_used) : 0.f, w1 = live ? ex2(z[i + 1] - m_used) : 0.f;
        lsum += w0 + w1;
        const float v0 = w0 * bm.vs, v1 = w1 * bm.vs;
        hi[i / 2] = h2_pack(v0, v1);
        const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi[i / 2]));
        lo[i / 2] = h2_pack(v0 - hf.x, v1 - hf.y);
      }
      uint8_t* prow = psm + (col >> 3) * C::P_SBO + (col & 7) * 16;
#pragma unroll
      for (int c8 = 0; c8 < BS / 8; ++c8) {
        *reinterpret_cast<uint4*>(prow + c8 * 128) = make_uint4(hi[4 * c8], hi[4 * c8 + 1], hi[4 * c8 + 2], hi[4 * c8 + 3]);
        *reinterpret_cast<uint4*>(prow + C::PB + c8 * 128) =
            make_uint4(lo[4 * c8], lo[4 * c8 + 1], lo[4 * c8 + 2], lo[4 * c8 + 3]);
      }
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    aborted = __syncthreads_or(!ok) != 0;
    tc::fence_after_sync();
    if (aborted) {
      abort_at = j;
      break;
    }
    if (tid == 0) {
      // ---- O += P V (high then low weights), then refill the block's stage ----
#pragma unroll
      for (int ks = 0; ks < BS / 16; ++ks) {
        const uint64_t bd = tc::smem_desc(v_base + par * C::VH + ks * 4096, 1024, 2048, tc::kLayoutSw128);
        tc::mma_f16(tmem + kOCol, tc::smem_desc(p_base + ks * 256, 128, C::P_SBO, tc::kLayoutNone), bd, C::ID_PV,
                    (j > 0 || ks > 0) ? 1u : 0u);
        tc::mma_f16(tmem + kOCol, tc::smem_desc(p_base + C::PB + ks * 256, 128, C::P_SBO, tc::kLayoutNone), bd,
                    C::ID_PV, 1u);
      }
      if (j + C::NS < nblk) issue(j + C::NS);
    }
  }

  // ---- the last products complete; then the column's output or partial ----
  bool done_ok = true;
  if (tid == 0) tc::commit(mma_bar);
  done_ok = mbar_wait_bounded(mma_bar, mma_phase & 1u);
  ++mma_phase;
  tc::fence_after_sync();
  if (aborted || !done_ok) {
    if (tid == 0) {
      record_error(p.dev_error, PKV_DEVERR_TIMEOUT);
      for (int k = abort_at; k < issued; ++k) (void)mbar_wait_bounded(&bars[k % C::NS], (uint32_t)((k / C::NS) & 1));
    }
  } else {
    // (every lane takes part in the tensor-memory loads; only valid columns store)
    const bool have_o = nblk > 0;
    if constexpr (!PREFIX) {
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      uint4* o = reinterpret_cast<uint4*>(p.out + qrow * kD);
#pragma unroll 1
      for (int c16 = 0; c16 < kD / 16; ++c16) {
        uint32_t r[16];
        if (have_o) {
          tc::ld_x16(t_lane + kOCol + 16 * c16, r);
          tc::wait_ld();
        }
        uint32_t hv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          hv[i] = have_o ? h2_pack(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv) : 0u;
        if (cvalid) {
          o[2 * c16] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
          o[2 * c16 + 1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
        }
      }
    } else {
      const int GT = p.gt, HGd = p.num_q_heads / p.gt;
      const int sm = cvalid ? p.members[gstart + tok] : 0;
      const int h = kvh * G + gc % G;
      const long long sl = ((long long)sm * HGd + h / GT) * p.splits + split;
      if (cvalid) {
        float* ml = p.pml + (sl * GT + h % GT) * 2;
        ml[0] = m_used == -INFINITY ? -1.0e30f : m_used;
        ml[1] = lsum;
      }
      float4* acc = reinterpret_cast<float4*>(p.pacc + (sl * GT + h % GT) * kD);
#pragma unroll 1
      for (int c16 = 0; c16 < kD / 16; ++c16) {
        uint32_t r[16];
        if (have_o) {
          tc::ld_x16(t_lane + kOCol + 16 * c16, r);
          tc::wait_ld();
        }
        if (cvalid) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            acc[4 * c16 + i] = have_o ? make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                     __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace prefill_tc
}  // namespace pkv
