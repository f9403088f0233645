// gqa_tc.cuh -- paged decode attention for grouped queries on the fifth-generation tensor cores
// (tcgen05, sm_100a): INT8 K with INT8 or INT4 V, head_dim 128, 8 query heads per unit.
//
// What it computes is the decode of decode_kernel.cuh for one (sequence, head group) unit: the
// online-softmax attention of the group's 8 queries over the sequence's blocks (in the
// shared-prefix decode: over the blocks after the shared ones), with the unit's blocks cut into
// splits whose partial states are merged by the last split to finish (the merge of the decode,
// which also folds in the prefix pass's partials). How, per CTA (one split of one unit), in steps
// of 128 tokens (a "chunk"):
//   * S^T = K q^T: tcgen05.mma kind::i8, M = the chunk's 128 tokens, N = 16 (the unit's 8 heads, 8
//     zero rows), K = 32 dims per instruction. A = the int8 K codes exactly as the tiled copy left
//     them (K-major, 128-byte swizzle: no thread touches them); B = q on a 22-bit fixed-point grid
//     per head in three exact signed byte planes. int32 accumulators in tensor memory (two chunk
//     buffers), combined per token into the exact integer dot product (the decode's dp4a scheme);
//   * O^T += V^T P^T: tcgen05.mma kind::f16, M = 128 dims, N = 16 heads, K = 16 tokens. A = the V
//     codes turned into exact fp16 by the consumer threads (INT4: the zero point folded in),
//     MN-major; B = the weights p * scale_V in fp16 high and low parts (p keeps ~22 bits), K-major.
//     The fp32 accumulator stays in tensor memory; a head's column is rescaled in place only when
//     a score exceeds the head's running maximum by more than 2^8.
// Roles (320 threads): a producer warp reads each chunk's block ids and scales ahead of time and
// issues its tiled copies once its stage is free; an MMA warp issues S(c) as soon as chunk c's K
// has landed and P V(c) once the consumers say its operands are written; 8 consumer warps: tensor-
// memory lane = token (scores) = dim (output), the four warps of a part taking 4 of the 8 heads.
// Converted V and the weights have two buffers each; every wait is bounded and gives up when any
// warp has raised the CTA's stop flag.
#pragma once

#include "common.cuh"
#include "decode_kernel.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace pkv {
namespace gqa_tc {

constexpr int kConsumers = 256;             // 8 warps: lane quarter w % 4, heads part w / 4
constexpr int kWarpProd = kConsumers / 32;  // block facts and copies
constexpr int kWarpMma = kWarpProd + 1;     // tensor memory and the MMAs
constexpr int kThreads = kConsumers + 64;
constexpr int kTok = 128;  // tokens per chunk: M of S^T
constexpr int kD = 128;
constexpr int kGT = 8;     // query heads of a unit
constexpr int kHP = 4;     // heads of a consumer part
constexpr int kN = 16;     // N of both MMAs (the unit's heads, padded)
constexpr float kGrowLog2 = 8.f;
constexpr uint32_t kTmemCols = 128;  // S^T of two chunks at [0, 48) and [48, 96); O^T at [96, 112)
constexpr uint32_t kSCols = 48;
constexpr uint32_t kOCol = 96;

template <int VT, int BS>
struct Cfg {
  static constexpr int BPC = kTok / BS;  // blocks per chunk
  static constexpr int K_TILE = BS * kD;
  static constexpr int V_ROW = VT == PKV_INT4_ASYM ? kD / 2 : kD;
  static constexpr int V_TILE = BS * V_ROW;
  static constexpr bool V_SWZ = V_ROW % 128 == 0;
  static constexpr int RAW_V = kTok * kD;  // a raw chunk: K rows, then V rows
  static constexpr int RAW = (RAW_V + kTok * V_ROW + 1023) / 1024 * 1024;
  static constexpr int NS = 3;
  static constexpr int QP = kN * 128;       // one q plane: 16 rows x 128 bytes, 128-byte swizzle
  static constexpr int VH = kTok * kD * 2;  // V fp16, MN-major atoms of 8 tokens x 64 dims
  static constexpr int PB = kN * kTok * 2;  // one part (high or low) of the weights, K-major
  static constexpr int OFF_QP = 0;
  static constexpr int OFF_RAW = 3 * QP;  // 6 KiB
  static constexpr int OFF_VH = OFF_RAW + NS * RAW;
  static constexpr int OFF_P = OFF_VH + 2 * VH;
  static constexpr int OFF_RED = OFF_P + 2 * 2 * PB;          // [2 parts][4 quarters][4 heads] floats
  static constexpr int OFF_QINV = OFF_RED + 2 * 4 * kHP * 4;  // [8] floats
  static constexpr int OFF_META = OFF_QINV + kGT * 4;         // [NS][BPC] block facts
  // full[NS], empty[NS], ready[2], s[2], pv[2], end
  static constexpr int OFF_BAR = (OFF_META + NS * BPC * 16 + 7) / 8 * 8;
  static constexpr int NBAR = 2 * NS + 7;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;  // tensor-memory address, ticket, stop flag
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;    // + alignment slack
  // S^T: M = 128 tokens x N = 16 heads, s8 x s8 -> s32, both K-major
  static constexpr uint32_t ID_S = tc::idesc(2, 1, 1, 0, 0, kTok, kN);
  // O^T: M = 128 dims x N = 16 heads, f16 x f16 -> f32, A MN-major, B K-major
  static constexpr uint32_t ID_PV = tc::idesc(1, 0, 0, 1, 0, kD, kN);
  static_assert(kTok % BS == 0 && K_TILE % 1024 == 0 && RAW % 1024 == 0 && RAW_V % 1024 == 0, "tiles");
  static_assert(OFF_RAW % 1024 == 0 && OFF_VH % 1024 == 0 && OFF_P % 1024 == 0 && PB % 1024 == 0, "atoms");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct BlockFacts {
  int valid;
  float ks, vs, zp;
};

struct GqaSplit {
  int32_t splits;     // splits per unit (grid x)
  int32_t per_split;  // blocks per split, a whole number of chunks
};

__device__ __forceinline__ uint32_t h2_sub_(uint32_t a, uint32_t b) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2_pack_(float lo, float hi) {
  const __half2 r = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&r);
}
// 128-byte swizzle: byte offset of 16-byte unit u of row r inside an 8-row atom
__device__ __forceinline__ int sw(int r, int u) { return (r & 7) * 128 + (((u ^ r) & 7) << 4); }
__device__ __forceinline__ void mbar_arrive_(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
constexpr uint32_t kH2Bias8 = 0x64806480u;  // fp16 1024 + 128
// the four consumer warps of a heads part meet at named barrier 1 + part (with an OR of a flag)
__device__ __forceinline__ void part_sync(int part) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + part) : "memory");
}
__device__ __forceinline__ bool part_sync_or(int part, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %2, 0;\n\tbar.red.or.pred q, %1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(1 + part), "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
// all consumer warps (named barrier 5, plain or with an OR of a flag); the consumers and the MMA
// warp at the end (barrier 6)
__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync 5, %0;" ::"n"(kConsumers) : "memory"); }
__device__ __forceinline__ bool cons_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 5, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kConsumers)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void end_sync() { asm volatile("bar.sync 6, %0;" ::"n"(kConsumers + 32) : "memory"); }
// A bounded wait that also gives up as soon as another warp has raised the stop flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const volatile int* flag) {
  for (uint32_t i = 0; i < kMaxWaitIters; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*flag != 0) return false;
  }
  return false;
}

template <int VT, int BS>
__global__ void __launch_bounds__(kThreads, 1)
    gqa_decode_tc_kernel(const DecodeParams p, const GqaSplit gs, const __grid_constant__ TileMaps tm) {
  using C = Cfg<VT, BS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* const smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hg = blockIdx.y, s = blockIdx.z;
  const int HG = p.num_q_heads / kGT;
  const int kvh = (hg * kGT) / p.group;
  const long long unit = (long long)s * HG + hg;

  // ---- this CTA's blocks ----
  const int cap = min(p.max_context_len, p.max_blocks_per_seq * BS);
  const int raw_len = p.context_lens[s];
  const int L = max(0, min(raw_len, cap));
  const int nb = (L + BS - 1) / BS;
  int sb = 0;
  if (p.shared_blocks != nullptr && L > 0) {
    const int v = p.shared_blocks[s];
    sb = max(0, min(v, min(nb - 1, p.max_shared_blocks)));
    if (sb != v && split == 0 && tid == 0) record_error(p.dev_error, PKV_DEVERR_SHARED);
  }
  if (raw_len != L && split == 0 && hg == 0 && tid == 0) record_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN);
  // (every unit has its own CTAs, so a walk order changes nothing here; its entries are still checked)
  if (p.seq_order != nullptr && split == 0 && hg == 0 && tid == 0) {
    const int a = p.seq_order[s];
    if (a < 0 || a >= p.num_seqs) record_error(p.dev_error, PKV_DEVERR_SEQ_ORDER);
  }
  if (nb == 0) {  // nothing to attend over: the outputs are 0
    if (split == 0)
      for (int e = tid; e < kGT * kD / 8; e += kThreads)
        reinterpret_cast<uint4*>(p.out + ((size_t)s * p.num_q_heads + (size_t)hg * kGT) * kD)[e] =
            make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const int jb = sb + split * gs.per_split;
  if (jb >= nb) return;
  const int je = min(nb, jb + gs.per_split);
  const int n_splits = (nb - sb + gs.per_split - 1) / gs.per_split;  // splits of this unit with blocks
  const int nblk = je - jb;
  const int nch = (nblk + C::BPC - 1) / C::BPC;

  uint8_t* const qp = smem + C::OFF_QP;
  uint8_t* const raw = smem + C::OFF_RAW;
  uint8_t* const vh = smem + C::OFF_VH;
  uint8_t* const pw = smem + C::OFF_P;
  float* const red = reinterpret_cast<float*>(smem + C::OFF_RED);
  float* const qinv_s = reinterpret_cast<float*>(smem + C::OFF_QINV);
  BlockFacts* const meta = reinterpret_cast<BlockFacts*>(smem + C::OFF_META);
  uint64_t* const bar_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // a raw chunk landed (tx)
  uint64_t* const bar_empty = bar_full + C::NS;   // a raw chunk's V converted and K consumed (8 warps)
  uint64_t* const bar_ready = bar_empty + C::NS;  // a chunk's converted V and weights written (8 warps)
  uint64_t* const bar_s = bar_ready + 2;          // S^T of a chunk complete (commit)
  uint64_t* const bar_pv = bar_s + 2;             // O^T += V^T P^T of a chunk complete (commit)
  uint64_t* const bar_end = bar_pv + 2;           // every MMA complete (commit)
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  uint32_t* const ticket = tmem_slot + 1;
  volatile int* const stop = reinterpret_cast<volatile int*>(tmem_slot + 2);
  const int32_t* table = p.block_tables + (size_t)s * p.max_blocks_per_seq + jb;

  // ---- producer warp, lane b < blocks of chunk k: the block's id and facts (read ahead), then
  // its copies once the chunk's stage is free ----
  BlockFacts fb;
  int frow = 0;
  size_t fmi = 0;
  auto fetch = [&](int k) {
    const int nbk = min(C::BPC, nblk - k * C::BPC);
    fb.valid = 0;
    fb.ks = fb.vs = fb.zp = 0.f;
    frow = 0;
    fmi = 0;
    if (lane < nbk) {
      const int rawid = table[k * C::BPC + lane];
      const bool valid = rawid >= 0 && rawid < p.num_blocks;
      if (!valid) record_error(p.dev_error, PKV_DEVERR_BLOCK_ID);
      const size_t mi = (size_t)(valid ? rawid : 0) * p.num_kv_heads + kvh;
      fb.valid = valid ? 1 : 0;
      fb.ks = p.k_scale[mi];
      fb.vs = p.v_scale[mi];
      fb.zp = VT == PKV_INT4_ASYM ? (float)p.v_zp[mi] : 0.f;
      frow = (int)(mi * BS);
      fmi = mi;
    }
  };
  auto publish = [&](int k) {
    const int st = k % C::NS;
    const int nbk = min(C::BPC, nblk - k * C::BPC);
    if (lane < C::BPC) meta[st * C::BPC + lane] = fb;
    __syncwarp();  // the lanes' facts precede lane 0's arrival (release) on the stage's barrier
    if (lane == 0) mbar_arrive_expect_tx(&bar_full[st], (uint32_t)(nbk * (C::K_TILE + C::V_TILE)));
    __syncwarp();
    if (lane < nbk) {
      uint8_t* dst = raw + st * C::RAW;
      tma_load_2d(dst + lane * C::K_TILE, &tm.k, 0, frow, &bar_full[st]);
      if constexpr (C::V_SWZ) {
        tma_load_2d(dst + C::RAW_V + lane * C::V_TILE, &tm.v, 0, frow, &bar_full[st]);
      } else {
        bulk_g2s(dst + C::RAW_V + lane * C::V_TILE, static_cast<const uint8_t*>(p.v_codes) + fmi * C::V_TILE,
                 (uint32_t)C::V_TILE, &bar_full[st]);
      }
    }
  };
  int produced = 0;
  if (warp == kWarpMma) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == kWarpProd) {
    if (lane == 0) {
      for (int i = 0; i < C::NBAR; ++i) {
        const bool per_warp = i >= C::NS && i < 2 * C::NS + 2;  // empty and ready: one arrival per consumer warp
        mbar_init(&bar_full[i], per_warp ? (uint32_t)(kConsumers / 32) : 1u);
      }
      *stop = 0;
      fence_mbar_init();
    }
    __syncwarp();
    for (; produced < min(C::NS, nch); ++produced) {
      fetch(produced);
      publish(produced);
    }
  }

  // ---- consumers: q on a 22-bit fixed-point grid per head, three signed byte planes (B of S^T;
  // rows 8-15 zero), warp w the rows 2w and 2w+1; the weights start at zero ----
  if (warp < kConsumers / 32) {
    for (int hh = 0; hh < 2; ++hh) {
      const int h = 2 * warp + hh;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (h < kGT) {
        const uint2 w2 = *reinterpret_cast<const uint2*>(
            p.q + ((size_t)s * p.num_q_heads + (size_t)hg * kGT + h) * kD + 4 * lane);
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w2.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&w2.y));
        x[0] = a.x;
        x[1] = a.y;
        x[2] = b.x;
        x[3] = b.y;
      }
      float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      int ex = 0;
      (void)frexpf(amax, &ex);
      const int shift = amax > 0.f ? 22 - ex : 0;
      const float up = __int_as_float((127 + shift) << 23);
      uint32_t pl[3] = {0u, 0u, 0u};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int qi = __float2int_rn(x[k] * up);
        const int b0 = ((qi + 128) & 0xFF) - 128;
        const int r1 = (qi - b0) >> 8;
        const int b1 = ((r1 + 128) & 0xFF) - 128;
        const int b2 = (r1 - b1) >> 8;
        pl[0] |= (uint32_t)(b0 & 0xFF) << (8 * k);
        pl[1] |= (uint32_t)(b1 & 0xFF) << (8 * k);
        pl[2] |= (uint32_t)(b2 & 0xFF) << (8 * k);
      }
      const int d = 4 * lane;  // dims d .. d+3 of row h
#pragma unroll
      for (int k = 0; k < 3; ++k)
        *reinterpret_cast<uint32_t*>(qp + k * C::QP + (h >> 3) * 1024 + sw(h, d >> 4) + (d & 15)) = pl[k];
      if (h < kGT && lane == 0) qinv_s[h] = __int_as_float((127 - shift) << 23);
    }
    for (int e = tid; e < 2 * 2 * C::PB / 16; e += kConsumers)
      reinterpret_cast<uint4*>(pw)[e] = make_uint4(0u, 0u, 0u, 0u);
    tc::fence_proxy_async_smem();  // read by the tensor core
  }
  tc::fence_before_sync();
  __syncthreads();  // barriers initialised, tensor memory allocated, q laid out
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpProd) {
    for (; produced < nch; ++produced) {
      fetch(produced);
      const int st = produced % C::NS;
      const bool pok = wait_or_abort(&bar_empty[st], (uint32_t)(((produced / C::NS) - 1) & 1), stop);
      if (!__all_sync(0xffffffffu, pok)) break;
      publish(produced);
    }
    // the copies issued last have landed before this warp leaves (those before them were consumed)
    if (lane == 0)
      for (int j = max(0, produced - C::NS); j < produced; ++j)
        (void)mbar_wait_bounded(&bar_full[j % C::NS], (uint32_t)((j / C::NS) & 1));
    return;
  }

  if (warp == kWarpMma) {
    if (lane == 0) {
      const uint64_t dq = tc::smem_desc(smem_addr(qp), 16, 1024, tc::kLayoutSw128);
      const uint64_t dk = tc::smem_desc(smem_addr(raw), 16, 1024, tc::kLayoutSw128);
      const uint64_t dvh = tc::smem_desc(smem_addr(vh), 1024, 2048, tc::kLayoutSw128);
      const uint64_t dpw = tc::smem_desc(smem_addr(pw), 16, 1024, tc::kLayoutSw128);
      bool mok = true;
      for (int c = 0; c <= nch && mok; ++c) {
        if (c < nch) {  // S^T(c) as soon as its K has landed (its tensor-memory buffer was read before ready(c-2))
          const int st = c % C::NS;
          mok = wait_or_abort(&bar_full[st], (uint32_t)((c / C::NS) & 1), stop);
          if (!mok) break;
          tc::fence_after_sync();
#pragma unroll
          for (int pl = 0; pl < 3; ++pl)
#pragma unroll
            for (int kk = 0; kk < kD / 32; ++kk)
              tc::mma_i8(tmem + (uint32_t)((c & 1) * kSCols + pl * kN),
                         dk + (uint64_t)((st * C::RAW + kk * 32) >> 4), dq + (uint64_t)((pl * C::QP + kk * 32) >> 4),
                         C::ID_S, kk > 0 ? 1u : 0u);
          tc::commit(&bar_s[c & 1]);
        }
        if (c >= 1) {  // O^T += V^T P^T of chunk c-1 once its operands are written
          const int pc = c - 1;
          mok = wait_or_abort(&bar_ready[pc & 1], (uint32_t)((pc >> 1) & 1), stop);
          if (!mok) break;
          tc::fence_after_sync();
#pragma unroll
          for (int ks = 0; ks < kTok / 16; ++ks) {
            const uint64_t ad = dvh + (uint64_t)(((pc & 1) * C::VH + ks * 4096) >> 4);
            const uint64_t bd = dpw + (uint64_t)(((pc & 1) * 2 * C::PB + (ks >> 2) * 2048 + (ks & 3) * 32) >> 4);
            tc::mma_f16(tmem + kOCol, ad, bd, C::ID_PV, (pc > 0 || ks > 0) ? 1u : 0u);
            tc::mma_f16(tmem + kOCol, ad, bd + (uint64_t)(C::PB >> 4), C::ID_PV, 1u);
          }
          tc::commit(&bar_pv[pc & 1]);
        }
      }
      if (!mok && *stop == 0) {  // a wait of this warp ran out: stop everyone
        record_error(p.dev_error, PKV_DEVERR_TIMEOUT);
        *stop = 1;
      }
      tc::commit(bar_end);
    }
    __syncwarp();
    (void)mbar_wait_bounded(bar_end, 0u);
    tc::fence_before_sync();
    end_sync();  // the consumers' last tensor-memory reads are done
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
    return;
  }

  // ---- consumer warps ----
  const int q4 = warp & 3, part = warp >> 2;
  const int row = q4 * 32 + lane;  // tensor-memory lane: this thread's token (S^T), its dim (O^T)
  const uint32_t t_lane = tmem + ((uint32_t)(q4 * 32) << 16);
  float qinv[kHP];
#pragma unroll
  for (int j = 0; j < kHP; ++j) qinv[j] = qinv_s[kHP * part + j];
  bool ok = true;
  auto fail = [&]() {
    if (*stop == 0) {
      record_error(p.dev_error, PKV_DEVERR_TIMEOUT);
      *stop = 1;
    }
    ok = false;
  };
  auto warp_arrive = [&](uint64_t* bar) {
    __syncwarp();
    if (lane == 0) mbar_arrive_(bar);
  };
  float m_used[kHP], lsum[kHP];
#pragma unroll
  for (int j = 0; j < kHP; ++j) {
    m_used[j] = -INFINITY;
    lsum[j] = 0.f;
  }
  for (int c = 0; c < nch; ++c) {
    const int st = c % C::NS;
    if (ok && !wait_or_abort(&bar_full[st], (uint32_t)((c / C::NS) & 1), stop)) fail();
    // P V(c-2) done: its V and weight buffers take chunk c
    if (c >= 2 && ok && !wait_or_abort(&bar_pv[c & 1], (uint32_t)(((c - 2) >> 1) & 1), stop)) fail();
    // ---- V of the chunk -> exact fp16 ----
    if (ok) {
      const uint8_t* rs = raw + st * C::RAW;
      const BlockFacts* mt = meta + st * C::BPC;
      uint8_t* vd = vh + (c & 1) * C::VH;
#pragma unroll 4
      for (int k = 0; k < kTok * 16 / kConsumers; ++k) {  // 128 tokens x 16 units of 8 dims
        const int e = tid + kConsumers * k;
        const int tk = e >> 4, u = e & 15;
        uint32_t h[4];
        if constexpr (VT == PKV_INT4_ASYM) {
          const float zp = mt[tk / BS].zp;
          const uint32_t zb = h2_pack_(1024.f + zp, 1024.f + zp);
          const uint32_t x = *reinterpret_cast<const uint32_t*>(rs + C::RAW_V + tk * C::V_ROW + 4 * u);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t t = x >> (8 * b);
            h[b] = h2_sub_((t & 0xFu) | ((t << 12) & 0xF0000u) | 0x64006400u, zb);
          }
        } else {
          const uint2 x =
              *reinterpret_cast<const uint2*>(rs + C::RAW_V + tk * 128 + ((((u >> 1) ^ tk) & 7) << 4) + ((u & 1) << 3));
          const uint32_t u0 = x.x ^ 0x80808080u, u1 = x.y ^ 0x80808080u;
          h[0] = h2_sub_(__byte_perm(u0, 0x64646464u, 0x5140), kH2Bias8);
          h[1] = h2_sub_(__byte_perm(u0, 0x64646464u, 0x5342), kH2Bias8);
          h[2] = h2_sub_(__byte_perm(u1, 0x64646464u, 0x5140), kH2Bias8);
          h[3] = h2_sub_(__byte_perm(u1, 0x64646464u, 0x5342), kH2Bias8);
        }
        *reinterpret_cast<uint4*>(vd + (tk >> 3) * 2048 + (u >> 3) * 1024 + sw(tk, u)) =
            make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
    tc::fence_proxy_async_smem();
    // ---- this thread's token: its scores for the part's 4 heads ----
    const BlockFacts bm = meta[st * C::BPC + row / BS];  // (read before the stage is handed back)
    const int pos = (jb + c * C::BPC) * BS + row;
    const bool in = bm.valid && (c * C::BPC + row / BS) < nblk && pos < L;
    if (ok && !wait_or_abort(&bar_s[c & 1], (uint32_t)((c >> 1) & 1), stop)) fail();
    tc::fence_after_sync();
    uint32_t s0[4], s1[4], s2[4];
    const uint32_t sbase = t_lane + (uint32_t)((c & 1) * kSCols + kHP * part);
    tc::ld_x4(sbase + 0 * kN, s0);
    tc::ld_x4(sbase + 1 * kN, s1);
    tc::ld_x4(sbase + 2 * kN, s2);
    tc::wait_ld();
    tc::fence_before_sync();
    warp_arrive(&bar_empty[st]);  // this warp's V converted and its scores read: the stage may be refilled
    float z[kHP];
    bool need = false;
    const float fz = bm.ks * p.scale_log2;
#pragma unroll
    for (int j = 0; j < kHP; ++j) {
      const float rs_ = __fmaf_rn((float)(int)s2[j], 65536.f, (float)((int)s1[j] * 256 + (int)s0[j]));
      z[j] = in ? rs_ * (qinv[j] * fz) : -INFINITY;
      need = need || z[j] > m_used[j] + kGrowLog2;
    }
    // the part's four warps agree on a stop, then on a score beyond a running maximum (then the
    // chunk's maxima are taken)
    float* rb = red + part * 4 * kHP;
    if (part_sync_or(part, !ok || *stop != 0)) {
      ok = false;
      break;
    }
    const bool any_need = part_sync_or(part, need);
    if (any_need) {
#pragma unroll
      for (int j = 0; j < kHP; ++j) {
        float mx = z[j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) rb[q4 * kHP + j] = mx;
      }
      part_sync(part);
      float al[kHP];
      bool rescale = false;
#pragma unroll
      for (int j = 0; j < kHP; ++j) {
        const float cm = fmaxf(fmaxf(rb[j], rb[kHP + j]), fmaxf(rb[2 * kHP + j], rb[3 * kHP + j]));
        al[j] = 1.f;
        if (cm > m_used[j] + kGrowLog2) {  // (-inf + 8 is -inf: the first visible chunk sets it)
          al[j] = m_used[j] == -INFINITY ? 0.f : ex2(m_used[j] - cm);
          m_used[j] = cm;
          lsum[j] *= al[j];
          rescale = rescale || c > 0;
        }
      }
      part_sync(part);  // the maxima are read before the buffer is written again
      if (rescale) {    // (the part's decision) its heads' columns of O^T, this thread's dim, once P V(c-1) is done
        if (ok && !wait_or_abort(&bar_pv[(c - 1) & 1], (uint32_t)(((c - 1) >> 1) & 1), stop)) fail();
        tc::fence_after_sync();
        uint32_t r[4];
        tc::ld_x4(t_lane + kOCol + (uint32_t)(kHP * part), r);
        tc::wait_ld();
#pragma unroll
        for (int j = 0; j < kHP; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * al[j]);
        tc::st_x4(t_lane + kOCol + (uint32_t)(kHP * part), r);
        tc::wait_st();
      }
    }
    // ---- weights, V scale folded in, fp16 high and low parts: rows 4 part + j of P^T, this token ----
    {
      uint8_t* pb = pw + (c & 1) * 2 * C::PB;
      const int off = (row >> 6) * 2048 + (((row & 63) >> 3) << 4) + (row & 7) * 2;
#pragma unroll
      for (int j = 0; j < kHP; ++j) {
        const int h = kHP * part + j;
        const float w = (in && m_used[j] != -INFINITY) ? ex2(z[j] - m_used[j]) : 0.f;
        lsum[j] += w;
        const float v = w * bm.vs;
        const __half hi = __float2half_rn(v);
        const __half lo = __float2half_rn(v - __half2float(hi));
        const int a = h * 128 + (off ^ ((h & 7) << 4));  // the row's swizzle of the 16-byte unit
        *reinterpret_cast<__half*>(pb + a) = hi;
        *reinterpret_cast<__half*>(pb + C::PB + a) = lo;
      }
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();  // the rescale's tensor-memory stores precede P V(c)
    warp_arrive(&bar_ready[c & 1]);
  }

  // ---- every MMA issued has completed (the MMA warp commits once it has stopped) ----
  const bool done = mbar_wait_bounded(bar_end, 0u);
  ok = ok && done && *stop == 0;
  tc::fence_after_sync();
  // the part's heads' total weights over the CTA's tokens
  float* rb = red + part * 4 * kHP;
#pragma unroll
  for (int j = 0; j < kHP; ++j) {
    float v = lsum[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) rb[q4 * kHP + j] = v;
  }
  cons_sync();
  const int n_pref = sb > 0 ? p.prefix_splits : 0;
  const bool direct = n_splits == 1 && n_pref == 0;
  if (ok) {
    float l[kHP];
#pragma unroll
    for (int j = 0; j < kHP; ++j) l[j] = (rb[j] + rb[kHP + j]) + (rb[2 * kHP + j] + rb[3 * kHP + j]);
    uint32_t r[4];
    tc::ld_x4(t_lane + kOCol + (uint32_t)(kHP * part), r);  // O^T[dim row][heads of the part]
    tc::wait_ld();
    const int d = row;
    if (direct) {
#pragma unroll
      for (int j = 0; j < kHP; ++j) {
        const float inv = l[j] > 0.f ? 1.f / l[j] : 0.f;
        p.out[((size_t)s * p.num_q_heads + (size_t)hg * kGT + kHP * part + j) * kD + d] =
            __float2half_rn(__uint_as_float(r[j]) * inv);
      }
    } else {
      // this split's partial of the unit (the merge's layout: slot, head, dim)
      const long long slot = unit * gs.splits + split;
#pragma unroll
      for (int j = 0; j < kHP; ++j)
        p.ws_acc[((size_t)slot * kGT + kHP * part + j) * kD + d] = __uint_as_float(r[j]);
      if (q4 == 0 && lane < kHP) {
        const int j = lane;
        p.ws_ml[((size_t)slot * kGT + kHP * part + j) * 2 + 0] = m_used[j] == -INFINITY ? kNegBig : m_used[j];
        p.ws_ml[((size_t)slot * kGT + kHP * part + j) * 2 + 1] = l[j];
      }
    }
  }
  // every consumer's part of the partial precedes the ticket; the last split of the unit merges
  // (the decision is the same for every consumer: a stop anywhere skips the ticket and the merge)
  const bool bad = cons_sync_or(!ok);
  if (!bad && !direct) {
    if (tid == 0) {
      fence_acq_rel_gpu();
      *ticket = atomic_inc_relaxed_gpu(&p.ws_count[unit], (uint32_t)n_splits - 1u);
    }
    cons_sync();
    if (*ticket == (uint32_t)n_splits - 1u && warp == 0) {
      if (lane == 0) fence_acq_rel_gpu();
      __syncwarp();
      merge_partials<kGT, kD>(p, unit * gs.splits, n_splits, unit * p.prefix_splits, n_pref, s, hg, lane);
    }
  }
  tc::fence_before_sync();
  end_sync();  // then the MMA warp frees the tensor memory
}

}  // namespace gqa_tc
}  // namespace pkv
