// prefill_tc.cuh -- multi-query paged attention on the fifth-generation tensor cores (tcgen05):
// chunked prefill and the shared-prefix pass of the decode (sm_100a).
//
// What it computes is what prefill_kernel.cuh states (the same work split per CTA: 128 query
// columns of one KV head, a range of blocks of one block table, causal limits for a prefill,
// partial softmax states for the shared-prefix pass). How:
//   * the CTA's 128 columns are the M = 128 rows of every MMA; the blocks are taken 64 tokens (a
//     "chunk": 4 blocks of 16 or 2 of 32) at a time, the N of S = Q K^T and the K of O += P V;
//   * 16 consumer warps: column `col` is tensor-memory lane `col`, served by the four warps of
//     its lane quarter (w % 4), each taking 16 of the chunk's tokens (and 32 dims of O), so a
//     column's softmax needs one exchange of a number among the four warps and no shuffles; a
//     producer warp reads each chunk's block ids and scales ahead of time and issues its copies
//     once its stage is free (full / empty mbarriers); an MMA warp owns tensor memory and issues
//     every MMA when the consumers' mbarrier arrivals say its operands are written;
//   * the tiled copies bring the chunk's int8 K rows and int8 / packed int4 V rows; the threads
//     turn both into exact fp16 (K: the code; V: code - zero point) in the 128-byte-swizzled
//     layouts the MMAs read (K K-major, V MN-major); q is fp16 already and is laid out once;
//   * S = Q K^T: tcgen05.mma kind::f16 (fp16 q times exact codes, fp32 accumulation), two chunk
//     buffers in tensor memory, so S of the next chunk runs on the tensor core while the threads
//     work on this one;
//   * O += P V: the weights p * scale_V split into fp16 high and low parts (p keeps ~22 bits), two
//     MMAs per 16 tokens; the fp32 accumulator stays in tensor memory for the whole block range and
//     is rescaled in place only when a column's running maximum grows by more than 2^8.
// Roles: 16 consumer warps (conversion, softmax, weights, output), a producer warp (block facts,
// copies) and an MMA warp (tensor memory, every MMA). One chunk c, every consumer thread: convert
// chunk c+1 and arrive on "converted", wait S(c), softmax of c, weights of c and arrive on
// "weights written". The MMA warp issues S(c+1) after "converted" (and hands the raw stage back to
// the producer), P V(c) after "weights written". Converted V has three buffers and the weights
// two, so neither is overwritten while a product may still read it; S has two tensor-memory
// buffers, so S(c+1) runs while the consumers work on chunk c.
// MMA completion is tracked with tcgen05.commit on mbarriers; every wait is bounded.
#pragma once

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace pkv {
namespace prefill_tc {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kT = 64;                      // tokens per chunk
constexpr int kParts = 4;                   // consumer warps per tensor-memory lane quarter
constexpr int kTokPart = kT / kParts;       // a consumer warp's tokens of a chunk (softmax)
constexpr int kDimPart = 128 / kParts;      // ... and its dims of O (rescale, output)
constexpr int kConsumers = 128 * kParts;
constexpr int kWarpProd = kConsumers / 32;  // block facts and copies
constexpr int kWarpMma = kWarpProd + 1;     // tensor memory and the MMAs
constexpr int kThreads = kConsumers + 64;
constexpr int kCols = 128;
constexpr int kD = 128;
constexpr float kGrowLog2 = 8.f;
constexpr uint32_t kTmemCols = 256;  // S of two chunks at columns [0, 64) and [64, 128); O at [128, 256)
constexpr uint32_t kOCol = 128;

template <int VT, int BS>
struct Cfg {
  static constexpr int BPC = kT / BS;  // blocks per chunk
  static constexpr int K_ROW = kD;
  static constexpr int V_ROW = VT == PKV_INT4_ASYM ? kD / 2 : kD;
  static constexpr int K_TILE = BS * K_ROW, V_TILE = BS * V_ROW;  // one (block, KV head) tile
  static constexpr bool V_SWZ = V_ROW % 128 == 0;                 // INT8 V: tiled, swizzled copy
  static constexpr int RAW_V = kT * K_ROW;                        // a raw chunk: K rows, then V rows
  static constexpr int RAW = (RAW_V + kT * V_ROW + 1023) / 1024 * 1024;
  static constexpr int NS = 2;                // raw chunk stages
  static constexpr int QB = 2 * kCols * 128;  // q fp16: two 64-dim atom columns of 128 rows x 128 B
  static constexpr int KB = 2 * kT * 128;     // converted K chunk: two atom columns of 64 rows
  static constexpr int VB = kT * kD * 2;      // converted V chunk: 8 token groups x 2 dim atoms
  static constexpr int PB = kCols * kT * 2;   // one part (high or low) of a chunk's weights
  static constexpr int NVB = 3;
  static constexpr int NMETA = 4;  // chunk slots of per-block facts
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RAW = OFF_Q + QB;
  static constexpr int OFF_K = OFF_RAW + NS * RAW;
  static constexpr int OFF_V = OFF_K + 2 * KB;
  static constexpr int OFF_P = OFF_V + NVB * VB;
  static constexpr int OFF_RED = OFF_P + 2 * 2 * PB;  // [2 uses][kParts][128 columns] floats
  static constexpr int OFF_META = OFF_RED + 2 * kParts * kCols * 4;
  // full[NS], empty[NS], conv[2], pdone[2], s[2], pv[2], end
  static constexpr int OFF_BAR = OFF_META + NMETA * BPC * 16;
  static constexpr int OFF_TMEM = OFF_BAR + (2 * NS + 9) * 8;  // tensor-memory address, stop flag
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;  // + alignment slack
  // S: M = 128 columns x N = 64 tokens, f16 x f16 -> f32, both K-major
  static constexpr uint32_t ID_S = tc::idesc(1, 0, 0, 0, 0, kCols, kT);
  // PV: M = 128 columns x N = 128 dims, f16 x f16 -> f32, A K-major, B MN-major
  static constexpr uint32_t ID_PV = tc::idesc(1, 0, 0, 0, 1, kCols, kD);
  static_assert(kT % BS == 0 && BS % kTokPart == 0, "whole blocks per chunk, a warp's tokens in one block");
  static_assert(OFF_RAW % 1024 == 0 && RAW % 1024 == 0 && RAW_V % 1024 == 0 && K_TILE % 1024 == 0, "tiled copies");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_P % 1024 == 0 && PB % 1024 == 0, "swizzle atoms");
  static_assert(OFF_BAR % 8 == 0, "mbarriers");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct BlockMeta {
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
// fp16 1024 + 128: subtracted from 0x64XX (= 1024 + XX) where XX is a code biased by +128
constexpr uint32_t kH2Bias8 = 0x64806480u;
// 8 int8 codes (two words) -> 4 half2 of their exact values
__device__ __forceinline__ void s8x8_to_h2(uint2 x, uint32_t (&h)[4]) {
  const uint32_t u0 = x.x ^ 0x80808080u, u1 = x.y ^ 0x80808080u;
  h[0] = h2_sub(__byte_perm(u0, 0x64646464u, 0x5140), kH2Bias8);
  h[1] = h2_sub(__byte_perm(u0, 0x64646464u, 0x5342), kH2Bias8);
  h[2] = h2_sub(__byte_perm(u1, 0x64646464u, 0x5140), kH2Bias8);
  h[3] = h2_sub(__byte_perm(u1, 0x64646464u, 0x5342), kH2Bias8);
}
// the kParts warps serving the same 32 columns (w % 4 == q4) meet at named barrier 1 + q4
__device__ __forceinline__ void quarter_sync(int q4) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + q4), "n"(32 * kParts) : "memory");
}
// ... and the OR of a flag over them
__device__ __forceinline__ bool quarter_sync_or(int q4, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %2, 0;\n\tbar.red.or.pred q, %1, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(1 + q4), "r"((uint32_t)v), "n"(32 * kParts)
      : "memory");
  return r != 0;
}
// the consumer warps and the MMA warp meet once at the end (named barrier 5)
__device__ __forceinline__ void end_sync() { asm volatile("bar.sync 5, %0;" ::"n"(kConsumers + 32) : "memory"); }
// A bounded wait that also gives up as soon as another warp has raised the stop flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const volatile int* flag) {
  for (uint32_t i = 0; i < kMaxWaitIters; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*flag != 0) return false;
  }
  return false;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// 128-byte swizzle: byte offset of 16-byte unit u of row r inside an 8-row atom
__device__ __forceinline__ int sw(int r, int u) { return (r & 7) * 128 + (((u ^ r) & 7) << 4); }

}  // namespace

template <int VT, int BS, bool PREFIX>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_tc_kernel(const PrefillParams p, const __grid_constant__ TileMaps tm) {
  using C = Cfg<VT, BS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* const smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, part = warp >> 2;  // (consumer warps)
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
        for (int e = tid; e < ncols * (kD / 8); e += kThreads) {
          const int gc = col0 + e / (kD / 8);
          uint4* o =
              reinterpret_cast<uint4*>(p.out + ((size_t)(q0 + gc / G) * p.num_q_heads + (size_t)kvh * G + gc % G) * kD);
          o[e % (kD / 8)] = make_uint4(0u, 0u, 0u, 0u);
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
  const int nch = (nblk + C::BPC - 1) / C::BPC;

  uint8_t* const qsm = smem + C::OFF_Q;
  uint8_t* const raw = smem + C::OFF_RAW;
  uint8_t* const ksm = smem + C::OFF_K;
  uint8_t* const vsm = smem + C::OFF_V;
  uint8_t* const psm = smem + C::OFF_P;
  float* const red = reinterpret_cast<float*>(smem + C::OFF_RED);
  BlockMeta* const meta = reinterpret_cast<BlockMeta*>(smem + C::OFF_META);
  uint64_t* const bar_full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // a raw chunk landed (tx)
  uint64_t* const bar_empty = bar_full + C::NS;   // a raw chunk converted (MMA warp)
  uint64_t* const bar_conv = bar_empty + C::NS;   // converted K / V of a chunk written (consumer warps)
  uint64_t* const bar_pdone = bar_conv + 2;       // weights of a chunk written (consumer warps)
  uint64_t* const bar_s = bar_pdone + 2;          // S of a chunk complete (commit)
  uint64_t* const bar_pv = bar_s + 2;             // P V of a chunk complete (commit)
  uint64_t* const bar_end = bar_pv + 2;           // every product complete (commit)
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_TMEM + 4);
  const int32_t* table = p.block_tables + (size_t)s_tab * p.max_blocks_per_seq + jb;

  // ---- producer warp: each lane owns one block of a chunk; the block ids and scales are read
  // before the stage is free, then the facts are published and the copies issued ----
  int produced = 0;
  BlockMeta pm;     // this lane's block of chunk `produced`
  int prow = 0;     // its first row in the K / V code arrays (tiled copies)
  size_t pmi = 0;   // its (block, KV head) tile
  auto fetch = [&](int k) {  // global reads for chunk k (lane < blocks of the chunk)
    const int nb = min(C::BPC, nblk - k * C::BPC);
    pm.valid = 0;
    pm.ks = pm.vs = pm.zp = 0.f;
    prow = 0;
    pmi = 0;
    if (lane < nb) {
      const int rawid = table[k * C::BPC + lane];
      const bool valid = rawid >= 0 && rawid < p.num_blocks;
      if (!valid) record_error(p.dev_error, PKV_DEVERR_BLOCK_ID);
      const size_t mi = (size_t)(valid ? rawid : 0) * p.num_kv_heads + kvh;
      pm.valid = valid ? 1 : 0;
      pm.ks = p.k_scale[mi];
      pm.vs = p.v_scale[mi];
      pm.zp = VT == PKV_INT4_ASYM ? (float)p.v_zp[mi] : 0.f;
      prow = (int)(mi * BS);
      pmi = mi;
    }
  };
  auto publish = [&](int k) {  // the stage of chunk k is free: facts, then the copies
    const int st = k % C::NS;
    const int nb = min(C::BPC, nblk - k * C::BPC);
    if (lane < C::BPC) meta[(k % C::NMETA) * C::BPC + lane] = pm;
    __syncwarp();  // the lanes' facts precede lane 0's arrival (release) on the stage's barrier
    if (lane == 0) mbar_arrive_expect_tx(&bar_full[st], (uint32_t)(nb * (C::K_TILE + C::V_TILE)));
    __syncwarp();
    if (lane < nb) {
      uint8_t* dst = raw + st * C::RAW;
      tma_load_2d(dst + lane * C::K_TILE, &tm.k, 0, prow, &bar_full[st]);
      if constexpr (C::V_SWZ) {
        tma_load_2d(dst + C::RAW_V + lane * C::V_TILE, &tm.v, 0, prow, &bar_full[st]);
      } else {
        bulk_g2s(dst + C::RAW_V + lane * C::V_TILE, static_cast<const uint8_t*>(p.v_codes) + pmi * C::V_TILE,
                 (uint32_t)C::V_TILE, &bar_full[st]);
      }
    }
  };

  if (warp == kWarpMma) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == kWarpProd) {
    if (lane == 0) {
      for (int i = 0; i < 2 * C::NS + 9; ++i)  // conv and pdone take one arrival per consumer warp
        mbar_init(&bar_full[i], (i >= 2 * C::NS && i < 2 * C::NS + 4) ? (uint32_t)(kConsumers / 32) : 1u);
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncwarp();
    for (; produced < min(C::NS, nch); ++produced) {  // the first stages are free
      fetch(produced);
      publish(produced);
    }
  }

  // ---- q (fp16) -> the A operand of S: K-major, 128-byte swizzle, two 64-dim atom columns ----
  auto q_row_of = [&](int c, bool& okc) -> size_t {  // row of q for column c of this CTA
    const int gc = col0 + c;
    okc = c < ncols;
    if constexpr (!PREFIX) {
      return (size_t)(q0 + gc / G) * p.num_q_heads + (size_t)kvh * G + gc % G;
    } else {
      const int sm = okc ? p.members[gstart + gc / G] : -1;
      okc = okc && sm >= 0 && sm < p.num_seqs;
      return (size_t)max(sm, 0) * p.num_q_heads + (size_t)kvh * G + gc % G;
    }
  };
  if (tid < kConsumers) {
#pragma unroll 1
    for (int e = tid; e < kCols * (kD / 8); e += kConsumers) {
      const int c = e >> 4, u = e & 15;  // column, 8-dim unit
      bool okc;
      const size_t r = q_row_of(c, okc);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (okc) v = reinterpret_cast<const uint4*>(p.q + r * kD)[u];
      *reinterpret_cast<uint4*>(qsm + (u >> 3) * (kCols * 128) + (c >> 3) * 1024 + sw(c, u)) = v;
    }
    tc::fence_proxy_async_smem();  // q is read by the tensor core
  }
  tc::fence_before_sync();
  __syncthreads();  // barriers initialised, tensor memory allocated, q laid out
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpProd) {
    // the remaining chunks, each once the chunk NS before it has been converted
    for (; produced < nch; ++produced) {
      fetch(produced);
      const int st = produced % C::NS;
      bool pok = wait_or_abort(&bar_empty[st], (uint32_t)(((produced / C::NS) - 1) & 1), abort_flag);
      if (!__all_sync(kFull, pok)) break;
      publish(produced);
    }
    // the copies issued last have landed before this warp leaves (those before them were
    // consumed; no later chunk shares their stages' phases)
    if (lane == 0)
      for (int j = max(0, produced - C::NS); j < produced; ++j)
        (void)mbar_wait_bounded(&bar_full[j % C::NS], (uint32_t)((j / C::NS) & 1));
    return;
  }

  if (warp == kWarpMma) {
    // ---- MMA warp: S(c) once chunk c is converted, P V(c-1) once its weights are written ----
    if (lane == 0) {
      const uint64_t dq = tc::smem_desc(smem_addr(qsm), 16, 1024, tc::kLayoutSw128);
      const uint64_t dk = tc::smem_desc(smem_addr(ksm), 16, 1024, tc::kLayoutSw128);
      const uint64_t dp = tc::smem_desc(smem_addr(psm), 16, 1024, tc::kLayoutSw128);
      const uint64_t dv = tc::smem_desc(smem_addr(vsm), 1024, 2048, tc::kLayoutSw128);
      bool mok = true;
      for (int c = 0; c <= nch; ++c) {
        if (c < nch) {
          mok = wait_or_abort(&bar_conv[c & 1], (uint32_t)((c >> 1) & 1), abort_flag);
          if (!mok) break;
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)  // (descriptor start fields advance in 16-byte units)
            tc::mma_f16(tmem + (uint32_t)((c & 1) * kT), dq + (uint64_t)(((kk >> 2) * (kCols * 128) + (kk & 3) * 32) >> 4),
                        dk + (uint64_t)(((c & 1) * C::KB + (kk >> 2) * (kT * 128) + (kk & 3) * 32) >> 4), C::ID_S,
                        kk > 0 ? 1u : 0u);
          tc::commit(&bar_s[c & 1]);
          mbar_arrive(&bar_empty[c % C::NS]);  // chunk c's raw stage may be refilled
        }
        if (c >= 1) {
          const int pc = c - 1;
          mok = wait_or_abort(&bar_pdone[pc & 1], (uint32_t)((pc >> 1) & 1), abort_flag);
          if (!mok) break;
          tc::fence_after_sync();
#pragma unroll
          for (int ks = 0; ks < kT / 16; ++ks) {
            const uint64_t bd = dv + (uint64_t)(((pc % C::NVB) * C::VB + ks * 4096) >> 4);
            const uint64_t ad = dp + (uint64_t)(((pc & 1) * 2 * C::PB + ks * 32) >> 4);
            tc::mma_f16(tmem + kOCol, ad, bd, C::ID_PV, (pc > 0 || ks > 0) ? 1u : 0u);
            tc::mma_f16(tmem + kOCol, ad + (uint64_t)(C::PB >> 4), bd, C::ID_PV, 1u);
          }
          tc::commit(&bar_pv[pc & 1]);
        }
      }
      if (!mok && *abort_flag == 0) {  // a wait of this warp ran out: stop everyone
        record_error(p.dev_error, PKV_DEVERR_TIMEOUT);
        *abort_flag = 1;
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
  // this thread's column: tensor-memory lane q4 * 32 + lane; its part of each chunk: tokens
  // [part * kTokPart, +kTokPart) for the softmax, dims [part * kDimPart, +kDimPart) of O
  const int col = q4 * 32 + lane;
  bool cvalid;
  const size_t qrow = q_row_of(col, cvalid);
  const int tok = (col0 + col) / G;
  const int lim = !cvalid ? 0 : (PREFIX ? INT_MAX : pos0 + tok + 1);

  // chunk c (its raw stage has landed) -> converted K buffer c % 2, V buffer c % 3
  auto convert = [&](int c) {
    const uint8_t* rs = raw + (c % C::NS) * C::RAW;
    uint8_t* kd = ksm + (c & 1) * C::KB;
    uint8_t* vd = vsm + (c % C::NVB) * C::VB;
#pragma unroll
    for (int k = 0; k < kT * 16 / kConsumers; ++k) {  // K: 64 rows x 16 units of 8 codes
      const int e = tid + kConsumers * k;
      const int r = e >> 4, u = e & 15;
      const uint2 x = *reinterpret_cast<const uint2*>(rs + r * 128 + ((((u >> 1) ^ r) & 7) << 4) + ((u & 1) << 3));
      uint32_t h[4];
      s8x8_to_h2(x, h);
      *reinterpret_cast<uint4*>(kd + (u >> 3) * (kT * 128) + (r >> 3) * 1024 + sw(r, u)) =
          make_uint4(h[0], h[1], h[2], h[3]);
    }
    const BlockMeta* mt = meta + (c % C::NMETA) * C::BPC;
#pragma unroll
    for (int k = 0; k < kT * 16 / kConsumers; ++k) {  // V: 64 tokens x 16 units of 8 dims
      const int e = tid + kConsumers * k;
      const int tk = e >> 4, u = e & 15;
      uint32_t h[4];
      if constexpr (VT == PKV_INT4_ASYM) {
        const float zp = mt[tk / BS].zp;
        const uint32_t zb = h2_pack(1024.f + zp, 1024.f + zp);
        const uint32_t x = *reinterpret_cast<const uint32_t*>(rs + C::RAW_V + tk * C::V_ROW + 4 * u);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const uint32_t t = x >> (8 * b);
          h[b] = h2_sub((t & 0xFu) | ((t << 12) & 0xF0000u) | 0x64006400u, zb);
        }
      } else {
        const uint2 x =
            *reinterpret_cast<const uint2*>(rs + C::RAW_V + tk * 128 + ((((u >> 1) ^ tk) & 7) << 4) + ((u & 1) << 3));
        s8x8_to_h2(x, h);
      }
      // MN-major atoms of 8 tokens x 64 dims: token groups 2048 bytes apart, dim atoms 1024
      *reinterpret_cast<uint4*>(vd + (tk >> 3) * 2048 + (u >> 3) * 1024 + sw(tk, u)) =
          make_uint4(h[0], h[1], h[2], h[3]);
    }
    tc::fence_proxy_async_smem();  // read next by the tensor core
  };
  // one arrival per warp: the lanes' writes (each fenced for the tensor core) precede lane 0's
  auto warp_arrive = [&](uint64_t* bar) {
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
  };

  const uint32_t t_lane = tmem + ((uint32_t)(q4 * 32) << 16);  // this warp's lanes
  bool ok = true;
  auto fail = [&]() {  // a wait ran out or another warp gave up: everyone stops at its next check
    if (*abort_flag == 0) {
      record_error(p.dev_error, PKV_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    ok = false;
  };
  if (nch > 0) {
    if (!wait_or_abort(&bar_full[0], 0u, abort_flag)) fail();
    convert(0);
    warp_arrive(&bar_conv[0]);
  }

  float m_used = -INFINITY;
  float2 lsum2 = make_float2(0.f, 0.f);
  for (int c = 0; c < nch; ++c) {
    // ---- P V(c-2) done: its V buffer (next: chunk c+1) and weight buffer (next: chunk c) are free ----
    if (c >= 2 && ok && !wait_or_abort(&bar_pv[c & 1], (uint32_t)(((c - 2) >> 1) & 1), abort_flag)) fail();
    // ---- S(c) (issued while chunk c-1 was worked on): this thread's column, its part of the
    // chunk's tokens (one block); the load completes while chunk c+1 is converted ----
    if (ok && !wait_or_abort(&bar_s[c & 1], (uint32_t)((c >> 1) & 1), abort_flag)) fail();
    tc::fence_after_sync();
    uint32_t sr[kTokPart];
    tc::ld_x16(t_lane + (uint32_t)((c & 1) * kT + kTokPart * part), sr);
    if (c + 1 < nch && ok) {
      if (!wait_or_abort(&bar_full[(c + 1) % C::NS], (uint32_t)(((c + 1) / C::NS) & 1), abort_flag)) fail();
      convert(c + 1);
    }
    tc::wait_ld();
    if (c + 1 < nch && ok) {
      tc::fence_before_sync();  // this thread's reads of S(c-1) and S(c) precede the next MMAs
      warp_arrive(&bar_conv[(c + 1) & 1]);
    }
    const BlockMeta bm = meta[(c % C::NMETA) * C::BPC + (kTokPart * part) / BS];
    const int t0 = (jb + c * C::BPC) * BS + kTokPart * part;  // position of the part's first token
    const float2 f2 = make_float2(bm.ks * p.scale_log2, bm.ks * p.scale_log2);
    float2 z[kTokPart / 2];
#pragma unroll
    for (int i = 0; i < kTokPart / 2; ++i)
      z[i] = __fmul2_rn(make_float2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), f2);
    if (!(bm.valid && t0 + kTokPart <= lim)) {  // some token of the part is masked (rare)
#pragma unroll
      for (int i = 0; i < kTokPart / 2; ++i) {
        if (!(bm.valid && t0 + 2 * i < lim)) z[i].x = -INFINITY;
        if (!(bm.valid && t0 + 2 * i + 1 < lim)) z[i].y = -INFINITY;
      }
    }
    float mx[kTokPart / 4];
#pragma unroll
    for (int i = 0; i < kTokPart / 4; ++i)
      mx[i] = fmaxf(fmaxf(z[i].x, z[i].y), fmaxf(z[i + kTokPart / 4].x, z[i + kTokPart / 4].y));
#pragma unroll
    for (int w = kTokPart / 8; w >= 1; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
    // the exchange among the quarter's warps (alternate buffers: a partner may still be reading the
    // previous chunk's); the barrier also spreads a stop to all of them
    float* rb = red + (c & 1) * kParts * kCols;
    rb[part * kCols + col] = mx[0];
    if (quarter_sync_or(q4, !ok || *abort_flag != 0)) {
      ok = false;
      break;
    }
    float bmax = rb[col];
#pragma unroll
    for (int j = 1; j < kParts; ++j) bmax = fmaxf(bmax, rb[j * kCols + col]);
    // (-inf + 8 is -inf: the first visible chunk sets the maximum)
    const bool grow = bmax > m_used + kGrowLog2;
    float al = 1.f;
    if (grow) {
      al = m_used == -INFINITY ? 0.f : ex2(m_used - bmax);
      lsum2 = __fmul2_rn(lsum2, make_float2(al, al));
    }
    // a column whose O holds earlier chunks is rescaled in place, once P V(c-1) has completed; each
    // warp scales its part of the dims (tensor-memory loads and stores are warp-wide: the lanes that
    // need no rescale multiply by 1)
    const bool rescale = grow && c > 0 && m_used != -INFINITY;
    const float al_r = rescale ? al : 1.f;
    if (grow) m_used = bmax;
    if (__any_sync(kFull, rescale)) {
      if (ok && !wait_or_abort(&bar_pv[(c - 1) & 1], (uint32_t)(((c - 1) >> 1) & 1), abort_flag)) fail();
      tc::fence_after_sync();
#pragma unroll 1
      for (int c16 = 0; c16 < kDimPart / 16; ++c16) {
        uint32_t r[16];
        const uint32_t ta = t_lane + kOCol + (uint32_t)(kDimPart * part + 16 * c16);
        tc::ld_x16(ta, r);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * al_r);
        tc::st_x16(ta, r);
      }
      tc::wait_st();
    }
    // ---- weights (V scale folded in), fp16 high and low parts: the A operand of P V(c) ----
    {
      uint8_t* prow_p = psm + (c & 1) * 2 * C::PB + (col >> 3) * 1024;
      const float2 mneg = make_float2(-m_used, -m_used), vs2 = make_float2(bm.vs, bm.vs);
      const bool live = m_used != -INFINITY;
#pragma unroll
      for (int u8 = 0; u8 < kTokPart / 8; ++u8) {  // 8 tokens per 16-byte unit
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float2 w = make_float2(0.f, 0.f);
          if (live) {
            const float2 d = __fadd2_rn(z[4 * u8 + k], mneg);
            w = make_float2(ex2(d.x), ex2(d.y));
          }
          lsum2 = __fadd2_rn(lsum2, w);
          const float2 v = __fmul2_rn(w, vs2);
          hi[k] = h2_pack(v.x, v.y);
          const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi[k]));
          const float2 l = __fadd2_rn(v, make_float2(-hf.x, -hf.y));
          lo[k] = h2_pack(l.x, l.y);
        }
        const int u = (kTokPart / 8) * part + u8;
        *reinterpret_cast<uint4*>(prow_p + sw(col, u)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(prow_p + C::PB + sw(col, u)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();  // the rescale's tensor-memory stores precede P V(c)
    warp_arrive(&bar_pdone[c & 1]);
  }

  // ---- every product issued has completed (the MMA warp commits once it has stopped) ----
  const bool done = mbar_wait_bounded(bar_end, 0u);
  ok = ok && done && *abort_flag == 0;
  tc::fence_after_sync();
  // the column's total weight: the parts' sums (in the buffer the last chunk did not use)
  float* rb = red + (nch & 1) * kParts * kCols;
  rb[part * kCols + col] = lsum2.x + lsum2.y;
  quarter_sync(q4);
  float ltot = 0.f;
#pragma unroll
  for (int j = 0; j < kParts; ++j) ltot += rb[j * kCols + col];
  if (ok) {
    // (every lane takes part in the tensor-memory loads; only valid columns store)
    const bool have_o = nch > 0;
    if constexpr (!PREFIX) {
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      uint4* o = reinterpret_cast<uint4*>(p.out + qrow * kD + kDimPart * part);
#pragma unroll 1
      for (int c16 = 0; c16 < kDimPart / 16; ++c16) {
        uint32_t r[16];
        if (have_o) {
          tc::ld_x16(t_lane + kOCol + (uint32_t)(kDimPart * part + 16 * c16), r);
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
      const int gc = col0 + col;
      const int sm = cvalid ? p.members[gstart + gc / G] : 0;
      const int h = kvh * G + gc % G;
      const long long sl = ((long long)sm * HGd + h / GT) * p.splits + split;
      if (cvalid && part == 0) {
        float* ml = p.pml + (sl * GT + h % GT) * 2;
        ml[0] = m_used == -INFINITY ? -1.0e30f : m_used;
        ml[1] = ltot;
      }
      float4* acc = reinterpret_cast<float4*>(p.pacc + (sl * GT + h % GT) * kD + kDimPart * part);
#pragma unroll 1
      for (int c16 = 0; c16 < kDimPart / 16; ++c16) {
        uint32_t r[16];
        if (have_o) {
          tc::ld_x16(t_lane + kOCol + (uint32_t)(kDimPart * part + 16 * c16), r);
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
  end_sync();  // then the MMA warp frees the tensor memory
}

}  // namespace prefill_tc
}  // namespace pkv
