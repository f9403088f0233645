// decode.cu -- decode-phase paged attention over the block-quantized KV cache (sm_100a).
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
// How (B200 design, not taken from the pages):
//   * grid = (query-head groups, partitions, sequences). A CTA owns one KV head, `GT` query heads
//     of its group and one partition of `partition_tokens` tokens of one sequence.
//   * Each of the NW warps streams every NW-th block of the partition through its own ring of NS
//     shared-memory stages. One lane issues two 1-D bulk asynchronous copies per block (the
//     contiguous bs x D K tile and V tile of this head, 1-4 KiB each) that complete on the
//     stage's mbarrier; the warp then reads the tile with 16-byte shared loads.
//   * Lane mapping: a lane owns 16 consecutive dims (D/16 lanes per token row) and bs/(32*16/D)
//     token rows of each block. Codes become exact floats through the float bit layout (no I2F),
//     dot products accumulate in fp32, the per-block scale multiplies the 16-term dot once.
//   * Online softmax per warp in the log2 domain (ex2.approx); warps are merged through shared
//     memory at the end; a sequence with one partition is written out directly, otherwise the
//     partition's (max, sum, accumulator) goes to the workspace and the last of the sequence's
//     partition CTAs to finish merges them (split-K in one launch, no second kernel).
#include "common.cuh"
#include "internal.h"

namespace pkv {

namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr float kNegBig = -1.0e30f;  // finite "minus infinity" for running maxima

template <int KT, int VT, int BS, int D, int GT>
struct Cfg {
  static constexpr int NW = 4;  // warps per CTA
  static constexpr int K_ROW = (KT == PKV_FP16) ? 2 * D : D;
  static constexpr int V_ROW = (VT == PKV_FP16) ? 2 * D : (VT == PKV_INT8_SYM ? D : D / 2);
  static constexpr int K_TILE = BS * K_ROW;
  static constexpr int V_TILE = BS * V_ROW;
  static constexpr int STAGE = K_TILE + V_TILE;
  // ~64 KiB of stages per CTA, 2..4 stages per warp
  static constexpr int NS_RAW = 65536 / (NW * STAGE);
  static constexpr int NS = NS_RAW < 2 ? 2 : (NS_RAW > 4 ? 4 : NS_RAW);
  static constexpr int CH = D / 16;    // lanes per token row
  static constexpr int TG = 32 / CH;   // token rows a warp covers per pass
  static constexpr int TPL = BS / TG;  // token rows per lane per block
  static constexpr int THREADS = 32 * NW;
  static constexpr int SMEM_STAGES = NW * NS * STAGE;
  static constexpr int SMEM_MERGE_ACC = NW * GT * D * 4;
  static constexpr int SMEM_MERGE_ML = NW * GT * 2 * 4;
  static constexpr int SMEM_BARS = NW * NS * 8;
  static constexpr int SMEM = SMEM_STAGES + SMEM_MERGE_ACC + SMEM_MERGE_ML + SMEM_BARS;
  static_assert(D % 16 == 0 && CH <= 32 && 32 % CH == 0, "head_dim");
  static_assert(BS % TG == 0, "block_size must cover the token rows of a warp pass");
  static_assert(K_TILE % 16 == 0 && V_TILE % 16 == 0 && STAGE % 16 == 0, "bulk copy granularity");
};

// 16 consecutive K values of one token row (lane chunk) -> 8 float2 (dims in order)
template <int KT>
__device__ __forceinline__ void load_k16(const uint8_t* p, float2 f[8]) {
  if constexpr (KT == PKV_INT8_SYM) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    s8x4_to_f32x2(w.x, f[0], f[1]);
    s8x4_to_f32x2(w.y, f[2], f[3]);
    s8x4_to_f32x2(w.z, f[4], f[5]);
    s8x4_to_f32x2(w.w, f[6], f[7]);
  } else {
    const uint4 w0 = *reinterpret_cast<const uint4*>(p);
    const uint4 w1 = *reinterpret_cast<const uint4*>(p + 16);
    const uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
  }
}

// 16 consecutive V values of one token row (lane chunk) -> 8 float2 of (code - zp);
// neg_bias = -(2^23 + zp) in both lanes (INT4 only)
template <int VT>
__device__ __forceinline__ void load_v16(const uint8_t* p, float2 neg_bias, float2 f[8]) {
  if constexpr (VT == PKV_INT8_SYM) {
    load_k16<PKV_INT8_SYM>(p, f);
  } else if constexpr (VT == PKV_INT4_ASYM) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    u4x8_to_f32x2(w.x, neg_bias, f);
    u4x8_to_f32x2(w.y, neg_bias, f + 4);
  } else {
    load_k16<PKV_FP16>(p, f);
  }
}

template <int KT, int VT, int BS, int D, int GT>
__global__ void __launch_bounds__(Cfg<KT, VT, BS, D, GT>::THREADS)
    paged_decode_kernel(const DecodeParams p) {
  using C = Cfg<KT, VT, BS, D, GT>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  float* merge_acc = reinterpret_cast<float*>(smem + C::SMEM_STAGES);                 // [NW][GT][D]
  float* merge_ml = reinterpret_cast<float*>(smem + C::SMEM_STAGES + C::SMEM_MERGE_ACC);  // [NW][GT][2]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_STAGES + C::SMEM_MERGE_ACC + C::SMEM_MERGE_ML);

  const int h0 = blockIdx.x * GT;  // first query head of this CTA
  const int part = blockIdx.y;
  const int s = blockIdx.z;
  const int g = h0 / p.group;  // KV head shared by the CTA's query heads
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = lane % C::CH;   // 16-dim chunk of this lane
  const int tg = lane / C::CH;  // token-row group of this lane
  const int PT = p.partition_tokens;

  // ---- pipeline set-up: this warp's NS stages and barriers (no memory dependence) ----
  uint8_t* my_stages = stages + (size_t)warp * C::NS * C::STAGE;
  uint64_t* my_bars = bars + warp * C::NS;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < C::NS; ++st) mbar_init(&my_bars[st], 1);
    fence_mbar_init();
  }

  // ---- first round of global loads, all independent of one another ----
  // The partition's first block index does not depend on the context length, so this warp's
  // block-table entries are read speculatively (in bounds of the table row) together with the
  // length; entries past the sequence's end are never used.
  const int blk_begin = (part * PT) / BS;
  const int j_lane = blk_begin + warp + C::NW * lane;
  int b_raw = -1;
  if (lane * C::NW * BS < PT && j_lane < p.max_blocks_per_seq)
    b_raw = p.block_tables[(size_t)s * p.max_blocks_per_seq + j_lane];
  int L = p.context_lens[s];

  // query heads of the CTA, this lane's 16 dims
  float2 qf[GT][8];
#pragma unroll
  for (int hh = 0; hh < GT; ++hh) {
    const __half* qp = p.q + ((size_t)s * p.num_q_heads + h0 + hh) * D + c * 16;
    const uint4 w0 = *reinterpret_cast<const uint4*>(qp);
    const uint4 w1 = *reinterpret_cast<const uint4*>(qp + 8);
    const uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) qf[hh][i] = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
  }
  // INT8 K: q . k is computed exactly in integers. Each head's q is put on a fixed-point grid of
  // 2^-shift (22 bits below its largest magnitude; fp16 q loses nothing above 2^-22 of its max)
  // and split into three signed byte planes, q_fixed = 2^16 b2 + 2^8 b1 + b0, so a 4-code word
  // costs three dp4a with int32 accumulation and no code ever has to be converted to float.
  uint32_t qplane[GT][3][4];
  float qinv[GT];  // 2^-shift
  if constexpr (KT == PKV_INT8_SYM) {
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fmaxf(fabsf(qf[hh][i].x), fabsf(qf[hh][i].y)));
#pragma unroll
      for (int off = 1; off < C::CH; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
      int e = 0;
      (void)frexpf(amax, &e);                    // amax < 2^e
      const int shift = amax > 0.f ? 22 - e : 0;  // |q| * 2^shift < 2^22
      const float up = __int_as_float((127 + shift) << 23);
      qinv[hh] = __int_as_float((127 - shift) << 23);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t p0 = 0, p1 = 0, p2 = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 pr = qf[hh][(4 * w + k) / 2];
          const int qi = __float2int_rn((((4 * w + k) & 1) ? pr.y : pr.x) * up);
          const int b0 = ((qi + 128) & 0xFF) - 128;
          const int r1 = (qi - b0) >> 8;
          const int b1 = ((r1 + 128) & 0xFF) - 128;
          const int b2 = (r1 - b1) >> 8;
          p0 |= (uint32_t)(b0 & 0xFF) << (8 * k);
          p1 |= (uint32_t)(b1 & 0xFF) << (8 * k);
          p2 |= (uint32_t)(b2 & 0xFF) << (8 * k);
        }
        qplane[hh][0][w] = p0;
        qplane[hh][1][w] = p1;
        qplane[hh][2][w] = p2;
      }
    }
  }

  // ---- context length (validated; clamped on error) and this warp's share of the partition ----
  {
    const int cap = min(p.max_context_len, p.max_blocks_per_seq * BS);
    if (L < 0 || L > cap) {
      if (part == 0 && blockIdx.x == 0 && threadIdx.x == 0) record_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN);
      L = max(0, min(L, cap));
    }
  }
  const int num_parts = (L + PT - 1) / PT;
  if (part >= (num_parts > 0 ? num_parts : 1)) return;  // beyond this sequence's partitions (CTA-uniform)

  const int t_begin = part * PT;
  const int t_end = min(L, t_begin + PT);
  const int n_blk = t_end > t_begin ? (t_end - t_begin + BS - 1) / BS : 0;
  // this warp's blocks: blk_begin + warp + NW * k, k < my_blocks (<= 32 by the partition cap)
  const int my_blocks = n_blk > warp ? (n_blk - warp + C::NW - 1) / C::NW : 0;

  const bool my_valid = lane < my_blocks && b_raw >= 0 && b_raw < p.num_blocks;
  if (lane < my_blocks && !my_valid) record_error(p.dev_error, PKV_DEVERR_BLOCK_ID);
  const int my_b = my_valid ? b_raw : 0;  // block 0 stands in for an invalid id (its tokens are masked)
  __syncwarp();  // barrier initialisation by lane 0 is visible to the warp

  const size_t head_tile = (size_t)p.num_kv_heads;
  auto issue = [&](int st, int b) {
    const size_t tile = (size_t)b * head_tile + g;
    uint8_t* dst = my_stages + (size_t)st * C::STAGE;
    mbar_arrive_expect_tx(&my_bars[st], (uint32_t)C::STAGE);
    bulk_g2s(dst, static_cast<const uint8_t*>(p.k_codes) + tile * C::K_TILE, (uint32_t)C::K_TILE, &my_bars[st]);
    bulk_g2s(dst + C::K_TILE, static_cast<const uint8_t*>(p.v_codes) + tile * C::V_TILE, (uint32_t)C::V_TILE,
             &my_bars[st]);
  };

  // ---- fill the ring: the first NS tiles of this warp are in flight from here on ----
#pragma unroll
  for (int k = 0; k < C::NS; ++k) {
    const int b = __shfl_sync(kFull, my_b, k);
    if (lane == 0 && k < my_blocks) issue(k, b);
  }

  // ---- per-block scales / zero points: their latency overlaps the copies in flight ----
  float my_ks = 0.f, my_vs = 0.f, my_zp = 0.f;
  if (lane < my_blocks) {
    const size_t meta = (size_t)my_b * p.num_kv_heads + g;
    if constexpr (KT != PKV_FP16) my_ks = p.k_scale[meta];
    if constexpr (VT != PKV_FP16) my_vs = p.v_scale[meta];
    if constexpr (VT == PKV_INT4_ASYM) my_zp = (float)p.v_zp[meta];
  }

  float m_run[GT], l_run[GT];
  float2 acc[GT][8];  // this lane's 16 dims, as pairs
#pragma unroll
  for (int hh = 0; hh < GT; ++hh) {
    m_run[hh] = kNegBig;
    l_run[hh] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[hh][j] = make_float2(0.f, 0.f);
  }

  bool aborted = false;
  int k_stop = my_blocks;  // first block not consumed (differs from my_blocks after a timeout)
  for (int k = 0; k < my_blocks; ++k) {
    const int st = k % C::NS;
    const uint32_t parity = (uint32_t)((k / C::NS) & 1);
    const bool ok = __all_sync(kFull, mbar_wait_bounded(&my_bars[st], parity));
    if (!ok) {
      if (lane == 0) record_error(p.dev_error, PKV_DEVERR_TIMEOUT);
      aborted = true;
      k_stop = k;
      break;
    }
    const float ks = __shfl_sync(kFull, my_ks, k) * p.scale_log2;  // per-block K scale, log2 domain
    const float vs = __shfl_sync(kFull, my_vs, k);
    const float nzb = -(kMagic + __shfl_sync(kFull, my_zp, k));
    const float2 neg_zp_bias = make_float2(nzb, nzb);
    const bool valid = __shfl_sync(kFull, my_valid ? 1 : 0, k) != 0;
    const int tok0 = (blk_begin + warp + C::NW * k) * BS;
    const uint8_t* kt = my_stages + (size_t)st * C::STAGE;
    const uint8_t* vt = kt + C::K_TILE;

    // q . k for this lane's rows and dims, reduced over the CH lanes of a row
    float z[C::TPL][GT];
#pragma unroll
    for (int i = 0; i < C::TPL; ++i) {
      const int row = tg + C::TG * i;
      const uint8_t* krow = kt + row * C::K_ROW + c * (C::K_ROW / C::CH);
      if constexpr (KT == PKV_INT8_SYM) {
        const uint4 w = *reinterpret_cast<const uint4*>(krow);
        const int kw[4] = {(int)w.x, (int)w.y, (int)w.z, (int)w.w};
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
        load_k16<KT>(krow, kf);
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
    for (int i = 0; i < C::TPL; ++i)
#pragma unroll
      for (int hh = 0; hh < GT; ++hh)
#pragma unroll
        for (int off = 1; off < C::CH; off <<= 1) z[i][hh] += __shfl_xor_sync(kFull, z[i][hh], off);

    // scale, mask, online softmax update (log2 domain)
    float pv[C::TPL][GT];
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      float mloc = -INFINITY;
#pragma unroll
      const float zscale = (KT == PKV_FP16) ? p.scale_log2 : ks * qinv[hh];
      for (int i = 0; i < C::TPL; ++i) {
        const int t = tok0 + tg + C::TG * i;
        float zz = z[i][hh] * zscale;
        zz = (valid && t < t_end) ? zz : -INFINITY;
        z[i][hh] = zz;
        mloc = fmaxf(mloc, zz);
      }
#pragma unroll
      for (int off = C::CH; off < 32; off <<= 1) mloc = fmaxf(mloc, __shfl_xor_sync(kFull, mloc, off));
      // the running max is warp-uniform; rescale only when it grows (rare after the first blocks)
      if (mloc > m_run[hh]) {
        const float alpha = ex2(m_run[hh] - mloc);
        m_run[hh] = mloc;
        l_run[hh] *= alpha;
        const float2 alpha2 = make_float2(alpha, alpha);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[hh][j] = __fmul2_rn(acc[hh][j], alpha2);
      }
      const float m_new = m_run[hh];
      float lsum = 0.f;
#pragma unroll
      for (int i = 0; i < C::TPL; ++i) {
        const float pr = ex2(z[i][hh] - m_new);
        lsum += pr;
        pv[i][hh] = (VT == PKV_FP16) ? pr : pr * vs;
      }
      l_run[hh] += lsum;
    }

    // p . v_hat for this lane's rows and dims
#pragma unroll
    for (int i = 0; i < C::TPL; ++i) {
      const int row = tg + C::TG * i;
      float2 vf[8];
      load_v16<VT>(vt + row * C::V_ROW + c * (C::V_ROW / C::CH), neg_zp_bias, vf);
#pragma unroll
      for (int hh = 0; hh < GT; ++hh) {
        const float2 pv2 = make_float2(pv[i][hh], pv[i][hh]);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[hh][j] = __ffma2_rn(pv2, vf[j], acc[hh][j]);
      }
    }

    // stage st is free again: refill it with block k + NS
    __syncwarp();
    const int kn = k + C::NS;
    const int bn = __shfl_sync(kFull, my_b, kn & 31);
    // (the warp's reads of this stage have completed: their values were consumed above)
    if (lane == 0 && kn < my_blocks) issue(st, bn);
  }

  if (aborted) {
    // A copy never completed (the output of this CTA is unspecified; dev_error says so).
    // Wait, again bounded, for the copies this warp issued and did not consume, so that no bulk
    // copy is still writing this CTA's shared memory when it exits; then contribute nothing.
    if (lane == 0) {
      for (int k = k_stop; k < min(k_stop + C::NS, my_blocks); ++k)
        (void)mbar_wait_bounded(&my_bars[k % C::NS], (uint32_t)((k / C::NS) & 1));
    }
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      m_run[hh] = kNegBig;
      l_run[hh] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[hh][j] = make_float2(0.f, 0.f);
    }
  }

  // ---- reduce the warp's state over its token-row groups ----
#pragma unroll
  for (int hh = 0; hh < GT; ++hh) {
#pragma unroll
    for (int off = C::CH; off < 32; off <<= 1) l_run[hh] += __shfl_xor_sync(kFull, l_run[hh], off);
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int off = C::CH; off < 32; off <<= 1) {
        acc[hh][j].x += __shfl_xor_sync(kFull, acc[hh][j].x, off);
        acc[hh][j].y += __shfl_xor_sync(kFull, acc[hh][j].y, off);
      }
  }
  if (tg == 0) {
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      float4* dst = reinterpret_cast<float4*>(merge_acc + ((size_t)warp * GT + hh) * D + c * 16);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        dst[j] = make_float4(acc[hh][2 * j].x, acc[hh][2 * j].y, acc[hh][2 * j + 1].x, acc[hh][2 * j + 1].y);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      merge_ml[(warp * GT + hh) * 2 + 0] = m_run[hh];
      merge_ml[(warp * GT + hh) * 2 + 1] = l_run[hh];
    }
  }
  __syncthreads();

  // ---- merge the warps; write the final output or this partition's partial ----
  const bool single = num_parts <= 1;
  for (int o = threadIdx.x; o < GT * D; o += C::THREADS) {
    const int hh = o / D, d = o % D;
    float M = kNegBig;
#pragma unroll
    for (int w = 0; w < C::NW; ++w) M = fmaxf(M, merge_ml[(w * GT + hh) * 2]);
    float Lsum = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < C::NW; ++w) {
      const float e = ex2(merge_ml[(w * GT + hh) * 2] - M);
      Lsum = fmaf(merge_ml[(w * GT + hh) * 2 + 1], e, Lsum);
      A = fmaf(merge_acc[((size_t)w * GT + hh) * D + d], e, A);
    }
    const int h = h0 + hh;
    if (single) {
      p.out[((size_t)s * p.num_q_heads + h) * D + d] = __float2half_rn(Lsum > 0.f ? A / Lsum : 0.f);
    } else {
      const size_t idx = ((size_t)s * p.num_q_heads + h) * p.max_partitions + part;
      p.ws_acc[idx * D + d] = A;
      if (d == 0) {
        p.ws_ml[idx * 2 + 0] = M;
        p.ws_ml[idx * 2 + 1] = Lsum;
      }
    }
  }
  if (single) return;

  // ---- split-K merge by the last partition CTA of this (sequence, head group) to finish ----
  // Every partition CTA publishes its partial, then bumps a counter with atomicInc, which wraps
  // back to 0 when the last of num_parts arrivals takes it: the counter is left at zero for the
  // next call without a reset. The CTA that sees num_parts - 1 merges
  //   out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p.
  __shared__ uint32_t s_ticket;
  __syncthreads();  // every partial write of this CTA precedes thread 0's fence (CTA scope)
  if (threadIdx.x == 0) {
    __threadfence();  // release: the CTA's partial is visible device-wide before the counter moves
    s_ticket = atomicInc(&p.ws_count[(size_t)s * gridDim.x + blockIdx.x], (uint32_t)(num_parts - 1));
    __threadfence();  // acquire side for the merging CTA
  }
  __syncthreads();
  if (s_ticket != (uint32_t)(num_parts - 1)) return;
  for (int o = threadIdx.x; o < GT * D; o += C::THREADS) {
    const int hh = o / D, d = o % D;
    const size_t base = ((size_t)s * p.num_q_heads + h0 + hh) * p.max_partitions;
    float M = kNegBig;
    for (int i = 0; i < num_parts; ++i) M = fmaxf(M, __ldcg(&p.ws_ml[(base + i) * 2]));
    float Lsum = 0.f, A = 0.f;
    for (int i = 0; i < num_parts; ++i) {
      const float e = ex2(__ldcg(&p.ws_ml[(base + i) * 2]) - M);
      Lsum = fmaf(__ldcg(&p.ws_ml[(base + i) * 2 + 1]), e, Lsum);
      A = fmaf(__ldcg(&p.ws_acc[(base + i) * D + d]), e, A);
    }
    p.out[((size_t)s * p.num_q_heads + h0 + hh) * D + d] = __float2half_rn(Lsum > 0.f ? A / Lsum : 0.f);
  }
}

template <int KT, int VT, int BS, int D, int GT>
cudaError_t launch_one(const DecodeParams& p, const DecodeShape& sh, cudaStream_t stream) {
  using C = Cfg<KT, VT, BS, D, GT>;
  auto kern = paged_decode_kernel<KT, VT, BS, D, GT>;
  static unsigned long long configured = 0;  // one bit per device; benign race (same value)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured |= bit;
  }
  dim3 grid(p.num_q_heads / GT, p.max_partitions, sh.num_seqs);
  kern<<<grid, C::THREADS, C::SMEM, stream>>>(p);
  return cudaGetLastError();
}

template <int KT, int VT, int BS, int D>
cudaError_t dispatch_gt(const DecodeParams& p, const DecodeShape& sh, cudaStream_t stream) {
  switch (sh.heads_per_cta) {
    case 1: return launch_one<KT, VT, BS, D, 1>(p, sh, stream);
    case 2: return launch_one<KT, VT, BS, D, 2>(p, sh, stream);
    case 4: return launch_one<KT, VT, BS, D, 4>(p, sh, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int KT, int VT, int BS>
cudaError_t dispatch_d(const DecodeParams& p, const DecodeShape& sh, cudaStream_t stream) {
  switch (sh.head_dim) {
    case 64: return dispatch_gt<KT, VT, BS, 64>(p, sh, stream);
    case 128: return dispatch_gt<KT, VT, BS, 128>(p, sh, stream);
    case 256: return dispatch_gt<KT, VT, BS, 256>(p, sh, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int KT, int VT>
cudaError_t dispatch_bs(const DecodeParams& p, const DecodeShape& sh, cudaStream_t stream) {
  switch (sh.block_size) {
    case 16: return dispatch_d<KT, VT, 16>(p, sh, stream);
    case 32: return dispatch_d<KT, VT, 32>(p, sh, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int32_t decode_heads_per_cta(int32_t group) {
  if (group % 4 == 0) return 4;
  if (group % 2 == 0) return 2;
  return 1;
}

int32_t decode_max_partition_tokens(int32_t block_size) {
  return 32 * 4 * block_size;  // 32 blocks per warp (one id per lane) x 4 warps
}

bool decode_supported(int32_t k_dtype, int32_t v_dtype, int32_t block_size, int32_t head_dim) {
  const bool dt = (k_dtype == PKV_INT8_SYM && (v_dtype == PKV_INT8_SYM || v_dtype == PKV_INT4_ASYM)) ||
                  (k_dtype == PKV_FP16 && v_dtype == PKV_FP16);
  // an FP16 cache with head_dim 256 and 32-token blocks needs 32 KiB per stage: two stages for
  // each of four warps exceed the 227 KiB of shared memory a CTA can have
  if (k_dtype == PKV_FP16 && head_dim == 256 && block_size == 32) return false;
  return dt && (block_size == 16 || block_size == 32) && (head_dim == 64 || head_dim == 128 || head_dim == 256);
}

cudaError_t launch_decode(const DecodeParams& p, const DecodeShape& sh, cudaStream_t stream) {
  if (sh.k_dtype == PKV_INT8_SYM && sh.v_dtype == PKV_INT8_SYM)
    return dispatch_bs<PKV_INT8_SYM, PKV_INT8_SYM>(p, sh, stream);
  if (sh.k_dtype == PKV_INT8_SYM && sh.v_dtype == PKV_INT4_ASYM)
    return dispatch_bs<PKV_INT8_SYM, PKV_INT4_ASYM>(p, sh, stream);
  if (sh.k_dtype == PKV_FP16 && sh.v_dtype == PKV_FP16) return dispatch_bs<PKV_FP16, PKV_FP16>(p, sh, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pkv
