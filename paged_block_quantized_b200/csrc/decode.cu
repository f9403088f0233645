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
// How (B200 design, not taken from the pages): a persistent, stream-K kernel.
//   * A "unit" is (sequence s, head group hg): GT query heads sharing one KV head. Every unit
//     contributes ceil(L_s / bs) blocks to one global stream, ordered (s, hg, block). The grid
//     is a fixed set of worker warps (a few CTAs per SM, each warp independent); warp w owns
//     the contiguous stream range [w*T/W, (w+1)*T/W), so every warp gets the same number of
//     blocks whatever the length mix.
//   * Each warp streams its range through its own ring of NS shared-memory stages: lane 0
//     issues two 1-D bulk asynchronous copies per block (the contiguous bs x D K tile and V tile
//     of this head, 1-4 KiB each) that complete on the stage's mbarrier, up to NS blocks ahead
//     and straight across unit boundaries; the warp reads tiles with 16-byte shared loads.
//   * Block ids are read 32 at a time ("windows", one id per lane) one window ahead; per-block
//     scales are fetched when the window's first copy is issued, NS blocks before use.
//   * q . k for INT8 K is exact integer arithmetic: q on a 22-bit fixed-point grid split into
//     three signed byte planes, three dp4a per 4 codes. V codes become exact floats through the
//     float bit layout (PRMT + paired FADD, no I2F); p . v accumulates with paired FFMA.
//   * Online softmax in the log2 domain (ex2.approx), rescaling only when the running max grows.
//   * A unit processed entirely by one warp is written out directly. A unit split across warps
//     gets one partial (max, sum, acc) per warp in the workspace; the last warp to finish (a
//     self-resetting atomicInc ticket) merges them. No CTA barrier, no second kernel.
#include "common.cuh"
#include "internal.h"

namespace pkv {

namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr float kNegBig = -1.0e30f;  // finite "minus infinity" for running maxima

// Shared-memory budget of one CTA's copy rings and the CTA-per-SM caps by heads per warp
// (overridable at build time for tuning sweeps).
#ifndef PKV_DECODE_SMEM_TARGET
#define PKV_DECODE_SMEM_TARGET 32768
#endif
#ifndef PKV_DECODE_CPS_GT1
#define PKV_DECODE_CPS_GT1 4
#endif
#ifndef PKV_DECODE_MAX_STAGES
#define PKV_DECODE_MAX_STAGES 6
#endif

template <int KT, int VT, int BS, int D, int GT>
struct Cfg {
  static constexpr int K_ROW = (KT == PKV_FP16) ? 2 * D : D;
  static constexpr int V_ROW = (VT == PKV_FP16) ? 2 * D : (VT == PKV_INT8_SYM ? D : D / 2);
  static constexpr int K_TILE = BS * K_ROW;
  static constexpr int V_TILE = BS * V_ROW;
  static constexpr int STAGE = K_TILE + V_TILE;
  static constexpr int NW = (4 * 2 * STAGE <= 200 * 1024) ? 4 : 2;  // warps per CTA
  // stages per warp from the CTA's shared-memory budget, at least 2
  static constexpr int NS_RAW = PKV_DECODE_SMEM_TARGET / (NW * STAGE);
  static constexpr int NS = NS_RAW < 2 ? 2 : (NS_RAW > PKV_DECODE_MAX_STAGES ? PKV_DECODE_MAX_STAGES : NS_RAW);
  static constexpr int CH = D / 16;    // lanes per token row (16 dims each)
  static constexpr int TG = 32 / CH;   // token rows a warp covers per pass
  static constexpr int TPL = BS / TG;  // token rows per lane per block
  static constexpr int THREADS = 32 * NW;
  static constexpr int SMEM_STAGES = NW * NS * STAGE;
  static constexpr int SMEM = SMEM_STAGES + NW * NS * 8;
  // resident CTAs per SM: bounded by shared memory (227 KiB per SM) and by the registers a
  // thread needs for GT heads of state
  static constexpr int CPS_SMEM = (220 * 1024) / (SMEM + 1024);
  static constexpr int CPS_CAP = (GT == 1) ? PKV_DECODE_CPS_GT1 : (GT == 2 ? 3 : 2);  // 128 / 170 / 255 regs
  static constexpr int CTAS_PER_SM = CPS_SMEM < 1 ? 1 : (CPS_SMEM > CPS_CAP ? CPS_CAP : CPS_SMEM);
  static_assert(D % 16 == 0 && CH <= 32 && 32 % CH == 0, "head_dim");
  static_assert(BS % TG == 0, "block_size must cover the token rows of a warp pass");
  static_assert(K_TILE % 16 == 0 && V_TILE % 16 == 0 && STAGE % 16 == 0, "bulk copy granularity");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// 16 consecutive fp16 values of one token row (lane chunk) -> 8 float2 (dims in order)
__device__ __forceinline__ void load_h16(const uint8_t* p, float2 f[8]) {
  const uint4 w0 = *reinterpret_cast<const uint4*>(p);
  const uint4 w1 = *reinterpret_cast<const uint4*>(p + 16);
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
    load_h16(p, f);
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
  int s, hg, j0, n;     // sequence, head group, first block, blocks in the window (0 = none)
  int g;                // KV head of the head group
  int L, nblk;          // clamped length of the sequence and its block count
  int r0;               // position of block j0 relative to the warp's first position
  long long seq_p0;     // stream position of the sequence's first block (head group 0)
};

struct WinLanes {
  int b;        // physical block (0 stands in for an invalid id)
  int raw;      // block id as read from the table
  bool valid;
  bool meta;    // scales fetched (warp-uniform)
  float ks, vs, zp;
};

template <int KT, int VT, int BS, int D, int GT>
__global__ void __launch_bounds__(Cfg<KT, VT, BS, D, GT>::THREADS, Cfg<KT, VT, BS, D, GT>::CTAS_PER_SM)
    paged_decode_kernel(const DecodeParams p) {
  using C = Cfg<KT, VT, BS, D, GT>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = lane % C::CH;   // 16-dim chunk of this lane
  const int tg = lane / C::CH;  // token-row group of this lane
  const int W = gridDim.x * C::NW;
  const int w = blockIdx.x * C::NW + warp;
  const int HG = p.num_q_heads / GT;
  const int S = p.num_seqs;

  uint8_t* my_stages = smem + (size_t)warp * C::NS * C::STAGE;
  uint64_t* my_bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_STAGES) + warp * C::NS;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < C::NS; ++st) mbar_init(&my_bars[st], 1);
    fence_mbar_init();
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
    int sum = (L + BS - 1) / BS;
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
  if (w >= We) return;
  const long long start = (long long)w * T / We;
  const long long end = (long long)(w + 1) * T / We;

  // ---- pass 2: the unit and block of `start` ----
  Win cur;
  int Lchunk = 0, chunk_base = 0;  // lane holds the clamped length of sequence chunk_base + lane
  {
    long long acc0 = 0;
    for (int base = 0;; base += 32) {
      const int s = base + lane;
      const int L = s < S ? clamp_len(p, p.context_lens[s], BS) : 0;
      const long long cnt = (long long)((L + BS - 1) / BS) * HG;
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
        cur.L = __shfl_sync(kFull, L, f);
        cur.nblk = (cur.L + BS - 1) / BS;
        cur.seq_p0 = acc0 + __shfl_sync(kFull, incl - cnt, f);
        Lchunk = L;
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
      Lchunk = (s + lane < S) ? clamp_len(p, p.context_lens[s + lane], BS) : 0;
    }
    return __shfl_sync(kFull, Lchunk, s - chunk_base);
  };

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
        b.L = L;
        b.nblk = (L + BS - 1) / BS;
      }
      b.g = (b.hg * GT) / p.group;
    }
    b.n = min(min(32, b.nblk - b.j0), n_total - b.r0);
    return b;
  };

  // phase A of a window: block ids (one per lane); phase B (at its first copy): scales
  auto load_ids = [&](const Win& a, WinLanes& r) {
    r.meta = false;
    r.raw = -1;
    if (lane < a.n) r.raw = p.block_tables[(size_t)a.s * p.max_blocks_per_seq + a.j0 + lane];
  };
  auto load_meta = [&](const Win& a, WinLanes& r) {
    r.valid = lane < a.n && r.raw >= 0 && r.raw < p.num_blocks;
    if (lane < a.n && !r.valid) record_error(p.dev_error, PKV_DEVERR_BLOCK_ID);
    r.b = r.valid ? r.raw : 0;
    r.ks = r.vs = r.zp = 0.f;
    if (lane < a.n) {
      const size_t meta = (size_t)r.b * p.num_kv_heads + a.g;
      if constexpr (KT != PKV_FP16) r.ks = p.k_scale[meta];
      if constexpr (VT != PKV_FP16) r.vs = p.v_scale[meta];
      if constexpr (VT == PKV_INT4_ASYM) r.zp = (float)p.v_zp[meta];
    }
    r.meta = true;
  };

  WinLanes rc, rn;
  load_ids(cur, rc);
  Win nxt = next_win(cur);
  load_ids(nxt, rn);
  // Everything above reads only what the host wrote before the preceding kernel (lengths,
  // tables). From here on the pool is read, which the preceding kernel (the store of the new
  // tokens) may still be writing: wait for it to complete (no-op without a programmatic launch).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  load_meta(cur, rc);
  __syncwarp();  // barrier initialisation by lane 0 is visible to the warp

  // ---- per-unit state ----
  float2 qf[GT][8];
  uint32_t qplane[GT][3][4];
  float qinv[GT];
  float m_run[GT], l_run[GT];
  float2 acc[GT][8];
  int seg_j0 = cur.j0;  // first block of the current segment within its unit

  auto begin_unit = [&](const Win& a) {
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      const __half* qp = p.q + ((size_t)a.s * p.num_q_heads + (size_t)a.hg * GT + hh) * D + c * 16;
      const uint4 w0 = *reinterpret_cast<const uint4*>(qp);
      const uint4 w1 = *reinterpret_cast<const uint4*>(qp + 8);
      const uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) qf[hh][i] = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
      m_run[hh] = kNegBig;
      l_run[hh] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[hh][j] = make_float2(0.f, 0.f);
    }
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
        for (int off = 1; off < C::CH; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
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
  };
  begin_unit(cur);

  // ---- the copy ring ----
  auto issue = [&](int st, int b, int g) {
    const size_t tile = (size_t)b * p.num_kv_heads + g;
    uint8_t* dst = my_stages + (size_t)st * C::STAGE;
    mbar_arrive_expect_tx(&my_bars[st], (uint32_t)C::STAGE);
    bulk_g2s(dst, static_cast<const uint8_t*>(p.k_codes) + tile * C::K_TILE, (uint32_t)C::K_TILE, &my_bars[st]);
    bulk_g2s(dst + C::K_TILE, static_cast<const uint8_t*>(p.v_codes) + tile * C::V_TILE, (uint32_t)C::V_TILE,
             &my_bars[st]);
  };
  // positions relative to `start`: consumed (cpos) and issued (ipos); stage / parity of each
  int cpos = 0, ipos = 0, cst = 0, ist = 0;
  uint32_t cpar = 0;
  // issue every position below min(cpos + NS, n_total) whose window is known (cur or nxt); a
  // stage is reused only after the position NS before it has been consumed
  auto issue_ahead = [&]() {
    const int lim = min(cpos + C::NS, n_total);
    while (ipos < lim) {
      int b, g;
      if (ipos < cur.r0 + cur.n) {
        b = __shfl_sync(kFull, rc.b, ipos - cur.r0);
        g = cur.g;
      } else if (nxt.n > 0 && ipos < nxt.r0 + nxt.n) {
        if (!rn.meta) load_meta(nxt, rn);
        b = __shfl_sync(kFull, rn.b, ipos - nxt.r0);
        g = nxt.g;
      } else {
        break;
      }
      if (lane == 0) issue(ist, b, g);
      ist = (ist + 1 == C::NS) ? 0 : ist + 1;
      ++ipos;
    }
  };

  bool aborted = false;
  while (cpos < n_total) {
    if (cpos == cur.r0 + cur.n) {  // step into the next window
      const bool new_unit = (nxt.s != cur.s) || (nxt.hg != cur.hg);
      cur = nxt;
      rc = rn;
      if (!rc.meta) load_meta(cur, rc);
      nxt = next_win(cur);
      load_ids(nxt, rn);
      if (new_unit) {
        begin_unit(cur);
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
    const float ks = __shfl_sync(kFull, rc.ks, kw_i) * p.scale_log2;  // per-block K scale, log2 domain
    const float vs = __shfl_sync(kFull, rc.vs, kw_i);
    const float nzb = -(kMagic + __shfl_sync(kFull, rc.zp, kw_i));
    const float2 neg_zp_bias = make_float2(nzb, nzb);
    const bool valid = __shfl_sync(kFull, rc.valid ? 1 : 0, kw_i) != 0;
    const int tok0 = (cur.j0 + kw_i) * BS;
    const uint8_t* kt = my_stages + (size_t)st * C::STAGE;
    const uint8_t* vt = kt + C::K_TILE;

    float z[C::TPL][GT];
#pragma unroll
    for (int i = 0; i < C::TPL; ++i) {
      const int row = tg + C::TG * i;
      const uint8_t* krow = kt + row * C::K_ROW + c * (C::K_ROW / C::CH);
      if constexpr (KT == PKV_INT8_SYM) {
        const uint4 wv = *reinterpret_cast<const uint4*>(krow);
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
        load_h16(krow, kf);
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

    float pv[C::TPL][GT];
#pragma unroll
    for (int hh = 0; hh < GT; ++hh) {
      const float zscale = (KT == PKV_FP16) ? p.scale_log2 : ks * qinv[hh];
      float mloc = -INFINITY;
#pragma unroll
      for (int i = 0; i < C::TPL; ++i) {
        const int t = tok0 + tg + C::TG * i;
        float zz = z[i][hh] * zscale;
        zz = (valid && t < cur.L) ? zz : -INFINITY;
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
    __syncwarp();  // the stage's reads are complete (their values were consumed above)
    ++cpos;
    if (++cst == C::NS) {
      cst = 0;
      cpar ^= 1u;
    }

    // ---- end of a segment: the unit's last block, or the end of this warp's range ----
    const int j_end = cur.j0 + kw_i + 1;
    if (j_end == cur.nblk || cpos == n_total) {
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
      const long long u = (long long)cur.s * HG + cur.hg;
      if (seg_j0 == 0 && j_end == cur.nblk) {
        // the whole unit was processed by this warp: write the output
        if (tg == 0) {
#pragma unroll
          for (int hh = 0; hh < GT; ++hh) {
            const float inv = l_run[hh] > 0.f ? 1.f / l_run[hh] : 0.f;
            __half2* o = reinterpret_cast<__half2*>(
                p.out + ((size_t)cur.s * p.num_q_heads + (size_t)cur.hg * GT + hh) * D + c * 16);
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = __floats2half2_rn(acc[hh][j].x * inv, acc[hh][j].y * inv);
          }
        }
      } else {
        // one segment of a split unit: publish the partial; the last warp to finish merges
        const long long slot = u + w;
        if (tg == 0) {
#pragma unroll
          for (int hh = 0; hh < GT; ++hh) {
            float4* dst = reinterpret_cast<float4*>(p.ws_acc + ((size_t)slot * GT + hh) * D + c * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_float4(acc[hh][2 * j].x, acc[hh][2 * j].y, acc[hh][2 * j + 1].x, acc[hh][2 * j + 1].y);
          }
        }
        if (lane == 0) {
#pragma unroll
          for (int hh = 0; hh < GT; ++hh) {
            p.ws_ml[((size_t)slot * GT + hh) * 2 + 0] = m_run[hh];
            p.ws_ml[((size_t)slot * GT + hh) * 2 + 1] = l_run[hh];
          }
        }
        const long long unit_p0 = cur.seq_p0 + (long long)cur.hg * cur.nblk;
        const int w_first = owner_of(unit_p0, T, We);
        const int w_last = owner_of(unit_p0 + cur.nblk - 1, T, We);
        const uint32_t n_seg = (uint32_t)(w_last - w_first + 1);
        __syncwarp();  // the warp's partial writes precede lane 0's release below
        uint32_t ticket = 0;
        if (lane == 0) ticket = atomic_inc_acq_rel_gpu(&p.ws_count[u], n_seg - 1);
        ticket = __shfl_sync(kFull, ticket, 0);
        if (ticket == n_seg - 1) {
          for (int o = lane; o < GT * D; o += 32) {
            const int hh = o / D, d = o % D;
            float M = kNegBig;
            for (int wi = w_first; wi <= w_last; ++wi)
              M = fmaxf(M, __ldcg(&p.ws_ml[((size_t)(u + wi) * GT + hh) * 2]));
            float Ls = 0.f, A = 0.f;
            for (int wi = w_first; wi <= w_last; ++wi) {
              const size_t sl = (size_t)(u + wi) * GT + hh;
              const float e = ex2(__ldcg(&p.ws_ml[sl * 2]) - M);
              Ls = fmaf(__ldcg(&p.ws_ml[sl * 2 + 1]), e, Ls);
              A = fmaf(__ldcg(&p.ws_acc[sl * D + d]), e, A);
            }
            p.out[((size_t)cur.s * p.num_q_heads + (size_t)cur.hg * GT + hh) * D + d] =
                __float2half_rn(Ls > 0.f ? A / Ls : 0.f);
          }
        }
      }
#pragma unroll
      for (int hh = 0; hh < GT; ++hh) {
        m_run[hh] = kNegBig;
        l_run[hh] = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[hh][j] = make_float2(0.f, 0.f);
      }
      seg_j0 = j_end;  // (a new unit restarts it at its first block)
    }
  }

  if (aborted && lane == 0) {
    // A copy never completed (outputs touched by this warp are unspecified; dev_error says so).
    // Wait, again bounded, for the copies this warp issued and did not consume, so that no bulk
    // copy is still writing this CTA's shared memory when it exits.
    for (int k = cpos; k < ipos; ++k) (void)mbar_wait_bounded(&my_bars[k % C::NS], (uint32_t)((k / C::NS) & 1));
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
  // programmatic dependent launch: the kernel may start while the previous kernel in the stream
  // finishes; it waits for it (griddepcontrol.wait) before reading the pool
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sh.grid_ctas);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
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

// FN<KT, VT, BS, D, GT>(args...) for the instantiation matching `sh`
#define PKV_DISPATCH_GT(KT, VT, BS, D, FN, ...)       \
  switch (sh.heads_per_warp) {                        \
    case 1: return FN<KT, VT, BS, D, 1>(__VA_ARGS__); \
    case 2: return FN<KT, VT, BS, D, 2>(__VA_ARGS__); \
    case 4: return FN<KT, VT, BS, D, 4>(__VA_ARGS__); \
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
#define PKV_DISPATCH(FN, ...)                                                \
  if (sh.k_dtype == PKV_INT8_SYM && sh.v_dtype == PKV_INT8_SYM) {            \
    PKV_DISPATCH_BS(PKV_INT8_SYM, PKV_INT8_SYM, FN, __VA_ARGS__)             \
  } else if (sh.k_dtype == PKV_INT8_SYM && sh.v_dtype == PKV_INT4_ASYM) {    \
    PKV_DISPATCH_BS(PKV_INT8_SYM, PKV_INT4_ASYM, FN, __VA_ARGS__)            \
  } else if (sh.k_dtype == PKV_FP16 && sh.v_dtype == PKV_FP16) {             \
    PKV_DISPATCH_BS(PKV_FP16, PKV_FP16, FN, __VA_ARGS__)                     \
  }

}  // namespace

int32_t decode_heads_per_warp(int32_t group) {
  if (group % 4 == 0) return 4;
  if (group % 2 == 0) return 2;
  return 1;
}

bool decode_supported(int32_t k_dtype, int32_t v_dtype, int32_t block_size, int32_t head_dim) {
  const bool dt = (k_dtype == PKV_INT8_SYM && (v_dtype == PKV_INT8_SYM || v_dtype == PKV_INT4_ASYM)) ||
                  (k_dtype == PKV_FP16 && v_dtype == PKV_FP16);
  return dt && (block_size == 16 || block_size == 32) && (head_dim == 64 || head_dim == 128 || head_dim == 256);
}

bool decode_kernel_info(const DecodeShape& sh, DecodeKernelInfo* info) {
  PKV_DISPATCH(info_one, info)
  return false;
}

cudaError_t launch_decode(const DecodeParams& p, const DecodeShape& sh, cudaStream_t stream) {
  PKV_DISPATCH(launch_one, p, sh, stream)
  return cudaErrorInvalidValue;
}

}  // namespace pkv
