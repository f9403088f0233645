// gqa_tc.cu -- launch of the grouped-query decode on the fifth-generation tensor cores
// (gqa_tc.cuh): grid (splits, head groups, sequences), one CTA of 320 threads per SM.
#include <cstring>

#include "gqa_tc.cuh"

// 1: grouped-query decode shapes that gqa_tc.cuh covers use it; 0 (default: measured slower than
// the stream-K kernel's warp-level tensor-core engine on the same shapes): every decode uses the
// persistent stream-K kernel (decode_kernel.cuh)
#ifndef PKV_DECODE_GQA_TC
#define PKV_DECODE_GQA_TC 0
#endif

namespace pkv {

bool gqa_tc_eligible(const DecodeShape& sh, int32_t num_seqs, int32_t num_q_heads) {
  return PKV_DECODE_GQA_TC && sh.k_dtype == PKV_INT8_SYM &&
         (sh.v_dtype == PKV_INT8_SYM || sh.v_dtype == PKV_INT4_ASYM) && sh.head_dim == 128 &&
         sh.heads_per_warp == gqa_tc::kGT && (sh.block_size == 16 || sh.block_size == 32) && num_seqs <= 65535 &&
         num_q_heads / gqa_tc::kGT <= 65535;
}

namespace {

template <int VT, int BS>
cudaError_t launch_t(const DecodeParams& p, int64_t workers, cudaStream_t stream) {
  using C = gqa_tc::Cfg<VT, BS>;
  auto kern = gqa_tc::gqa_decode_tc_kernel<VT, BS>;
  static unsigned long long configured = 0;  // one bit per device; benign race
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!(configured & (1ull << (dev & 63)))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured |= 1ull << (dev & 63);
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // splits per unit: about four waves of one CTA per SM in all, each a whole number of 128-token
  // chunks, and never more partial slots (units x splits) than the workspace holds (units + workers)
  const int64_t HG = p.num_q_heads / gqa_tc::kGT;
  const int64_t units = (int64_t)p.num_seqs * HG;
  const int64_t cap_len = p.max_context_len < (int64_t)p.max_blocks_per_seq * BS ? p.max_context_len
                                                                                 : (int64_t)p.max_blocks_per_seq * BS;
  const int64_t max_blocks = (cap_len + BS - 1) / BS;
  const int64_t chunks = (max_blocks + C::BPC - 1) / C::BPC;
  int64_t splits = (4 * (int64_t)sms + units - 1) / units;
  const int64_t cap = 1 + workers / units;
  if (splits > cap) splits = cap;
  if (splits > chunks) splits = chunks;
  if (splits < 1) splits = 1;
  const int64_t per = (chunks + splits - 1) / splits * C::BPC;
  splits = per > 0 ? (max_blocks + per - 1) / per : 1;
  if (splits < 1) splits = 1;
  if (splits > 65535) return cudaErrorInvalidValue;
  gqa_tc::GqaSplit gs;
  gs.splits = (int32_t)splits;
  gs.per_split = (int32_t)(per > 0 ? per : C::BPC);
  TileMaps tm;
  memset(&tm, 0, sizeof(tm));
  const uint64_t rows = (uint64_t)p.num_blocks * p.num_kv_heads * BS;
  if (!encode_tile_map(&tm.k, p.k_codes, rows, gqa_tc::kD, BS)) return cudaErrorInvalidValue;
  if constexpr (C::V_SWZ) {
    if (!encode_tile_map(&tm.v, p.v_codes, rows, C::V_ROW, BS)) return cudaErrorInvalidValue;
  }
  dim3 grid((unsigned)splits, (unsigned)HG, (unsigned)p.num_seqs);
  kern<<<grid, gqa_tc::kThreads, C::SMEM, stream>>>(p, gs, tm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gqa_tc(const DecodeParams& p, const DecodeShape& sh, int64_t workers, cudaStream_t stream) {
  if (p.num_seqs == 0) return cudaSuccess;
  if (sh.v_dtype == PKV_INT8_SYM) {
    if (sh.block_size == 16) return launch_t<PKV_INT8_SYM, 16>(p, workers, stream);
    if (sh.block_size == 32) return launch_t<PKV_INT8_SYM, 32>(p, workers, stream);
  } else if (sh.v_dtype == PKV_INT4_ASYM) {
    if (sh.block_size == 16) return launch_t<PKV_INT4_ASYM, 16>(p, workers, stream);
    if (sh.block_size == 32) return launch_t<PKV_INT4_ASYM, 32>(p, workers, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pkv
