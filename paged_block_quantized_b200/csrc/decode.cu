// decode.cu -- the decode entry points behind the C ABI: heads per warp, supported shapes, and the
// dispatch to the kernel instantiations of each dtype pair (decode_i8i8.cu, decode_i8i4.cu,
// decode_f16.cu, decode_fp8.cu; the kernel itself is in decode_kernel.cuh).
#include <cudaTypedefs.h>

#include "internal.h"

namespace pkv {

bool encode_tile_map(CUtensorMap* map, const void* base, uint64_t rows, int row_bytes, int box_rows) {
  // the driver's encoder, looked up once through the runtime (no link against the driver library)
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if (row_bytes % 128 != 0 || row_bytes / 128 > 8 || box_rows <= 0 || box_rows > 256) return false;
  if (rows > (uint64_t)INT32_MAX) return false;  // the copies address rows with a signed 32-bit coordinate
  const cuuint32_t units = (cuuint32_t)(row_bytes / 128);
  const cuuint32_t rank = units == 1 ? 2 : 3;
  // innermost: 128 bytes; then (3-D only) the 128-byte units of a row; then the rows
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  dims[0] = 128;
  box[0] = 128;
  if (rank == 2) {
    dims[1] = rows;
    strides[0] = 128;
    box[1] = (cuuint32_t)box_rows;
  } else {
    dims[1] = units;
    dims[2] = rows;
    strides[0] = 128;
    strides[1] = (cuuint64_t)row_bytes;
    box[1] = units;
    box[2] = (cuuint32_t)box_rows;
  }
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int32_t decode_heads_per_warp(int32_t group, int32_t k_dtype, int32_t v_dtype, int32_t head_dim) {
  const bool mma = (k_dtype == PKV_INT8_SYM && (v_dtype == PKV_INT8_SYM || v_dtype == PKV_INT4_ASYM) && head_dim >= 128) ||
                   (k_dtype == PKV_FP16 && v_dtype == PKV_FP16) || (k_dtype == PKV_FP8_E4M3 && v_dtype == PKV_FP8_E4M3);
  if (mma && group % 8 == 0) return 8;
  if (group % 4 == 0) return 4;
  if (group % 2 == 0) return 2;
  return 1;
}

bool decode_supported(int32_t k_dtype, int32_t v_dtype, int32_t block_size, int32_t head_dim) {
  const bool dt = (k_dtype == PKV_INT8_SYM && (v_dtype == PKV_INT8_SYM || v_dtype == PKV_INT4_ASYM)) ||
                  (k_dtype == PKV_FP16 && v_dtype == PKV_FP16) ||
                  (k_dtype == PKV_FP8_E4M3 && v_dtype == PKV_FP8_E4M3 && head_dim >= 128);
  return dt && (block_size == 16 || block_size == 32) && (head_dim == 64 || head_dim == 128 || head_dim == 256);
}

bool decode_kernel_info(const DecodeShape& sh, DecodeKernelInfo* info) {
  if (sh.k_dtype == PKV_INT8_SYM && sh.v_dtype == PKV_INT8_SYM) return decode_info_i8i8(sh, info);
  if (sh.k_dtype == PKV_INT8_SYM && sh.v_dtype == PKV_INT4_ASYM) return decode_info_i8i4(sh, info);
  if (sh.k_dtype == PKV_FP16 && sh.v_dtype == PKV_FP16) return decode_info_f16(sh, info);
  if (sh.k_dtype == PKV_FP8_E4M3 && sh.v_dtype == PKV_FP8_E4M3) return decode_info_fp8(sh, info);
  return false;
}

namespace {
cudaError_t launch_any(const DecodeParams& p, const StepParams& sp, const DecodeShape& sh, cudaStream_t stream) {
  if (sh.k_dtype == PKV_INT8_SYM && sh.v_dtype == PKV_INT8_SYM) return launch_decode_i8i8(p, sp, sh, stream);
  if (sh.k_dtype == PKV_INT8_SYM && sh.v_dtype == PKV_INT4_ASYM) return launch_decode_i8i4(p, sp, sh, stream);
  if (sh.k_dtype == PKV_FP16 && sh.v_dtype == PKV_FP16) return launch_decode_f16(p, sp, sh, stream);
  if (sh.k_dtype == PKV_FP8_E4M3 && sh.v_dtype == PKV_FP8_E4M3) return launch_decode_fp8(p, sp, sh, stream);
  return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_decode(const DecodeParams& p, const DecodeShape& sh, cudaStream_t stream) {
  if (gqa_tc_eligible(sh, p.num_seqs, p.num_q_heads)) {
    DecodeKernelInfo info;
    if (!decode_kernel_info(sh, &info)) return cudaErrorInvalidValue;
    return launch_gqa_tc(p, sh, (int64_t)sh.grid_ctas * info.warps_per_cta, stream);
  }
  StepParams sp = {};
  sp.fused = 0;
  return launch_any(p, sp, sh, stream);
}

cudaError_t launch_decode_step(const DecodeParams& p, const StepParams& sp, const DecodeShape& sh,
                               cudaStream_t stream) {
  return launch_any(p, sp, sh, stream);
}

}  // namespace pkv
