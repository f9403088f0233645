// decode_fp8.cu -- the decode kernel's instantiations for E4M3 K and V (one translation unit per
// dtype pair, so that they compile in parallel). E4M3 tiles always take the tensor-core engine,
// whose 128-byte swizzled tiles need rows of 128 bytes or more: head_dim 128 and 256 only. The
// kernel is in decode_kernel.cuh.
#include "decode_kernel.cuh"

namespace pkv {

#define PKV_DISPATCH_D_FP8(BS, FN, ...)                                                     \
  switch (sh.head_dim) {                                                                    \
    case 128: PKV_DISPATCH_GT(PKV_FP8_E4M3, PKV_FP8_E4M3, BS, 128, FN, __VA_ARGS__) break;  \
    case 256: PKV_DISPATCH_GT(PKV_FP8_E4M3, PKV_FP8_E4M3, BS, 256, FN, __VA_ARGS__) break;  \
    default: break;                                                                         \
  }

cudaError_t launch_decode_fp8(const DecodeParams& p, const StepParams& sp, const DecodeShape& sh, cudaStream_t stream) {
  switch (sh.block_size) {
    case 16: PKV_DISPATCH_D_FP8(16, launch_one, p, sp, sh, stream) break;
    case 32: PKV_DISPATCH_D_FP8(32, launch_one, p, sp, sh, stream) break;
    default: break;
  }
  return cudaErrorInvalidValue;
}

bool decode_info_fp8(const DecodeShape& sh, DecodeKernelInfo* info) {
  switch (sh.block_size) {
    case 16: PKV_DISPATCH_D_FP8(16, info_one, info) break;
    case 32: PKV_DISPATCH_D_FP8(32, info_one, info) break;
    default: break;
  }
  return false;
}

}  // namespace pkv
