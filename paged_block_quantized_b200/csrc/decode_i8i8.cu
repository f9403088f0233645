// decode_i8i8.cu -- the decode kernel's instantiations for INT8 K / INT8 V (one translation unit per
// dtype pair, so that they compile in parallel). The kernel is in decode_kernel.cuh.
#include "decode_kernel.cuh"

namespace pkv {

cudaError_t launch_decode_i8i8(const DecodeParams& p, const StepParams& sp, const DecodeShape& sh, cudaStream_t stream) {
  PKV_DISPATCH_BS(PKV_INT8_SYM, PKV_INT8_SYM, launch_one, p, sp, sh, stream)
  return cudaErrorInvalidValue;
}

bool decode_info_i8i8(const DecodeShape& sh, DecodeKernelInfo* info) {
  PKV_DISPATCH_BS(PKV_INT8_SYM, PKV_INT8_SYM, info_one, info)
  return false;
}

}  // namespace pkv
