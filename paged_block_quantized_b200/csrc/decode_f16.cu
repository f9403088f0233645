// decode_f16.cu -- the decode kernel's instantiations for FP16 K / FP16 V (one translation unit per
// dtype pair, so that they compile in parallel). The kernel is in decode_kernel.cuh.
#include "decode_kernel.cuh"

namespace pkv {

cudaError_t launch_decode_f16(const DecodeParams& p, const StepParams& sp, const DecodeShape& sh, cudaStream_t stream) {
  PKV_DISPATCH_BS(PKV_FP16, PKV_FP16, launch_one, p, sp, sh, stream)
  return cudaErrorInvalidValue;
}

bool decode_info_f16(const DecodeShape& sh, DecodeKernelInfo* info) {
  PKV_DISPATCH_BS(PKV_FP16, PKV_FP16, info_one, info)
  return false;
}

}  // namespace pkv
