// store.cu -- the store kernel: quantize new K/V tokens and scatter them into pool blocks
// (sm_100a). The arithmetic and its sources are in store_impl.cuh.
//
// Work split: one warp per (token, KV head); a CTA holds the 4 heads of one token.
#include "store_impl.cuh"

namespace pkv {

namespace {

constexpr int kWarpsPerCta = 4;

template <int KT, int VT>
__global__ void __launch_bounds__(32 * kWarpsPerCta) store_quantized_kernel(const StoreParams p) {
  // a kernel launched after this one with programmatic serialization (the decode) may begin its
  // set-up now; it waits for this grid to complete before it reads the pool
  asm volatile("griddepcontrol.launch_dependents;");
  __shared__ __align__(16) uint8_t tables[kWarpsPerCta][256];  // per warp: a rebuild's code table
  store_detail::store_job<KT, VT>(p, blockIdx.x, blockIdx.y * kWarpsPerCta + (threadIdx.x >> 5), threadIdx.x & 31,
                                  tables[threadIdx.x >> 5]);
}

}  // namespace

cudaError_t launch_store(const StoreParams& p, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  dim3 grid(p.T, (p.num_kv_heads + kWarpsPerCta - 1) / kWarpsPerCta);
  const dim3 block(32 * kWarpsPerCta);
  if (p.k_dtype == PKV_INT8_SYM && p.v_dtype == PKV_INT8_SYM)
    store_quantized_kernel<PKV_INT8_SYM, PKV_INT8_SYM><<<grid, block, 0, stream>>>(p);
  else if (p.k_dtype == PKV_INT8_SYM && p.v_dtype == PKV_INT4_ASYM)
    store_quantized_kernel<PKV_INT8_SYM, PKV_INT4_ASYM><<<grid, block, 0, stream>>>(p);
  else if (p.k_dtype == PKV_INT8_SYM && p.v_dtype == PKV_FP16)
    store_quantized_kernel<PKV_INT8_SYM, PKV_FP16><<<grid, block, 0, stream>>>(p);
  else if (p.k_dtype == PKV_FP16 && p.v_dtype == PKV_INT8_SYM)
    store_quantized_kernel<PKV_FP16, PKV_INT8_SYM><<<grid, block, 0, stream>>>(p);
  else if (p.k_dtype == PKV_FP8_E4M3 && p.v_dtype == PKV_FP8_E4M3)
    store_quantized_kernel<PKV_FP8_E4M3, PKV_FP8_E4M3><<<grid, block, 0, stream>>>(p);
  else if (p.k_dtype == PKV_FP16 && p.v_dtype == PKV_INT4_ASYM)
    store_quantized_kernel<PKV_FP16, PKV_INT4_ASYM><<<grid, block, 0, stream>>>(p);
  else
    store_quantized_kernel<PKV_FP16, PKV_FP16><<<grid, block, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
