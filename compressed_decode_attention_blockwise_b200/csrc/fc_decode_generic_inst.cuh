// Explicit instantiation body of the generic decode launcher for one (K, V)
// coefficient type pair; included by the small fc_decode_generic_*.cu units so
// that the template instantiations compile in parallel.
#pragma once

#include "fc_decode.cuh"

namespace fc {

template <typename KT, typename VT>
int launch_decode_generic(const DecodeArgs& a, const Basis& basis, cudaStream_t stream) {
  const dim3 grid(unsigned(a.ns), unsigned(a.Hk), unsigned(a.B));
  const size_t smem = generic_dyn_smem(a.G, a.D, a.ns);
  auto go = [&](auto kernel) -> int {
    if (smem > 32 * 1024) {
      const cudaError_t e =
          cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      if (e != cudaSuccess) return FC_ERR_CUDA;
    }
    kernel<<<grid, kGenericWarps * 32, smem, stream>>>(a, basis);
    return cuda_status(cudaGetLastError());
  };
#define FC_G_CASES(VEC)                                                         \
  switch (a.G) {                                                                \
    case 1: return go(decode_generic_kernel<VEC, 1, KT, VT>);                   \
    case 2: return go(decode_generic_kernel<VEC, 2, KT, VT>);                   \
    case 4: return go(decode_generic_kernel<VEC, 4, KT, VT>);                   \
    case 8: return go(decode_generic_kernel<VEC, 8, KT, VT>);                   \
    case 16:                                                                    \
      if constexpr (VEC * 16 <= 64) return go(decode_generic_kernel<VEC, 16, KT, VT>); \
      return FC_ERR_UNSUPPORTED;                                                \
    default: return FC_ERR_UNSUPPORTED;                                         \
  }
  switch (a.D) {
    case 32: { FC_G_CASES(1) }
    case 64: { FC_G_CASES(2) }
    case 128: { FC_G_CASES(4) }
    case 256: { FC_G_CASES(8) }
    default: return FC_ERR_UNSUPPORTED;
  }
#undef FC_G_CASES
}

}  // namespace fc
