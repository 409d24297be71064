// Generic decode attention kernels for K coefficients of type __nv_bfloat16 and V
// coefficients of type __nv_bfloat16.
#include "fc_decode_generic_inst.cuh"

namespace fc {
template int launch_decode_generic<__nv_bfloat16, __nv_bfloat16>(const DecodeArgs&, const Basis&, cudaStream_t);
}  // namespace fc
