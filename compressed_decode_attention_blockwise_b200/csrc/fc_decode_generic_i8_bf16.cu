// Generic decode attention kernels for K coefficients of type int8_t and V
// coefficients of type __nv_bfloat16.
#include "fc_decode_generic_inst.cuh"

namespace fc {
template int launch_decode_generic<int8_t, __nv_bfloat16>(const DecodeArgs&, const Basis&, cudaStream_t);
}  // namespace fc
