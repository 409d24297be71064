// Generic decode attention kernels for K coefficients of type float and V
// coefficients of type float.
#include "fc_decode_generic_inst.cuh"

namespace fc {
template int launch_decode_generic<float, float>(const DecodeArgs&, const Basis&, cudaStream_t);
}  // namespace fc
