// Generic decode attention kernels for K coefficients of type int8_t and V
// coefficients of type int8_t.
#include "fc_decode_generic_inst.cuh"

namespace fc {
template int launch_decode_generic<int8_t, int8_t>(const DecodeArgs&, const Basis&, cudaStream_t);
}  // namespace fc
