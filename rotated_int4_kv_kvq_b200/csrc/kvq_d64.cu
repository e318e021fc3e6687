// Kernels and launchers for vectors of length d = 64.
#include "kvq_inst.cuh"

namespace kvq {
template cudaError_t launch_fwd<64>(int, int, const FwdLaunch&);
template cudaError_t launch_inv<64>(int, int, const InvLaunch&);
template cudaError_t launch_decode<64>(int, int, const DecodeLaunch&);
template cudaError_t launch_decode_wide<64>(int, int, const DecodeWideLaunch&);
template cudaError_t launch_window<64>(int, int, const WindowLaunch&);
template cudaError_t launch_attn<64>(int, int, const AttnLaunch&);
template cudaError_t read_status<64>(uint32_t*, bool);
}  // namespace kvq
