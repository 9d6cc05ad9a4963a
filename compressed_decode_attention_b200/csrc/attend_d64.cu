// Attention kernels for head dimension 64 (all bit-width pairs).
#include "attend_kernel.cuh"

namespace tq {
template cudaError_t launch_attend_d<64>(const AttendArgs&, const Codebook&, const Codebook&,
                                         const SignMask&, int, cudaStream_t);
}  // namespace tq
