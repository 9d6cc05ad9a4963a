// Attention kernels for head dimension 256 (all bit-width pairs).
#include "attend_kernel.cuh"

namespace tq {
template cudaError_t launch_attend_d<256>(const AttendArgs&, const Codebook&, const Codebook&,
                                         const SignMask&, int, cudaStream_t);
}  // namespace tq
