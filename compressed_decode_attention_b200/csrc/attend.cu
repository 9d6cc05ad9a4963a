// tq_attend's dispatch on the head dimension. The kernel, its design and
// its citations are in attend_kernel.cuh (one instantiation unit per d).
#include "tq_internal.h"

namespace tq {

cudaError_t launch_attend(const AttendArgs& a, const Codebook& cbk,
                          const Codebook& cbv, const SignMask& sm, int n_ctas,
                          cudaStream_t stream) {
  if (n_ctas > kMaxCtas) return cudaErrorInvalidValue;
  switch (a.d) {
    case 64: return launch_attend_d<64>(a, cbk, cbv, sm, n_ctas, stream);
    case 128: return launch_attend_d<128>(a, cbk, cbv, sm, n_ctas, stream);
    case 256: return launch_attend_d<256>(a, cbk, cbv, sm, n_ctas, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tq
