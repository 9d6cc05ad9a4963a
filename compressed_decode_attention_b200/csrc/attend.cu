// tq_attend: decode attention over the packed cache in one persistent,
// load-balanced kernel on the B200 tensor cores. The kernel template is in
// attend_kernel.cuh; this file dispatches on the head dimension.
//
// [ADAPTQ §How it works, item 3]: the query is rotated once; scores are
// formed from the packed indices through the codebook, without materializing
// the dequantized cache. [TQAI §Test Suite]: the target is
// softmax(Q·K^T/sqrt d)·V. [TQPLUS §2 Sparse V]: V rows with negligible
// weight are left out (block-local rule, include/tq.h).
//
// Work decomposition. The cache is a flat list of 64-position blocks in
// (batch, kv head, block) order; CTA c of Geff owns blocks
// [c·NB/Geff, (c+1)·NB/Geff). Geff = min(grid, #blocks), except that when all
// S (batch, kv head) segments have the same block count and S <= grid, Geff
// is the largest multiple of S within the grid (at most one CTA per block),
// so every CTA stays inside one segment. A CTA walks the (batch, kv head)
// segments of its range. Its 12 warps split each segment in whole blocks,
// merge in shared memory, and
// either write the output (segment = whole sequence) or leave a partial in a
// workspace slot; the last CTA to finish a sequence (atomic counter, no
// waiting) merges the partials and writes the output. No separate combine
// launch, no spin-waits on other CTAs.
//
// Per warp and chunk of up to 64 positions (GQA group of g <= 8 query heads),
// in four 16-position steps:
//   stage   bulk copies (cp.async.bulk, one lane) of the packed K/V rows and
//           fp16 norms into a per-warp ring of shared-memory slots, each
//           completed on its own mbarrier (bounded wait)
//   scores  mma.m16n8k16, fp16 in, fp32 accumulate, per 8 positions: A rows
//           0-7 = K codebook high parts, rows 8-15 = low parts of the same
//           positions (one shared-table entry per packed byte fills two
//           fragment registers); B = rotated query, fp16 high and low parts
//           in the 8 columns (g <= 4: 4 heads x {high, low}; g <= 8: two
//           column tiles). K high, K low and query low are summed, so scores
//           keep ~22 significant bits (fp16-only operands measured up to
//           1.2e-2 output error with x20 outlier channels).
//   softmax fp32, log2 domain; chunk maximum = sparse-V block maximum.
//   PV      mma.m16n8k16: A = V codebook values (fp16), coordinates x
//           positions; B = softmax weight x V norm (fp16), moved from the
//           score layout with movmatrix. V2: position pairs by byte permutes
//           of a 4-entry register table; V3/V4: pair table + movmatrix.
// Output, once per (batch, query head): D⊙(H·(acc/l))/d with shuffles.
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
