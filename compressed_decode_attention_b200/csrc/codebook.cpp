// Host-side Lloyd-Max solver for the standard normal, and the cached float
// codebooks the kernels receive as launch parameters.
//
// [TQAI §The Paper] ("We Built a Python Library That Cuts LLM Memory Usage by
// 80%"): after the rotation a coordinate is modelled as N(0, 1/d), so the
// optimal scalar quantizer is computed once, without data. [ADAPTQ §How it
// works, item 2]: scalar quantization with Max-Lloyd codebooks.
//
// Solved in N(0,1) units on the half line x >= 0 (the density is symmetric,
// so the middle threshold of an even number of levels is 0). Alternates
//   level_k     = E[X | b_k <= X < b_{k+1}]  = (phi(b_k) - phi(b_{k+1})) / mass
//   boundary_k  = (level_{k-1} + level_k) / 2
// in long double until no level moves by more than 1e-15.
#include <math.h>

#include <mutex>

#include "tq.h"
#include "tq_internal.h"

namespace tq {
namespace {

typedef long double real;

real normal_density(real x) {
  if (isinf(x)) return 0.0L;
  return expl(-0.5L * x * x) * 0.398942280401432677939946059934381868L;
}

// P(X > x) for x >= 0, without cancellation.
real tail(real x) {
  if (isinf(x)) return 0.0L;
  return 0.5L * erfcl(x * 0.707106781186547524400844362104849039L);
}

}  // namespace

int solve_lloyd_max(int bits, double* centroids, double* thresholds,
                    double* mse) {
  if (bits < 1 || bits > 8 || !centroids || !thresholds) return TQ_ERR_INVALID_ARG;
  const int levels = 1 << bits;
  const int half = levels / 2;
  real lev[128], bnd[129];  // positive half: bnd[0] = 0 ... bnd[half] = inf
  // Start: levels spread evenly in probability over the half line, using the
  // upper tail inverted by bisection.
  for (int k = 0; k < half; ++k) {
    const real target = 0.5L - 0.5L * (k + 0.5L) / half;  // P(X > level)
    real lo = 0.0L, hi = 40.0L;
    for (int it = 0; it < 200; ++it) {
      const real mid = 0.5L * (lo + hi);
      if (tail(mid) > target) lo = mid; else hi = mid;
    }
    lev[k] = 0.5L * (lo + hi);
  }
  bnd[0] = 0.0L;
  bnd[half] = INFINITY;
  bool converged = false;
  for (int it = 0; it < 1000000 && !converged; ++it) {
    for (int k = 1; k < half; ++k) bnd[k] = 0.5L * (lev[k - 1] + lev[k]);
    real move = 0.0L;
    for (int k = 0; k < half; ++k) {
      const real mass = tail(bnd[k]) - tail(bnd[k + 1]);
      const real next = (normal_density(bnd[k]) - normal_density(bnd[k + 1])) / mass;
      const real dk = fabsl(next - lev[k]);
      if (dk > move) move = dk;
      lev[k] = next;
    }
    converged = move < 1e-15L;
  }
  if (!converged) return TQ_ERR_NO_CONVERGENCE;
  for (int k = 1; k < half; ++k) bnd[k] = 0.5L * (lev[k - 1] + lev[k]);
  for (int k = 0; k < half; ++k) {
    centroids[half + k] = (double)lev[k];
    centroids[half - 1 - k] = -(double)lev[k];
  }
  thresholds[half - 1] = 0.0;
  for (int k = 1; k < half; ++k) {
    thresholds[half - 1 + k] = (double)bnd[k];
    thresholds[half - 1 - k] = -(double)bnd[k];
  }
  if (mse) {
    // E[X^2] - sum_j P_j c_j^2, which equals the distortion at a centroid
    // fixed point (E[X·Q(X)] = E[Q(X)^2]); both halves contribute equally.
    real kept = 0.0L;
    for (int k = 0; k < half; ++k)
      kept += (tail(bnd[k]) - tail(bnd[k + 1])) * lev[k] * lev[k];
    *mse = (double)(1.0L - 2.0L * kept);
  }
  return TQ_OK;
}

const Codebook* codebook_for(int bits) {
  static Codebook books[5];
  static int status[5];
  static std::once_flag once[5];
  if (bits < 1 || bits > 4) return nullptr;
  std::call_once(once[bits], [bits] {
    double c[16], t[15];
    status[bits] = solve_lloyd_max(bits, c, t, nullptr);
    Codebook& b = books[bits];
    b.bits = bits;
    for (int j = 0; j < kMaxLevels; ++j) {
      b.centroid[j] = j < (1 << bits) ? (float)c[j] : 0.0f;
      b.threshold[j] = j < (1 << bits) - 1 ? (float)t[j] : INFINITY;
    }
  });
  return status[bits] == TQ_OK ? &books[bits] : nullptr;
}

// SplitMix64 (Steele, Lea & Flood 2014): state starts at the seed; output i
// decides D_i (negative iff its top bit is set).
SignMask sign_mask(uint64_t seed) {
  SignMask m{};
  uint64_t state = seed;
  for (int i = 0; i < kMaxHeadDim; ++i) {   // d-bit masks are prefixes
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    if (z >> 63) m.w[i / 32] |= 1u << (i % 32);
  }
  return m;
}

}  // namespace tq
