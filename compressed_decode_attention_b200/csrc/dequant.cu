// tq_dequant kernel (verification path): packed rows -> float vectors.
//   domain 1: c[idx] / sqrt(d)                 (rotated unit vector)
//   domain 0: n · D ⊙ (H · c[idx]) / d         (original space)
// Same thread layout as the encoder: d/32 lanes per vector, 32 coordinates
// per lane, 256/(d/32) tokens of one kv head per 256-thread block. Levels
// come from a shared-memory copy of the codebook; each warp's rows are
// staged in shared memory and stored whole.
#include "encode_common.cuh"

namespace tq {
namespace {

constexpr int kDqThreads = 256;

// Levels of the lane's 32 fields, read from the shared-memory copy of the
// codebook.
template <int BITS>
__device__ __forceinline__ void unpack_lane(const uint8_t* row, int sub, const float* levels,
                                            float (&c)[32]) {
  uint32_t w[BITS + 1];
  const uint32_t* src = reinterpret_cast<const uint32_t*>(row + 4 * BITS * sub);
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] = src[k];
  w[BITS] = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) c[i] = levels[field<BITS>(w, i)];
}

template <int D>
__global__ void __launch_bounds__(kDqThreads)
dequant_kernel(const __grid_constant__ DequantArgs a,
               const __grid_constant__ Codebook cb,
               const __grid_constant__ SignMask sm) {
  constexpr int LPV = D / 32;
  constexpr int kWarpTok = 32 / LPV;         // tokens per warp
  constexpr int kChunks = D / 4;             // 16-byte chunks per output row
  // The codebook's levels in shared memory: a warp's lookups of distinct
  // levels fall in distinct banks and take one pass (a kernel parameter
  // indexed per lane is read once per distinct address).
  __shared__ float levels[kMaxLevels];
  // Each warp's output rows (its tokens are consecutive, so their rows are
  // one contiguous range of the output), staged so that the warp stores
  // them 512 contiguous bytes per instruction.
  __shared__ __align__(16) float4 stage[kDqThreads / 32][32 * 8];
  if (threadIdx.x < kMaxLevels) levels[threadIdx.x] = cb.centroid[threadIdx.x];
  __syncthreads();

  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane & (LPV - 1), t = lane / LPV;
  const int tok0 = blockIdx.x * (kDqThreads / LPV) + warp * kWarpTok;
  const int tok = tok0 + t;
  const bool valid = tok < a.n_tok;
  const unsigned gmask = ((1u << LPV) - 1u) << (lane & ~(LPV - 1));
  const size_t row = (size_t)h * a.cap_tok + (valid ? tok : 0);
  float c[32];
  if (valid) {
    const uint8_t* src = a.packed + row * (D * a.bits / 8);
    if (a.bits == 4) unpack_lane<4>(src, sub, levels, c);
    else if (a.bits == 3) unpack_lane<3>(src, sub, levels, c);
    else unpack_lane<2>(src, sub, levels, c);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) c[i] = 0.f;
  }

  // y_i = c_i · scale_i: scale_i = 1/sqrt(d) in the rotated domain; in the
  // original space c = H·c[idx] (the encoder's butterflies, two-wide) and
  // scale_i = D_i · n / d (a sign flip commutes exactly with the product)
  if (a.domain == 1) {
    // 1/sqrt(d), correctly rounded
    const float scale = D == 64 ? 0.125f : D == 128 ? 0.0883883476483184405501f : 0.0625f;
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 y = f2mul(make_float2(c[i], c[i + 1]), make_float2(scale, scale));
      c[i] = y.x;
      c[i + 1] = y.y;
    }
  } else {
    rotate_vector<LPV>(c, sub, gmask);
    const uint32_t m = sm.w[sub];
    const float scale = valid ? __half2float(__ushort_as_half(a.norms[row])) / (float)D : 0.f;
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 y = f2mul(make_float2(c[i], c[i + 1]),
                             make_float2(apply_sign(scale, m, i), apply_sign(scale, m, i + 1)));
      c[i] = y.x;
      c[i + 1] = y.y;
    }
  }
  // Chunk q = 8·sub + k of token t's row sits at q ^ s, s = lane & 7: the
  // eight lanes of each quarter-warp store to eight different bank groups,
  // and eight consecutive chunks of a row (one writer) are read back from
  // eight different bank groups.
  float4* st = stage[warp];
  const int s = lane & 7;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    st[t * kChunks + ((8 * sub + k) ^ s)] =
        make_float4(c[4 * k], c[4 * k + 1], c[4 * k + 2], c[4 * k + 3]);
  __syncwarp();
  float4* dst = reinterpret_cast<float4*>(a.out + ((size_t)h * a.n_tok + tok0) * D);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int g = 32 * j + lane;             // chunk of the warp's rows
    const int tt = g / kChunks, q = g % kChunks;
    const int sw = (tt * LPV + (q >> 3)) & 7;     // the writer's lane & 7
    if (tok0 + tt < a.n_tok) dst[g] = st[tt * kChunks + (q ^ sw)];
  }
}

}  // namespace

cudaError_t launch_dequant(const DequantArgs& a, const Codebook& cb,
                           const SignMask& sm, cudaStream_t stream) {
  const int tokens = kDqThreads / (a.d / 32);
  dim3 grid((a.n_tok + tokens - 1) / tokens, a.n_kv_heads, 1);
  switch (a.d) {
    case 64: dequant_kernel<64><<<grid, kDqThreads, 0, stream>>>(a, cb, sm); break;
    case 128: dequant_kernel<128><<<grid, kDqThreads, 0, stream>>>(a, cb, sm); break;
    case 256: dequant_kernel<256><<<grid, kDqThreads, 0, stream>>>(a, cb, sm); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace tq
