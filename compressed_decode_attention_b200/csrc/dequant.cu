// tq_dequant kernel (verification path): packed rows -> float vectors.
//   domain 1: c[idx] / sqrt(d)                 (rotated unit vector)
//   domain 0: n · D ⊙ (H · c[idx]) / d         (original space)
// Same thread layout as the encoder: four lanes per vector, 32 coordinates
// per lane, 64 tokens of one kv head per 256-thread block.
#include "device_common.cuh"

namespace tq {
namespace {

constexpr int kDqThreads = 256;
constexpr int kDqTokens = kDqThreads / 4;

template <int BITS>
__device__ __forceinline__ void unpack_lane(const uint8_t* row, int sub,
                                            const Codebook& cb, float (&c)[32]) {
  uint32_t w[BITS + 1];
  const uint32_t* src = reinterpret_cast<const uint32_t*>(row + 4 * BITS * sub);
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] = src[k];
  w[BITS] = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) c[i] = cb.centroid[field<BITS>(w, i)];
}

__global__ void __launch_bounds__(kDqThreads)
dequant_kernel(const __grid_constant__ DequantArgs a,
               const __grid_constant__ Codebook cb,
               const __grid_constant__ SignMask sm) {
  const int h = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;
  const int tok = blockIdx.x * kDqTokens + (threadIdx.x >> 2);
  if (tok >= a.n_tok) return;
  const unsigned gmask = 0xFu << (lane & ~3);
  const size_t row = (size_t)h * a.cap_tok + tok;
  const uint8_t* src = a.packed + row * (kHeadDim * a.bits / 8);
  float c[32];
  if (a.bits == 4) unpack_lane<4>(src, sub, cb, c);
  else if (a.bits == 3) unpack_lane<3>(src, sub, cb, c);
  else unpack_lane<2>(src, sub, cb, c);

  float scale;
  if (a.domain == 1) {
    scale = 0.0883883476483184405501f;   // 1/sqrt(128), correctly rounded
  } else {
    fwht_registers<32>(c);
    fwht_cross_lane<32>(c, gmask, 1, (sub & 1) != 0);
    fwht_cross_lane<32>(c, gmask, 2, (sub & 2) != 0);
    const uint32_t m = sm.w[sub];
#pragma unroll
    for (int i = 0; i < 32; ++i) c[i] = apply_sign(c[i], m, i);
    scale = __half2float(__ushort_as_half(a.norms[row])) / (float)kHeadDim;
  }
  float4* dst = reinterpret_cast<float4*>(a.out + ((size_t)h * a.n_tok + tok) * kHeadDim + 32 * sub);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    dst[k] = make_float4(c[4 * k] * scale, c[4 * k + 1] * scale,
                         c[4 * k + 2] * scale, c[4 * k + 3] * scale);
}

}  // namespace

cudaError_t launch_dequant(const DequantArgs& a, const Codebook& cb,
                           const SignMask& sm, cudaStream_t stream) {
  dim3 grid((a.n_tok + kDqTokens - 1) / kDqTokens, a.n_kv_heads, 1);
  dequant_kernel<<<grid, kDqThreads, 0, stream>>>(a, cb, sm);
  return cudaGetLastError();
}

}  // namespace tq
