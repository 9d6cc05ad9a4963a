// tq_dequant kernel (verification path): packed rows -> float vectors.
//   domain 1: c[idx] / sqrt(d)                 (rotated unit vector)
//   domain 0: n · D ⊙ (H · c[idx]) / d         (original space)
// Same thread layout as the encoder: d/32 lanes per vector, 32 coordinates
// per lane, 256/(d/32) tokens of one kv head per 256-thread block.
#include "device_common.cuh"

namespace tq {
namespace {

constexpr int kDqThreads = 256;

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

template <int D>
__global__ void __launch_bounds__(kDqThreads)
dequant_kernel(const __grid_constant__ DequantArgs a,
               const __grid_constant__ Codebook cb,
               const __grid_constant__ SignMask sm) {
  constexpr int LPV = D / 32;
  const int h = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int sub = lane & (LPV - 1);
  const int tok = blockIdx.x * (kDqThreads / LPV) + threadIdx.x / LPV;
  if (tok >= a.n_tok) return;
  const unsigned gmask = ((1u << LPV) - 1u) << (lane & ~(LPV - 1));
  const size_t row = (size_t)h * a.cap_tok + tok;
  const uint8_t* src = a.packed + row * (D * a.bits / 8);
  float c[32];
  if (a.bits == 4) unpack_lane<4>(src, sub, cb, c);
  else if (a.bits == 3) unpack_lane<3>(src, sub, cb, c);
  else unpack_lane<2>(src, sub, cb, c);

  float scale;
  if (a.domain == 1) {
    // 1/sqrt(d), correctly rounded
    scale = D == 64 ? 0.125f : D == 128 ? 0.0883883476483184405501f : 0.0625f;
  } else {
    fwht_registers<32>(c);
#pragma unroll
    for (int o = 1; o < LPV; o <<= 1) fwht_cross_lane<32>(c, gmask, o, (sub & o) != 0);
    const uint32_t m = sm.w[sub];
#pragma unroll
    for (int i = 0; i < 32; ++i) c[i] = apply_sign(c[i], m, i);
    scale = __half2float(__ushort_as_half(a.norms[row])) / (float)D;
  }
  float4* dst = reinterpret_cast<float4*>(a.out + ((size_t)h * a.n_tok + tok) * D + 32 * sub);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    dst[k] = make_float4(c[4 * k] * scale, c[4 * k + 1] * scale,
                         c[4 * k + 2] * scale, c[4 * k + 3] * scale);
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
