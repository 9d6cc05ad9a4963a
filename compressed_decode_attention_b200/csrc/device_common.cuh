// Device helpers shared by the kernels: 16-bit loads, sign flips, the
// in-register part of the Walsh-Hadamard transform, bit-field access.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tq.h"
#include "tq_internal.h"

namespace tq {

__device__ __forceinline__ float2 unpack16x2(uint32_t w, bool bf16) {
  if (bf16) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
  __half2 h = *reinterpret_cast<__half2*>(&w);
  return __half22float2(h);
}

// Multiply x by D_i in {+1,-1}: flip the sign bit where bit i of m is set.
__device__ __forceinline__ float apply_sign(float x, uint32_t m, int i) {
  return __uint_as_float(__float_as_uint(x) ^ (((m >> i) & 1u) << 31));
}

// Unnormalized Walsh-Hadamard butterflies over N contiguous registers
// (strides 1 .. N/2). Sylvester (natural) order.
template <int N>
__device__ __forceinline__ void fwht_registers(float (&x)[N]) {
#pragma unroll
  for (int s = 1; s < N; s <<= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if ((i & s) == 0) {
        const float a = x[i], b = x[i + s];
        x[i] = a + b;
        x[i + s] = a - b;
      }
    }
  }
}

// One butterfly stage across lanes: partner = lane ^ lane_bit. The lane whose
// bit is clear keeps a + b, the other keeps a - b (a = lower lane's value).
template <int N>
__device__ __forceinline__ void fwht_cross_lane(float (&x)[N], unsigned mask,
                                                int lane_bit, bool upper) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float p = __shfl_xor_sync(mask, x[i], lane_bit);
    x[i] = upper ? (p - x[i]) : (x[i] + p);
  }
}

// Field i of a little-endian bit stream of BITS-bit fields held in words w.
template <int BITS>
__device__ __forceinline__ uint32_t field(const uint32_t* w, int i) {
  const int p = i * BITS;
  const int k = p >> 5, off = p & 31;
  uint32_t v = w[k] >> off;
  if (off + BITS > 32) v |= w[k + 1] << (32 - off);
  return v & ((1u << BITS) - 1u);
}

__device__ __forceinline__ uint16_t f32_to_f16_bits(float x) {
  return __half_as_ushort(__float2half_rn(x));
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

}  // namespace tq
