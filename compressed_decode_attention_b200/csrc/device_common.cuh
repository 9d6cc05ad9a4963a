// Device helpers shared by the kernels: 16-bit loads, sign flips, the
// in-register part of the Walsh-Hadamard transform, bit-field access.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tq.h"
#include "tq_internal.h"

namespace tq {

// Index check of the bounds-checked build (compiled with TQ_DEBUG): a failed
// check sets TQ_DEV_DEBUG_CHECK and the caller skips the access (no trap: the
// context stays usable). Without TQ_DEBUG every check is the constant true.
__device__ __forceinline__ bool tq_check(bool ok, int* dev_status) {
#ifdef TQ_DEBUG
  if (!ok && dev_status) atomicOr(dev_status, TQ_DEV_DEBUG_CHECK);
  return ok;
#else
  (void)ok;
  (void)dev_status;
  return true;
#endif
}

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

namespace tq {

// Packed two-wide fp32 arithmetic (sm_100: add/sub/fma .f32x2), round to
// nearest per lane: bit-identical to the scalar operations.
__device__ __forceinline__ float2 f2add(float2 a, float2 b) {
  float2 r;
  asm("{.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;}\n"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 f2sub(float2 a, float2 b) {
  float2 r;
  asm("{.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;}\n"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 f2mul(float2 a, float2 b) {
  float2 r;
  asm("{.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;}\n"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}\n"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

// sat(a·b + c): the fused multiply-add clamped to [0, 1] (one rounding).
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 0xFFFFFFFF if a >= b else 0 (one compare-and-set).
__device__ __forceinline__ uint32_t set_ge(float a, float b) {
  uint32_t r;
  asm("set.ge.u32.f32 %0, %1, %2;\n" : "=r"(r) : "f"(a), "f"(b));
  return r;
}

}  // namespace tq
