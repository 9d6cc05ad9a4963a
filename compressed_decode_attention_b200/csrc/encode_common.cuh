// Per-vector encode shared by the encode kernel and the fused decode-step
// append: FP16 norm, randomized Hadamard rotation, Lloyd-Max index and
// LSB-first packing of one d-dimensional vector (d = 32·LPV: 64, 128 or 256)
// held by a group of LPV lanes, 32 consecutive coordinates per lane.
//
// [TQAI §The Paper]: keep the norm in FP16, rotate the unit vector,
// quantize each coordinate with the precomputed Lloyd-Max codebook.
// [ADAPTQ §How it works, item 1]: y = (1/sqrt d)·H·D·x with a fast
// Walsh-Hadamard transform. [TQAI §What's Next]: indices bit-packed at
// 2/3/4 bits.
#pragma once

#include "device_common.cuh"

namespace tq {

// XOR masks that flip the fp16/bf16 sign bits of coordinates 2j (bit 15) and
// 2j+1 (bit 31) of lane `sub`'s 16 half2 words where D = -1.
__device__ __forceinline__ void sign_masks(const SignMask& sm, int sub, uint32_t (&smask)[16]) {
  const uint32_t m = sm.w[sub];
#pragma unroll
  for (int j = 0; j < 16; ++j)
    smask[j] = (((m >> (2 * j)) & 1u) << 15) | (((m >> (2 * j + 1)) & 1u) << 31);
}

// Coordinates 32·sub .. 32·sub + 31 of the vector at src (fp16 or bf16),
// multiplied by D, as float.
__device__ __forceinline__ void load_signed(const uint16_t* src, int sub, bool bf16,
                                            const uint32_t (&smask)[16], float (&x)[32]) {
  const uint4* p = reinterpret_cast<const uint4*>(src + 32 * sub);
  uint4 raw[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) raw[k] = __ldcs(p + k);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t w4[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack16x2(w4[j] ^ smask[4 * k + j], bf16);
      x[8 * k + 2 * j] = f.x;
      x[8 * k + 2 * j + 1] = f.y;
    }
  }
}

// z = H·(D⊙x) in place for the vector held by a group of LPV lanes:
// coordinate 32·sub + i lives in register i of lane sub.
// Stride 1 in scalar form, strides 2..16 on register pairs, strides
// 32 .. 16·LPV across the lanes (x' = partner + sign·x, sign = -1 on the
// upper lane); every step rounds exactly like a scalar add or subtract.
template <int LPV>
__device__ __forceinline__ void rotate_vector(float (&x)[32], int sub, unsigned gmask) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float u = x[2 * j], v = x[2 * j + 1];
    x[2 * j] = u + v;
    x[2 * j + 1] = u - v;
  }
#pragma unroll
  for (int s = 2; s < 32; s <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      if ((i & s) == 0) {
        const float2 u = make_float2(x[i], x[i + 1]), v = make_float2(x[i + s], x[i + s + 1]);
        const float2 p = f2add(u, v), m = f2sub(u, v);
        x[i] = p.x; x[i + 1] = p.y;
        x[i + s] = m.x; x[i + s + 1] = m.y;
      }
    }
  }
#pragma unroll
  for (int o = 1; o < LPV; o <<= 1) {
    const float sg = (sub & o) ? -1.f : 1.f;
    const float2 sg2 = make_float2(sg, sg);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 v = make_float2(x[2 * j], x[2 * j + 1]);
      const float2 p = make_float2(__shfl_xor_sync(gmask, v.x, o), __shfl_xor_sync(gmask, v.y, o));
      const float2 r = f2fma(v, sg2, p);
      x[2 * j] = r.x;
      x[2 * j + 1] = r.y;
    }
  }
}

// Lloyd-Max indices of 32 rotated coordinates z (unnormalized Hadamard
// domain, z = H·(D⊙x)) of a vector whose norm is n, packed LSB-first into
// BITS words: idx = #{j : z/n >= t_j}. Shared by the FWHT encode (4 lanes
// per vector) and the tensor-core encode (one thread per vector, four calls),
// so the two take their decisions with the same arithmetic.
template <int BITS>
__device__ __forceinline__ void quantize_pack(const float (&x)[32], float n, const Codebook& cb,
                                              uint32_t (&words)[BITS]) {
  constexpr int kHalf = 1 << (BITS - 1);

  // idx = #{j : z/n >= t_j} over the symmetric table (t_{half-1} = 0), on
  // the FMA pipe. With a = |z| and the positive thresholds t_1 < .. < t_m
  // (m = half - 1, N(0,1) units), count = #{k : a >= n·t_k} is found by
  // binary search: each step's indicator [a >= n·t] is the saturated
  //   b = sat(a·(2^24/n) - t·2^24)
  // (1 at or above the threshold, 0 below it, fractional only within 2^-24
  // of it in zeta = z/n: inside the comparison window, where any index is
  // acceptable), and the next step's threshold is picked by the bits found
  // so far as a product-sum (exact for bits 0/1, off by at most an ulp of
  // t·2^24, i.e. ~2^-24 in zeta). With the odd number w = 2·count + 1:
  //   z >= 0: 2·idx = 2·(half + count)     = (2·half - 1) + w
  //   z <  0: 2·idx = 2·(half - 1 - count) = (2·half - 1) - w
  // so u = copysign(w, z) + (2·half - 1) = 2·idx, and 2^24 + u rounds to
  // an even number (fp32 spacing 2 there) whose mantissa bits are idx. A
  // zero vector keeps n = 0, z = 0 (made +0 by adding +0) and lands on
  // idx = half: its scale uses n = 1.
  constexpr float kTwo24 = 16777216.f;
  constexpr int NTH = kHalf - 1;                      // positive thresholds
  static_assert(NTH == 1 || NTH == 3 || NTH == 7, "2, 3 or 4 bits");
  const float big = __frcp_rn(n > 0.f ? n : 1.f) * kTwo24;
  float T[NTH];                                       // t_{k+1}·2^24
#pragma unroll
  for (int k = 0; k < NTH; ++k) T[k] = cb.threshold[kHalf + k] * kTwo24;
  constexpr float kOdd = (float)(2 * kHalf - 1);
  constexpr uint32_t kMagic = 0x4B800000u;            // bits of 2^24
  // the binary search's threshold differences, negated (-t·2^24 enters the
  // saturated FMA as its addend)
  const float2 one = make_float2(1.f, 1.f);
  auto ind = [&](float a0, float a1, float2 nt) {    // [a >= t] for both lanes
    return make_float2(fma_sat(a0, big, nt.x), fma_sat(a1, big, nt.y));
  };
  auto dup = [](float v) { return make_float2(v, v); };

  // words[w] accumulates bits(v) << off = (kMagic + idx) << off; the kMagic
  // parts are removed after the loop
#pragma unroll
  for (int w = 0; w < BITS; ++w) words[w] = 0;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float a0 = fabsf(x[i]), a1 = fabsf(x[i + 1]);
    float2 w2;
    if constexpr (NTH == 7) {
      const float2 b2 = ind(a0, a1, dup(-T[3]));                               // a >= t4
      const float2 b1 = ind(a0, a1, f2fma(b2, dup(T[1] - T[5]), dup(-T[1])));  // t6 or t2
      // t7, t5, t3 or t1: -t1 - b2·(t5 - t1) - b1·(t3 - t1) - b2·b1·(t7 - t5 - t3 + t1)
      float2 nt = f2fma(b2, dup(T[0] - T[4]), dup(-T[0]));
      nt = f2fma(b1, dup(T[0] - T[2]), nt);
      nt = f2fma(f2mul(b2, b1), dup((T[4] - T[6]) + (T[2] - T[0])), nt);
      const float2 b0 = ind(a0, a1, nt);
      w2 = f2fma(b2, dup(8.f), f2fma(b1, dup(4.f), f2fma(b0, dup(2.f), one)));
    } else if constexpr (NTH == 3) {
      const float2 b1 = ind(a0, a1, dup(-T[1]));                               // a >= t2
      const float2 b0 = ind(a0, a1, f2fma(b1, dup(T[0] - T[2]), dup(-T[0])));  // t3 or t1
      w2 = f2fma(b1, dup(4.f), f2fma(b0, dup(2.f), one));
    } else {
      w2 = f2fma(ind(a0, a1, dup(-T[0])), dup(2.f), one);
    }
    const float2 sg = f2add(make_float2(x[i], x[i + 1]), make_float2(0.f, 0.f));
    const float2 u = f2add(make_float2(copysignf(w2.x, sg.x), copysignf(w2.y, sg.y)),
                           make_float2(kOdd, kOdd));
    const float2 v = f2add(u, make_float2(kTwo24, kTwo24));
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const uint32_t b = __float_as_uint(e ? v.y : v.x);    // kMagic + idx
      const int p = (i + e) * BITS, w = p >> 5, off = p & 31;
      words[w] += b << off;
      if (off + BITS > 32) words[w + 1] += (b - kMagic) >> (32 - off);
    }
  }
#pragma unroll
  for (int w = 0; w < BITS; ++w) {
    uint32_t c = 0;                                   // the kMagic parts, mod 2^32
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int p = i * BITS;
      if ((p >> 5) == w) c += kMagic << (p & 31);
    }
    words[w] -= c;
  }
}

template <int BITS, int LPV>
__device__ __forceinline__ void encode_vector(
    float (&x)[32], const Codebook& cb, int sub, unsigned gmask,
    uint8_t* row_dst, uint16_t* norm_dst, int* dev_status) {
  // ||x||^2 over the group of LPV lanes (pairs of coordinates per fma)
  float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float2 v = make_float2(x[2 * j], x[2 * j + 1]);
    ss2 = f2fma(v, v, ss2);
  }
  float ss = ss2.x + ss2.y;
#pragma unroll
  for (int o = 1; o < LPV; o <<= 1) ss += __shfl_xor_sync(gmask, ss, o);
  const float n = sqrtf(ss);

  rotate_vector<LPV>(x, sub, gmask);
  uint32_t words[BITS];
  quantize_pack<BITS>(x, n, cb, words);

  if constexpr (BITS == 4) {
    *reinterpret_cast<uint4*>(row_dst + 16 * sub) =
        make_uint4(words[0], words[1], words[2], words[3]);
  } else if constexpr (BITS == 2) {
    *reinterpret_cast<uint2*>(row_dst + 8 * sub) = make_uint2(words[0], words[1]);
  } else {
    uint32_t* d32 = reinterpret_cast<uint32_t*>(row_dst + 12 * sub);
    d32[0] = words[0];
    d32[1] = words[1];
    d32[2] = words[2];
  }
  if (sub == 0) {
    *norm_dst = f32_to_f16_bits(fminf(n, 65504.f));
    if (n > 65504.f && dev_status) atomicOr(dev_status, TQ_DEV_NORM_SATURATED);
  }
}

}  // namespace tq
