// Merge of context-parallel attention records and the inverse rotation.
//
// Each device of a context-parallel group attends over its own slice of the
// positions (tq_attend_partial) and leaves, per (sequence, query head), a
// log-sum-exp record: acc[d] in the unnormalized Hadamard domain, the base-2
// maximum score m2 and the sum l of 2^(score - m2). Records of disjoint
// slices merge exactly:
//   M = max_p m2_p,  f_p = 2^(m2_p - M),  l = sum_p f_p l_p,  acc likewise,
// and the output is rotated back once, out = D⊙(H·(acc / l)) / d — the last
// step of single-pass decode attention (AdapTQ, "How it works", item 3:
// the value sum stays in the rotated domain until the end).
//
// One warp per record; lane i holds coordinates d/32·i .. d/32·i + d/32 - 1.
// Part factors are computed 32 parts at a time, one part per lane, and
// broadcast; the value loads of different parts are independent.
#include <math.h>

#include "device_common.cuh"

namespace tq {
namespace {

constexpr int kCombineWarps = 8;

template <int D>
__global__ void __launch_bounds__(32 * kCombineWarps)
combine_kernel(CombineArgs a, SignMask sm) {
  constexpr int Q = D / 32;
  const int lane = threadIdx.x & 31;
  const int rec = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  if (rec >= a.n_rec) return;
  const size_t part_stride = (size_t)a.n_rec * (D + 2);
  const float* base = a.partials + (size_t)rec * (D + 2);

  // global maximum over the parts (empty parts hold -inf)
  float M = -INFINITY;
  for (int p = lane; p < a.n_parts; p += 32) M = fmaxf(M, __ldg(base + p * part_stride + D));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));

  float acc[Q];
#pragma unroll
  for (int k = 0; k < Q; ++k) acc[k] = 0.f;
  float L = 0.f;
  if (M != -INFINITY) {
    for (int p0 = 0; p0 < a.n_parts; p0 += 32) {
      const int p = p0 + lane;
      float f = 0.f, lp = 0.f;
      if (p < a.n_parts) {
        const float2 ml = __ldg(reinterpret_cast<const float2*>(base + p * part_stride + D));
        f = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
        lp = ml.y;
      }
      float fl = f * lp;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) fl += __shfl_xor_sync(0xFFFFFFFFu, fl, o);
      L += fl;
      const int np = min(32, a.n_parts - p0);
#pragma unroll 4
      for (int j = 0; j < np; ++j) {
        const float fj = __shfl_sync(0xFFFFFFFFu, f, j);
        const float* v = base + (size_t)(p0 + j) * part_stride + Q * lane;
#pragma unroll
        for (int k = 0; k < Q; k += 2) {
          const float2 x = __ldg(reinterpret_cast<const float2*>(v + k));
          acc[k] = fmaf(fj, x.x, acc[k]);
          acc[k + 1] = fmaf(fj, x.y, acc[k + 1]);
        }
      }
    }
  } else if (lane == 0 && a.dev_status) {
    atomicOr(a.dev_status, TQ_DEV_CTX_EMPTY);      // no slice held a position
  }

  // out = D ⊙ (H · (acc / l)) / d; 0 when every slice was empty
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int k = 0; k < Q; ++k) acc[k] *= inv;
  fwht_registers<Q>(acc);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) fwht_cross_lane<Q>(acc, 0xFFFFFFFFu, o, lane & o);
#pragma unroll
  for (int k = 0; k < Q; ++k) {
    const int c = Q * lane + k;
    acc[k] = apply_sign(acc[k], sm.w[c >> 5], c & 31) * (1.f / D);
  }
  const size_t ob = (size_t)rec * D + Q * lane;
  if (a.out_dtype == TQ_F32) {
    float2* o = reinterpret_cast<float2*>(reinterpret_cast<float*>(a.out) + ob);
#pragma unroll
    for (int k = 0; k < Q / 2; ++k) o[k] = make_float2(acc[2 * k], acc[2 * k + 1]);
  } else {
    uint32_t* o = reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(a.out) + ob);
    const bool bf = a.out_dtype == TQ_BF16;
#pragma unroll
    for (int k = 0; k < Q / 2; ++k) {
      const uint32_t h0 = bf ? f32_to_bf16_bits(acc[2 * k]) : f32_to_f16_bits(acc[2 * k]);
      const uint32_t h1 = bf ? f32_to_bf16_bits(acc[2 * k + 1]) : f32_to_f16_bits(acc[2 * k + 1]);
      o[k] = h0 | (h1 << 16);
    }
  }
}

template <int D>
cudaError_t launch_d(const CombineArgs& a, const SignMask& sm, cudaStream_t stream) {
  const unsigned blocks = (unsigned)((a.n_rec + kCombineWarps - 1) / kCombineWarps);
  combine_kernel<D><<<blocks, 32 * kCombineWarps, 0, stream>>>(a, sm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, const SignMask& sm, cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_d<64>(a, sm, stream);
    case 128: return launch_d<128>(a, sm, stream);
    case 256: return launch_d<256>(a, sm, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tq
