// tq_attend kernels: split-K flash decoding over the packed cache on the
// CUDA cores in fp32, then a combine that merges the splits and applies the
// inverse rotation once.
//
// [ADAPTQ §How it works, item 3]: the query is rotated once; scores come from
// the packed indices through the codebook. [TQAI §Test Suite]: the target is
// softmax(Q·K^T/sqrt d)·V. [TQPLUS §2 Sparse V]: V rows whose weight is
// negligible are skipped (block-local rule, see include/tq.h).
//
// Work item = (batch b, kv head g, split of split_tokens positions); one
// 128-thread CTA each. Per 64-position tile (one sparse-V block):
//   stage   packed K/V rows and fp16 norms -> shared memory
//   scores  thread = (position, half of the GQA group); 128-term dot of the
//           rotated query with the K codebook values, times the K norm
//   softmax per head: block max (gate reference), running max, rescale
//   V       thread = coordinate; acc[h] += w·nV·cV[idx] in the rotated domain
// Scores run in the log2 domain: the rotated query carries log2(e)/d^{3/2}
// (rotation normalization, codebook's 1/sqrt(d), softmax's 1/sqrt(d)).
#include <math.h>

#include "device_common.cuh"

namespace tq {
namespace {

constexpr int kAttThreads = 128;
constexpr int kTile = kGateBlock;
constexpr int kRowWords = 16 + 1;      // up to 64-byte rows, one pad word
constexpr float kLog2e = 1.44269504088896340736f;

struct AttendSmem {
  float q[kMaxGroup][kHeadDim];
  float s[kMaxGroup][kTile];
  float wv[kMaxGroup][kTile];
  uint32_t krow[kTile][kRowWords];
  uint32_t vrow[kTile][kRowWords];
  float nk[kTile], nv[kTile];
  float cbk[kMaxLevels], cbv[kMaxLevels];
  float m[kMaxGroup], l[kMaxGroup], alpha[kMaxGroup];
};

__device__ __forceinline__ float load_elem(const void* p, int dtype, size_t i) {
  if (dtype == TQ_F32) return reinterpret_cast<const float*>(p)[i];
  const uint16_t v = reinterpret_cast<const uint16_t*>(p)[i];
  if (dtype == TQ_BF16) return __uint_as_float((uint32_t)v << 16);
  return __half2float(__ushort_as_half(v));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

template <int BK, int BV>
__global__ void __launch_bounds__(kAttThreads)
attend_splitk_kernel(const __grid_constant__ AttendArgs a,
                     const __grid_constant__ Codebook cbk,
                     const __grid_constant__ Codebook cbv,
                     const __grid_constant__ SignMask sm) {
  __shared__ AttendSmem sh;
  constexpr int RKW = kHeadDim * BK / 32;   // words per packed row
  constexpr int RVW = kHeadDim * BV / 32;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = min(a.ctx_lens[b], a.cap_tok);
  const int t0 = split * a.split_tokens;
  if (L <= 0 || t0 >= L) return;
  const int t1 = min(L, t0 + a.split_tokens);
  const int G = a.gqa;
  const int hq0 = g * G;

  if (tid < kMaxLevels) {
    sh.cbk[tid] = cbk.centroid[tid];
    sh.cbv[tid] = cbv.centroid[tid];
  }
  // q~ = H·(D⊙q), one coordinate per thread, all heads of the group.
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    if (h < G) {
      const float v = load_elem(a.q, a.q_dtype, ((size_t)b * a.n_q_heads + hq0 + h) * kHeadDim + tid);
      sh.q[h][tid] = apply_sign(v, sm.w[tid >> 5], tid & 31);
    }
  }
  __syncthreads();
  for (int s = 1; s < kHeadDim; s <<= 1) {
    float nv[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      if (h < G) {
        const float mine = sh.q[h][tid], other = sh.q[h][tid ^ s];
        nv[h] = (tid & s) ? other - mine : mine + other;
      }
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
      if (h < G) sh.q[h][tid] = nv[h];
    __syncthreads();
  }
  const float qscale = kLog2e / (128.0f * 11.3137084989847603904f);  // log2 e / d^{3/2}
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h)
    if (h < G) sh.q[h][tid] *= qscale;
  if (tid < G) {
    sh.m[tid] = -INFINITY;
    sh.l[tid] = 0.f;
  }
  float acc[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) acc[h] = 0.f;
  unsigned long long skipped = 0;
  __syncthreads();

  const size_t seq_row = ((size_t)b * a.n_kv_heads + g) * a.cap_tok;
  const uint32_t* kw = reinterpret_cast<const uint32_t*>(a.packed_k) + seq_row * RKW;
  const uint32_t* vw = reinterpret_cast<const uint32_t*>(a.packed_v) + seq_row * RVW;
  const uint16_t* nkp = a.norms_k + seq_row;
  const uint16_t* nvp = a.norms_v + seq_row;

  for (int tb = t0; tb < t1; tb += kTile) {
    const int nt = min(kTile, t1 - tb);
    for (int w = tid; w < kTile * RKW; w += kAttThreads) {
      const int r = w / RKW, c = w % RKW;
      sh.krow[r][c] = r < nt ? kw[(size_t)(tb + r) * RKW + c] : 0u;
    }
    for (int w = tid; w < kTile * RVW; w += kAttThreads) {
      const int r = w / RVW, c = w % RVW;
      sh.vrow[r][c] = r < nt ? vw[(size_t)(tb + r) * RVW + c] : 0u;
    }
    if (tid < kTile) {
      sh.nk[tid] = tid < nt ? __half2float(__ushort_as_half(nkp[tb + tid])) : 0.f;
      sh.nv[tid] = tid < nt ? __half2float(__ushort_as_half(nvp[tb + tid])) : 0.f;
    }
    __syncthreads();

    {  // scores: position tt, heads hh0, hh0 + 2, ...
      const int tt = tid & (kTile - 1);
      const int hh0 = tid >> 6;
      float dot[kMaxGroup / 2];
#pragma unroll
      for (int j = 0; j < kMaxGroup / 2; ++j) dot[j] = 0.f;
      const uint32_t* row = sh.krow[tt];
#pragma unroll
      for (int i = 0; i < kHeadDim; ++i) {
        const float c = sh.cbk[field<BK>(row, i)];
#pragma unroll
        for (int j = 0; j < kMaxGroup / 2; ++j)
          if (hh0 + 2 * j < G) dot[j] = fmaf(sh.q[hh0 + 2 * j][i], c, dot[j]);
      }
#pragma unroll
      for (int j = 0; j < kMaxGroup / 2; ++j)
        if (hh0 + 2 * j < G)
          sh.s[hh0 + 2 * j][tt] = tt < nt ? sh.nk[tt] * dot[j] : -INFINITY;
    }
    __syncthreads();

    for (int h = warp; h < G; h += kAttThreads / 32) {
      const float s0 = sh.s[h][lane], s1 = sh.s[h][lane + 32];
      const float mblk = warp_max(fmaxf(s0, s1));
      const float mold = sh.m[h];
      const float mnew = fmaxf(mold, mblk);
      const float w0 = exp2f(s0 - mnew), w1 = exp2f(s1 - mnew);
      const float sum = warp_sum(w0 + w1);
      float v0 = w0 * sh.nv[lane], v1 = w1 * sh.nv[lane + 32];
      if (a.tau > 0.f) {
        const bool g0 = lane < nt && exp2f(s0 - mblk) < a.tau;
        const bool g1 = lane + 32 < nt && exp2f(s1 - mblk) < a.tau;
        if (g0) v0 = 0.f;
        if (g1) v1 = 0.f;
        const unsigned n0 = __popc(__ballot_sync(0xFFFFFFFFu, g0));
        const unsigned n1 = __popc(__ballot_sync(0xFFFFFFFFu, g1));
        if (lane == 0) skipped += n0 + n1;
      }
      sh.wv[h][lane] = v0;
      sh.wv[h][lane + 32] = v1;
      if (lane == 0) {
        const float al = exp2f(mold - mnew);
        sh.alpha[h] = al;
        sh.l[h] = sh.l[h] * al + sum;
        sh.m[h] = mnew;
      }
    }
    __syncthreads();

#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
      if (h < G) acc[h] *= sh.alpha[h];
    for (int t = 0; t < nt; ++t) {
      const float c = sh.cbv[field<BV>(sh.vrow[t], tid)];
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h)
        if (h < G) acc[h] = fmaf(sh.wv[h][t], c, acc[h]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    if (h < G) {
      const size_t unit = ((size_t)b * a.n_q_heads + hq0 + h) * a.n_splits + split;
      a.part_acc[unit * kHeadDim + tid] = acc[h];
      if (tid == 0) {
        a.part_ml[unit * 2] = sh.m[h];
        a.part_ml[unit * 2 + 1] = sh.l[h];
      }
    }
  }
  if (a.skipped && lane == 0 && skipped) atomicAdd(a.skipped, skipped);
}

// Merge the splits of one (b, query head), then out = D⊙(H·(acc/l))/d.
__global__ void __launch_bounds__(kHeadDim)
attend_combine_kernel(const __grid_constant__ AttendArgs a,
                      const __grid_constant__ SignMask sm) {
  __shared__ float x[kHeadDim];
  const int hq = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int raw = a.ctx_lens[b];
  const int L = min(raw, a.cap_tok);
  if (tid == 0 && hq == 0 && a.dev_status) {
    if (raw > a.cap_tok) atomicOr(a.dev_status, TQ_DEV_CTX_CLAMPED);
    if (raw <= 0) atomicOr(a.dev_status, TQ_DEV_CTX_EMPTY);
  }
  float r = 0.f;
  if (L > 0) {
    const int ns = (L + a.split_tokens - 1) / a.split_tokens;
    const size_t u0 = ((size_t)b * a.n_q_heads + hq) * a.n_splits;
    float mx = -INFINITY;
    for (int s = 0; s < ns; ++s) mx = fmaxf(mx, a.part_ml[(u0 + s) * 2]);
    float den = 0.f, num = 0.f;
    for (int s = 0; s < ns; ++s) {
      const float e = exp2f(a.part_ml[(u0 + s) * 2] - mx);
      den = fmaf(a.part_ml[(u0 + s) * 2 + 1], e, den);
      num = fmaf(a.part_acc[(u0 + s) * kHeadDim + tid], e, num);
    }
    r = num / den;
  }
  x[tid] = r;
  __syncthreads();
  for (int s = 1; s < kHeadDim; s <<= 1) {
    const float mine = x[tid], other = x[tid ^ s];
    __syncthreads();
    x[tid] = (tid & s) ? other - mine : mine + other;
    __syncthreads();
  }
  const float o = apply_sign(x[tid], sm.w[tid >> 5], tid & 31) * (1.0f / kHeadDim);
  const size_t oi = ((size_t)b * a.n_q_heads + hq) * kHeadDim + tid;
  if (a.out_dtype == TQ_F32) reinterpret_cast<float*>(a.out)[oi] = o;
  else if (a.out_dtype == TQ_BF16) reinterpret_cast<uint16_t*>(a.out)[oi] = f32_to_bf16_bits(o);
  else reinterpret_cast<uint16_t*>(a.out)[oi] = f32_to_f16_bits(o);
}

template <int BK, int BV>
cudaError_t launch_pair(const AttendArgs& a, const Codebook& cbk,
                        const Codebook& cbv, const SignMask& sm,
                        cudaStream_t stream) {
  dim3 grid(a.n_splits, a.n_kv_heads, a.batch);
  attend_splitk_kernel<BK, BV><<<grid, kAttThreads, 0, stream>>>(a, cbk, cbv, sm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend(const AttendArgs& a, const Codebook& cbk,
                          const Codebook& cbv, const SignMask& sm,
                          cudaStream_t stream) {
  cudaError_t e;
  switch (a.bits_k * 8 + a.bits_v) {
    case 4 * 8 + 2: e = launch_pair<4, 2>(a, cbk, cbv, sm, stream); break;
    case 3 * 8 + 2: e = launch_pair<3, 2>(a, cbk, cbv, sm, stream); break;
    case 4 * 8 + 3: e = launch_pair<4, 3>(a, cbk, cbv, sm, stream); break;
    case 4 * 8 + 4: e = launch_pair<4, 4>(a, cbk, cbv, sm, stream); break;
    case 3 * 8 + 3: e = launch_pair<3, 3>(a, cbk, cbv, sm, stream); break;
    case 2 * 8 + 2: e = launch_pair<2, 2>(a, cbk, cbv, sm, stream); break;
    case 3 * 8 + 4: e = launch_pair<3, 4>(a, cbk, cbv, sm, stream); break;
    case 2 * 8 + 3: e = launch_pair<2, 3>(a, cbk, cbv, sm, stream); break;
    case 2 * 8 + 4: e = launch_pair<2, 4>(a, cbk, cbv, sm, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  dim3 cgrid(a.n_q_heads, a.batch);
  attend_combine_kernel<<<cgrid, kHeadDim, 0, stream>>>(a, sm);
  return cudaGetLastError();
}

}  // namespace tq
