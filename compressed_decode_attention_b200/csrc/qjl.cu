// Stage-2 residual sketch (QJL) of the keys and the unbiased score estimate.
//
// "We Built a Python Library That Cuts LLM Memory Usage by 80%", section
// "Why not both stages?": the method's second stage adds a one-bit
// correction of the stage-1 residual that makes inner products unbiased;
// that page leaves it out of softmax attention, so the library offers it as
// an inner-product (score) estimate. Definition (readings of that one
// sentence, frozen in tq.h): r~ = R·x - nK·c[idx]/sqrt(d) (the residual in
// rotated coordinates), bit_i = [(S·r~)_i >= 0] for an i.i.d. N(0,1) matrix
// S [d][d] that the caller supplies, gamma = fp16(||r~||), and
//   <q, x> ~ <q~, nK·c[idx]/sqrt(d)> + gamma·sqrt(pi/2)/d·<S·q~, 2·bit - 1>.
//
// tq_qjl_encode (qjl_encode_kernel): a CTA takes 64 tokens of one kv head.
//   1. d/32 lanes per key rebuild z = H·(D⊙x) in registers (the encoder's
//      rotation), read the key's stage-1 row and norm, and leave
//      r~·sqrt(d) = z - nK·c[idx] in shared memory with gamma.
//   2. S·r~ as a 64 x d x d fp32 product on the FMA pipe: S is staged 32
//      columns at a time (transposed) in shared memory; a thread owns 8
//      consecutive outputs of 64·8/d tokens, so its 8 sign bits form one
//      byte of each of its tokens' rows.
// tq_qjl_scores (qjl_scores_kernel): a CTA takes up to 1024 positions of one
//   (sequence, kv head). Its prologue rotates the GQA group's queries and
//   forms p = S·q~ (one warp per output row of S, coalesced); then every
//   thread scores its positions against the group from shared memory.
#include <math.h>

#include "encode_common.cuh"

namespace tq {
namespace {

constexpr int kQjlTokens = 64;        // tokens per encode CTA
constexpr int kQjlThreads = 256;
constexpr int kScorePositions = 1024; // positions per scores CTA

// ------------------------------------------------------------------ encode
template <int D>
struct QjlEncGeo {
  static constexpr int RS = D + 4;                 // residual row stride (floats)
  static constexpr int JC = 32;                    // S columns per staged chunk
  static constexpr int NO = D / 8;                 // threads across outputs
  static constexpr int NT = kQjlThreads / NO;      // threads across tokens
  static constexpr int TPT = kQjlTokens / NT;      // tokens per thread
  static constexpr size_t SMEM = (size_t)(kQjlTokens * RS + JC * D) * sizeof(float);
};

template <int D, int BITS>
__global__ void __launch_bounds__(kQjlThreads)
qjl_encode_kernel(const __grid_constant__ QjlEncodeArgs a,
                  const __grid_constant__ Codebook cb,
                  const __grid_constant__ SignMask sm) {
  using G = QjlEncGeo<D>;
  constexpr int LPV = D / 32;
  extern __shared__ __align__(16) float qsm[];
  float* rs = qsm;                                  // [64][RS] residual · sqrt(d)
  float* st = qsm + kQjlTokens * G::RS;             // [JC][D] chunk of S^T
  const int tid = threadIdx.x, lane = tid & 31;
  const int h = blockIdx.y;
  const int tok0 = blockIdx.x * kQjlTokens;
  const int ntok = min(kQjlTokens, a.n_tok - tok0);

  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  // ---- 1. residual of each key in rotated coordinates (times sqrt(d))
  {
    const int sub = lane & (LPV - 1);
    const unsigned gmask = ((1u << LPV) - 1u) << (lane & ~(LPV - 1));
    uint32_t smask[16];
    sign_masks(sm, sub, smask);
    constexpr int rowb = D * BITS / 8;
    for (int v = tid / LPV; v < kQjlTokens; v += kQjlThreads / LPV) {
      float* dst = rs + v * G::RS + 32 * sub;
      if (v >= ntok) {                              // rows past the end: zero
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[i] = 0.f;
        continue;
      }
      const int tok = tok0 + v;
      float x[32];
      load_signed(a.k + ((size_t)tok * a.n_kv_heads + h) * D, sub, a.is_bf16 != 0, smask, x);
      rotate_vector<LPV>(x, sub, gmask);
      const size_t row = (size_t)h * a.cap_tok + a.tok_offset + tok;
      // this lane's 32 fields: BITS words at byte 4·BITS·sub of the row
      const uint32_t* pr = reinterpret_cast<const uint32_t*>(a.packed_k + row * rowb) + BITS * sub;
      uint32_t w[BITS];
#pragma unroll
      for (int k = 0; k < BITS; ++k) w[k] = __ldg(pr + k);
      const float nk = __half2float(__ushort_as_half(a.norms_k[row]));
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float r = fmaf(-nk, cb.centroid[field<BITS>(w, i)], x[i]);
        dst[i] = r;
        ss = fmaf(r, r, ss);
      }
#pragma unroll
      for (int o = 1; o < LPV; o <<= 1) ss += __shfl_xor_sync(gmask, ss, o);
      if (sub == 0) {
        // ||r~|| = ||z - nK·c|| / sqrt(d)
        const float gmm = sqrtf(ss) * rsqrtf((float)D);
        a.gamma[row] = f32_to_f16_bits(fminf(gmm, 65504.f));
        if (gmm > 65504.f && a.dev_status) atomicOr(a.dev_status, TQ_DEV_NORM_SATURATED);
      }
    }
  }

  // ---- 2. u = S·r~ (the sign of r~·sqrt(d) is that of r~)
  const int oo = tid % G::NO, tt = tid / G::NO;
  float acc[G::TPT][8];
#pragma unroll
  for (int t = 0; t < G::TPT; ++t)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[t][k] = 0.f;
  for (int j0 = 0; j0 < D; j0 += G::JC) {
    __syncthreads();                                // residuals ready / chunk free
    // st[jj][o] = S[o][j0 + jj]: each thread copies float4 runs of rows of S
    for (int e = tid; e < D * G::JC / 4; e += kQjlThreads) {
      const int o = e / (G::JC / 4), jq = e % (G::JC / 4);
      const float4 s4 = __ldg(reinterpret_cast<const float4*>(a.S + (size_t)o * D + j0) + jq);
      st[(4 * jq + 0) * D + o] = s4.x;
      st[(4 * jq + 1) * D + o] = s4.y;
      st[(4 * jq + 2) * D + o] = s4.z;
      st[(4 * jq + 3) * D + o] = s4.w;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < G::JC; ++jj) {
      const float4 b0 = *reinterpret_cast<const float4*>(st + jj * D + 8 * oo);
      const float4 b1 = *reinterpret_cast<const float4*>(st + jj * D + 8 * oo + 4);
#pragma unroll
      for (int t = 0; t < G::TPT; ++t) {
        const float r = rs[(tt * G::TPT + t) * G::RS + j0 + jj];
        acc[t][0] = fmaf(r, b0.x, acc[t][0]);
        acc[t][1] = fmaf(r, b0.y, acc[t][1]);
        acc[t][2] = fmaf(r, b0.z, acc[t][2]);
        acc[t][3] = fmaf(r, b0.w, acc[t][3]);
        acc[t][4] = fmaf(r, b1.x, acc[t][4]);
        acc[t][5] = fmaf(r, b1.y, acc[t][5]);
        acc[t][6] = fmaf(r, b1.z, acc[t][6]);
        acc[t][7] = fmaf(r, b1.w, acc[t][7]);
      }
    }
  }
  // one byte (8 sign bits, LSB first) of each of this thread's tokens
#pragma unroll
  for (int t = 0; t < G::TPT; ++t) {
    const int v = tt * G::TPT + t;
    if (v >= ntok) continue;
    uint32_t byte = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) byte |= (acc[t][k] >= 0.f ? 1u : 0u) << k;
    const size_t row = (size_t)h * a.cap_tok + a.tok_offset + tok0 + v;
    a.sketch[row * (D / 8) + oo] = (uint8_t)byte;
  }
}

// ------------------------------------------------------------------ scores
template <int D, int BITS, int GMAX>
__global__ void __launch_bounds__(kQjlThreads)
qjl_scores_kernel(const __grid_constant__ QjlScoresArgs a,
                  const __grid_constant__ Codebook cb,
                  const __grid_constant__ SignMask sm) {
  constexpr int Q = D / 32;
  constexpr int NW = kQjlThreads / 32;
  constexpr int ROWB = D * BITS / 8;                // packed row bytes
  __shared__ __align__(16) float qt[GMAX][D];       // q~ = R·q
  __shared__ __align__(16) float qs[GMAX][D];       // q~ / d: stage-1 weights
  __shared__ __align__(16) float ps[GMAX][D];       // 2·(S·q~)·sqrt(pi/2)/d^{3/2}
  __shared__ float psum[GMAX];                      // sum_i ps/2 per head
  __shared__ float cs[16];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.y, b = blockIdx.z, G = a.gqa;
  const int t0 = blockIdx.x * kScorePositions;

  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  const int raw = a.ctx_lens[b];
  const int L = min(max(raw, 0), a.cap_tok);
  if (blockIdx.x == 0 && g == 0 && tid == 0 && a.dev_status && (raw > a.cap_tok || raw <= 0))
    atomicOr(a.dev_status, raw <= 0 ? TQ_DEV_CTX_EMPTY : TQ_DEV_CTX_CLAMPED);
  if (t0 >= L) return;

  if (tid < 16) cs[tid] = tid < (1 << BITS) ? cb.centroid[tid] : 0.f;
  // rotated queries, one warp per head: q~ = H·(D⊙q)/sqrt(d)
  for (int hh = warp; hh < GMAX; hh += NW) {
    float x[Q];
    if (hh < G) {
      const size_t qo = ((size_t)b * a.n_q_heads + (size_t)g * G + hh) * D + Q * lane;
#pragma unroll
      for (int k = 0; k < Q; ++k) {
        float v;
        if (a.q_dtype == TQ_F32) v = reinterpret_cast<const float*>(a.q)[qo + k];
        else if (a.q_dtype == TQ_BF16)
          v = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(a.q)[qo + k] << 16);
        else v = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(a.q)[qo + k]));
        const int c = Q * lane + k;
        x[k] = apply_sign(v, sm.w[c >> 5], c & 31);
      }
      fwht_registers<Q>(x);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) fwht_cross_lane<Q>(x, 0xFFFFFFFFu, o, lane & o);
    } else {
#pragma unroll
      for (int k = 0; k < Q; ++k) x[k] = 0.f;       // heads past the group: zeros
    }
    const float rsd = rsqrtf((float)D);
#pragma unroll
    for (int k = 0; k < Q; ++k) {
      qt[hh][Q * lane + k] = x[k] * rsd;
      qs[hh][Q * lane + k] = x[k] * (rsd * rsd * rsd);
    }
  }
  __syncthreads();
  // ps = 2·scale·S·q~: warp w takes rows w, w + NW, ...; lanes split a row
  // (coalesced reads of S); the butterfly leaves the sum in every lane
  const float scale = sqrtf(0.5f * 3.14159265358979f) / ((float)D * sqrtf((float)D));
  for (int o = warp; a.with_sketch && o < D; o += NW) {
    float part[GMAX];
#pragma unroll
    for (int hh = 0; hh < GMAX; ++hh) part[hh] = 0.f;
#pragma unroll
    for (int k = 0; k < Q; ++k) {
      const int j = lane + 32 * k;
      const float s = __ldg(a.S + (size_t)o * D + j);
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) part[hh] = fmaf(s, qt[hh][j], part[hh]);
    }
#pragma unroll
    for (int hh = 0; hh < GMAX; ++hh) {
      float v = part[hh];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
      if (lane == 0) ps[hh][o] = 2.f * scale * v;
    }
  }
  __syncthreads();
  if (a.with_sketch && warp < GMAX) {               // sum_i p_i (the -1 half of 2b - 1)
    float v = 0.f;
    for (int i = lane; i < D; i += 32) v += ps[warp][i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    if (lane == 0) psum[warp] = 0.5f * v;
  }
  __syncthreads();

  // ---- one position per thread:
  //   score = nK·sum_i qs_i·c[idx_i] + gamma·(sum_{bit_i = 1} ps_i - psum)
  const size_t hrow = ((size_t)b * a.n_kv_heads + g) * a.cap_tok;
  const int tend = min(L, t0 + kScorePositions);
  for (int t = t0 + tid; t < tend; t += kQjlThreads) {
    const size_t row = hrow + t;
    uint32_t w[ROWB / 4];
    {
      const uint2* pr = reinterpret_cast<const uint2*>(a.packed_k + row * ROWB);
#pragma unroll
      for (int k = 0; k < ROWB / 8; ++k) {
        const uint2 v = __ldg(pr + k);
        w[2 * k] = v.x;
        w[2 * k + 1] = v.y;
      }
    }
    const float nk = __half2float(__ushort_as_half(a.norms_k[row]));
    float s1[GMAX], s2[GMAX];
#pragma unroll
    for (int hh = 0; hh < GMAX; ++hh) s1[hh] = s2[hh] = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) {
      const float c = cs[field<BITS>(w, i)];
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) s1[hh] = fmaf(qs[hh][i], c, s1[hh]);
    }
    float score[GMAX];
#pragma unroll
    for (int hh = 0; hh < GMAX; ++hh) score[hh] = nk * s1[hh];
    if (a.with_sketch) {
      uint32_t sk[D / 32];
      const uint2* pk = reinterpret_cast<const uint2*>(a.sketch + row * (D / 8));
#pragma unroll
      for (int k = 0; k < D / 64; ++k) {
        const uint2 v = __ldg(pk + k);
        sk[2 * k] = v.x;
        sk[2 * k + 1] = v.y;
      }
      const float gm = __half2float(__ushort_as_half(a.gamma[row]));
#pragma unroll
      for (int i = 0; i < D; ++i) {
        const float bit = ((sk[i >> 5] >> (i & 31)) & 1u) ? 1.f : 0.f;
#pragma unroll
        for (int hh = 0; hh < GMAX; ++hh) s2[hh] = fmaf(bit, ps[hh][i], s2[hh]);
      }
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) score[hh] = fmaf(gm, s2[hh] - psum[hh], score[hh]);
    }
#pragma unroll
    for (int hh = 0; hh < GMAX; ++hh)
      if (hh < G) a.out[((size_t)b * a.n_q_heads + (size_t)g * G + hh) * a.cap_tok + t] = score[hh];
  }
}

template <int D, int BITS>
cudaError_t launch_encode_db(const QjlEncodeArgs& a, const Codebook& cb, const SignMask& sm,
                             cudaStream_t stream) {
  using G = QjlEncGeo<D>;
  static bool attr_set = false;
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(qjl_encode_kernel<D, BITS>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)G::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.n_tok + kQjlTokens - 1) / kQjlTokens, a.n_kv_heads, 1);
  cfg.blockDim = dim3(kQjlThreads);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qjl_encode_kernel<D, BITS>, a, cb, sm);
}

template <int D>
cudaError_t launch_encode_d(const QjlEncodeArgs& a, const Codebook& cb, const SignMask& sm,
                            cudaStream_t stream) {
  switch (a.bits_k) {
    case 2: return launch_encode_db<D, 2>(a, cb, sm, stream);
    case 3: return launch_encode_db<D, 3>(a, cb, sm, stream);
    default: return launch_encode_db<D, 4>(a, cb, sm, stream);
  }
}

template <int D, int BITS, int GMAX>
cudaError_t launch_scores_dbg(const QjlScoresArgs& a, const Codebook& cb, const SignMask& sm,
                              cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.cap_tok + kScorePositions - 1) / kScorePositions, a.n_kv_heads,
                     a.batch);
  cfg.blockDim = dim3(kQjlThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qjl_scores_kernel<D, BITS, GMAX>, a, cb, sm);
}

template <int D, int BITS>
cudaError_t launch_scores_db(const QjlScoresArgs& a, const Codebook& cb, const SignMask& sm,
                             cudaStream_t stream) {
  return a.gqa <= 4 ? launch_scores_dbg<D, BITS, 4>(a, cb, sm, stream)
                    : launch_scores_dbg<D, BITS, 8>(a, cb, sm, stream);
}

template <int D>
cudaError_t launch_scores_d(const QjlScoresArgs& a, const Codebook& cb, const SignMask& sm,
                            cudaStream_t stream) {
  switch (a.bits_k) {
    case 2: return launch_scores_db<D, 2>(a, cb, sm, stream);
    case 3: return launch_scores_db<D, 3>(a, cb, sm, stream);
    default: return launch_scores_db<D, 4>(a, cb, sm, stream);
  }
}

}  // namespace

cudaError_t launch_qjl_encode(const QjlEncodeArgs& a, const Codebook& cb, const SignMask& sm,
                              cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_encode_d<64>(a, cb, sm, stream);
    case 128: return launch_encode_d<128>(a, cb, sm, stream);
    case 256: return launch_encode_d<256>(a, cb, sm, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_qjl_scores(const QjlScoresArgs& a, const Codebook& cb, const SignMask& sm,
                              cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_scores_d<64>(a, cb, sm, stream);
    case 128: return launch_scores_d<128>(a, cb, sm, stream);
    case 256: return launch_scores_d<256>(a, cb, sm, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tq
