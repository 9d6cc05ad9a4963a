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
//      rotation), read the key's stage-1 row and norm, and leave the
//      residual z - nK·c[idx], scaled to unit length, in shared memory as
//      fp16 high/low parts, with gamma.
//   2. S·r~ on tensor cores (mma.sync m16n8k16, fp32 accumulate) as
//      Ahi·Bhi + Ahi·Blo + Alo·Bhi (~22 significant bits); S staged 64
//      columns at a time as fp16 high/low [output][column] tiles. Warp
//      ballots of the accumulator signs give the row bytes.
// tq_qjl_scores (qjl_scores_kernel): a CTA takes up to 512 positions of one
//   (sequence, kv head). Its prologue rotates the GQA group's queries and
//   forms p = S·q~ (a thread per row of S and group of heads); then every
//   thread scores two positions against the group, reading the group's
//   weights as 16-byte shared-memory broadcasts. Measured: 256 or 128
//   positions per CTA repeat the prologue too often, 1024 leave too few
//   CTAs for the latency-bound loop.
#include <atomic>
#include <math.h>

#include "encode_common.cuh"

namespace tq {
namespace {

constexpr int kQjlTokens = 64;        // tokens per encode CTA
constexpr int kQjlThreads = 256;
constexpr int kScoreThreads = 256;     // threads per scores CTA
constexpr int kScorePositions = 512;   // positions per scores CTA
static_assert(kScorePositions % kScoreThreads == 0, "whole positions per thread");

// ------------------------------------------------------------------ encode
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// fp16 high part and the fp16 rounding of the remainder: hi + lo carries
// about 22 significant bits of x
__device__ __forceinline__ void split_f16(float x, __half& hi, __half& lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}
// bit 2i of the result = bit i of the 4-bit x
__device__ __forceinline__ uint32_t spread4(uint32_t x) {
  return (x & 1u) | ((x & 2u) << 1) | ((x & 4u) << 2) | ((x & 8u) << 3);
}

template <int D>
struct QjlEncGeo {
  // S is staged 64 columns at a time for every 64-token unit (72 KB of
  // shared memory at d = 128: three CTAs per SM). Keeping all of S resident
  // in a persistent CTA (104 KB, two CTAs per SM) measured slower: the
  // kernel is latency-bound and gains more from the extra warps.
  static constexpr int AS = D + 8;                 // A row stride (halves): 16 B pad
  static constexpr int KC = D < 64 ? D : 64;       // S columns per staged chunk
  static constexpr int BS = KC + 8;                // S chunk row stride (halves)
  static constexpr int NT8 = D / 16;               // n-tiles of 8 outputs per warp
  static constexpr size_t A_BYTES = (size_t)kQjlTokens * AS * 2;
  static constexpr size_t B_BYTES = (size_t)D * BS * 2;
  static constexpr size_t SMEM = 2 * A_BYTES + 2 * B_BYTES;
  static_assert(D % KC == 0, "chunking");
};

// S[:, kc .. kc + KC) as fp16 high/low parts into [output][column] tiles.
template <int D, int KC, int BS>
__device__ __forceinline__ void stage_projection(const float* S, int kc, __half* bhi,
                                                 __half* blo, int tid) {
  for (int e = tid; e < D * KC / 4; e += kQjlThreads) {
    const int o = e / (KC / 4), q4 = e % (KC / 4);
    const float4 s4 = __ldg(reinterpret_cast<const float4*>(S + (size_t)o * D + kc) + q4);
    __half hx, lx, hy, ly, hz, lz, hw, lw;
    split_f16(s4.x, hx, lx);
    split_f16(s4.y, hy, ly);
    split_f16(s4.z, hz, lz);
    split_f16(s4.w, hw, lw);
    __half2* ph = reinterpret_cast<__half2*>(bhi + o * BS + 4 * q4);
    __half2* pl = reinterpret_cast<__half2*>(blo + o * BS + 4 * q4);
    ph[0] = __halves2half2(hx, hy);
    ph[1] = __halves2half2(hz, hw);
    pl[0] = __halves2half2(lx, ly);
    pl[1] = __halves2half2(lz, lw);
  }
}

template <int D, int BITS>
__global__ void __launch_bounds__(kQjlThreads)
qjl_encode_kernel(const __grid_constant__ QjlEncodeArgs a,
                  const __grid_constant__ Codebook cb,
                  const __grid_constant__ SignMask sm) {
  using G = QjlEncGeo<D>;
  constexpr int LPV = D / 32;
  constexpr int KC = G::KC;
  extern __shared__ __align__(128) uint8_t qsm[];
  __half* ahi = reinterpret_cast<__half*>(qsm);                       // [64][AS]
  __half* alo = reinterpret_cast<__half*>(qsm + G::A_BYTES);
  __half* bhi = reinterpret_cast<__half*>(qsm + 2 * G::A_BYTES);      // [D][BS]
  __half* blo = reinterpret_cast<__half*>(qsm + 2 * G::A_BYTES + G::B_BYTES);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int h = blockIdx.y;
  const int tok0 = blockIdx.x * kQjlTokens;
  const int ntok = min(kQjlTokens, a.n_tok - tok0);

  // ---- 1. residual of each key in rotated coordinates, scaled to unit
  // length (the signs of S·r~ do not change), as fp16 high/low parts
  {
    const int sub = lane & (LPV - 1);
    const unsigned gmask = ((1u << LPV) - 1u) << (lane & ~(LPV - 1));
    uint32_t smask[16];
    sign_masks(sm, sub, smask);
    constexpr int rowb = D * BITS / 8;
    for (int v = tid / LPV; v < kQjlTokens; v += kQjlThreads / LPV) {
      __half* dh = ahi + v * G::AS + 32 * sub;
      __half* dl = alo + v * G::AS + 32 * sub;
      if (v >= ntok) {                              // rows past the end: zero
#pragma unroll
        for (int i = 0; i < 32; ++i) dh[i] = dl[i] = __float2half_rn(0.f);
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
        x[i] = fmaf(-nk, cb.centroid[field<BITS>(w, i)], x[i]);   // r~·sqrt(d)
        ss = fmaf(x[i], x[i], ss);
      }
#pragma unroll
      for (int o = 1; o < LPV; o <<= 1) ss += __shfl_xor_sync(gmask, ss, o);
      const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        __half h0, l0, h1, l1;
        split_f16(x[i] * inv, h0, l0);
        split_f16(x[i + 1] * inv, h1, l1);
        *reinterpret_cast<__half2*>(dh + i) = __halves2half2(h0, h1);
        *reinterpret_cast<__half2*>(dl + i) = __halves2half2(l0, l1);
      }
      if (sub == 0) {
        // ||r~|| = ||z - nK·c|| / sqrt(d)
        const float gmm = sqrtf(ss) * rsqrtf((float)D);
        a.gamma[row] = f32_to_f16_bits(fminf(gmm, 65504.f));
        if (gmm > 65504.f && a.dev_status) atomicOr(a.dev_status, TQ_DEV_NORM_SATURATED);
      }
    }
  }

  // ---- 2. u = S·r~ on tensor cores: warp (mt, nh) takes tokens 16·mt ..
  // and outputs nh·d/2 .. ; S is staged KC columns at a time as fp16
  // high/low [output][column]; u = Ahi·Bhi + Ahi·Blo + Alo·Bhi in fp32
  const int mt = warp & 3, nh = warp >> 2;
  float acc[G::NT8][4];
#pragma unroll
  for (int n = 0; n < G::NT8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
  // ldmatrix lane addresses: A rows 16·mt + (lane & 15), column +8 for
  // lanes 16..31; B rows (outputs) n0 + (lane & 7) + 8·(lane >> 4), column
  // +8 for lanes 8..15 and 24..31
  const uint32_t a_hi = smem_u32(ahi + (16 * mt + (lane & 15)) * G::AS + ((lane >> 4) << 3));
  const uint32_t a_lo = smem_u32(alo + (16 * mt + (lane & 15)) * G::AS + ((lane >> 4) << 3));
  const int brow = nh * (D / 2) + (lane & 7) + ((lane >> 4) << 3);
  const uint32_t b_hi = smem_u32(bhi + brow * G::BS + (((lane >> 3) & 1) << 3));
  const uint32_t b_lo = smem_u32(blo + brow * G::BS + (((lane >> 3) & 1) << 3));
  for (int kc = 0; kc < D; kc += KC) {
    __syncthreads();                                // A ready / previous chunk used
    stage_projection<D, KC, G::BS>(a.S, kc, bhi, blo, tid);
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < KC / 16; ++kk) {
      uint32_t ah[4], al[4];
      ldsm4(a_hi + 2 * (kc + 16 * kk), ah);
      ldsm4(a_lo + 2 * (kc + 16 * kk), al);
#pragma unroll
      for (int n2 = 0; n2 < G::NT8 / 2; ++n2) {
        uint32_t bh[4], bl[4];
        const uint32_t off = 2 * (16 * n2 * G::BS + 16 * kk);
        ldsm4(b_hi + off, bh);
        ldsm4(b_lo + off, bl);
        mma_f16(acc[2 * n2], ah, bh[0], bh[1]);
        mma_f16(acc[2 * n2], ah, bl[0], bl[1]);
        mma_f16(acc[2 * n2], al, bh[0], bh[1]);
        mma_f16(acc[2 * n2 + 1], ah, bh[2], bh[3]);
        mma_f16(acc[2 * n2 + 1], ah, bl[2], bl[3]);
        mma_f16(acc[2 * n2 + 1], al, bh[2], bh[3]);
      }
    }
  }

  // ---- 3. sign bits: accumulator (n-tile n, element e) of lane (g, t) is
  // token 16·mt + g + 8·(e >> 1), output 8·n + 2t + (e & 1) of the warp's
  // half. Ballots collect the 8 outputs of each n-tile; lane (g, t = 0)
  // writes token g's byte and lane (g, t = 1) token g + 8's.
  const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int n = 0; n < G::NT8; ++n) {
    const uint32_t m0 = __ballot_sync(0xFFFFFFFFu, acc[n][0] >= 0.f);
    const uint32_t m1 = __ballot_sync(0xFFFFFFFFu, acc[n][1] >= 0.f);
    const uint32_t m2 = __ballot_sync(0xFFFFFFFFu, acc[n][2] >= 0.f);
    const uint32_t m3 = __ballot_sync(0xFFFFFFFFu, acc[n][3] >= 0.f);
    if (tq < 2) {
      const uint32_t e0 = tq ? m2 : m0, e1 = tq ? m3 : m1;
      const uint32_t byte = spread4((e0 >> (4 * gq)) & 15u) | (spread4((e1 >> (4 * gq)) & 15u) << 1);
      const int v = 16 * mt + gq + 8 * tq;
      if (v < ntok) {
        const size_t row = (size_t)h * a.cap_tok + a.tok_offset + tok0 + v;
        a.sketch[row * (D / 8) + nh * (D / 16) + n] = (uint8_t)byte;
      }
    }
  }
}

// ------------------------------------------------------------------ scores
template <int D, int BITS, int GMAX>
__global__ void __launch_bounds__(kScoreThreads)
qjl_scores_kernel(const __grid_constant__ QjlScoresArgs a,
                  const __grid_constant__ Codebook cb,
                  const __grid_constant__ SignMask sm) {
  constexpr int Q = D / 32;
  constexpr int NW = kScoreThreads / 32;
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
  // ps = 2·scale·S·q~: thread (o, j) takes row o of S against heads j·HPT ..
  // (j + 1)·HPT - 1. The row's 16-byte loads are independent of each other
  // (one round trip to L2, not one per row); q~ is read as broadcasts.
  const float scale = sqrtf(0.5f * 3.14159265358979f) / ((float)D * sqrtf((float)D));
  constexpr int TPR = kScoreThreads >= D ? kScoreThreads / D : 1;   // threads per row of S
  constexpr int HPT = (GMAX + TPR - 1) / TPR;                     // heads per thread
  for (int e = tid; a.with_sketch && e < D * TPR; e += kScoreThreads) {
    const int o = e / TPR, h0 = (e % TPR) * HPT;
    const float4* srow = reinterpret_cast<const float4*>(a.S + (size_t)o * D);
    float part[HPT];
#pragma unroll
    for (int k = 0; k < HPT; ++k) part[k] = 0.f;
#pragma unroll 8
    for (int j4 = 0; j4 < D / 4; ++j4) {
      const float4 s4 = __ldg(srow + j4);
#pragma unroll
      for (int k = 0; k < HPT; ++k) {
        if (h0 + k < GMAX) {
          const float4 q4 = reinterpret_cast<const float4*>(&qt[h0 + k][0])[j4];
          part[k] = fmaf(s4.x, q4.x, part[k]);
          part[k] = fmaf(s4.y, q4.y, part[k]);
          part[k] = fmaf(s4.z, q4.z, part[k]);
          part[k] = fmaf(s4.w, q4.w, part[k]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < HPT; ++k)
      if (h0 + k < GMAX) ps[h0 + k][o] = 2.f * scale * part[k];
  }
  __syncthreads();
  for (int hh = warp; a.with_sketch && hh < GMAX; hh += NW) {   // sum_i p_i (the -1 half of 2b - 1)
    float v = 0.f;
    for (int i = lane; i < D; i += 32) v += ps[hh][i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    if (lane == 0) psum[hh] = 0.5f * v;
  }
  __syncthreads();

  // ---- PP positions per thread (t, t + kScoreThreads, ...), so each
  // 16-byte broadcast read of qs / ps serves all of them:
  //   score = nK·sum_i qs_i·c[idx_i] + gamma·(sum_{bit_i = 1} ps_i - psum)
  // Every sum runs over i in ascending order, as in a one-position loop.
  const size_t hrow = ((size_t)b * a.n_kv_heads + g) * a.cap_tok;
  const int tend = min(L, t0 + kScorePositions);
  const float4* qs4 = reinterpret_cast<const float4*>(&qs[0][0]);
  const float4* ps4 = reinterpret_cast<const float4*>(&ps[0][0]);
  constexpr int PP = kScorePositions / kScoreThreads;
  for (int tb = t0 + tid; tb < tend; tb += PP * kScoreThreads) {
    bool ok[PP];
    size_t row[PP];
    uint32_t w[PP][ROWB / 4];
    float nk[PP];
#pragma unroll
    for (int u = 0; u < PP; ++u) {
      const int t = tb + u * kScoreThreads;
      ok[u] = t < tend;
      row[u] = hrow + (ok[u] ? t : tb);             // a valid row either way
      const uint2* pr = reinterpret_cast<const uint2*>(a.packed_k + row[u] * ROWB);
#pragma unroll
      for (int k = 0; k < ROWB / 8; ++k) {
        const uint2 v = __ldg(pr + k);
        w[u][2 * k] = v.x;
        w[u][2 * k + 1] = v.y;
      }
      nk[u] = __half2float(__ushort_as_half(a.norms_k[row[u]]));
    }
    float s1[PP][GMAX];
#pragma unroll
    for (int u = 0; u < PP; ++u)
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) s1[u][hh] = 0.f;
#pragma unroll
    for (int i4 = 0; i4 < D / 4; ++i4) {
      float c[PP][4];
#pragma unroll
      for (int u = 0; u < PP; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[u][e] = cs[field<BITS>(w[u], 4 * i4 + e)];
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) {
        const float4 q = qs4[hh * (D / 4) + i4];
#pragma unroll
        for (int u = 0; u < PP; ++u) {
          s1[u][hh] = fmaf(q.x, c[u][0], s1[u][hh]);
          s1[u][hh] = fmaf(q.y, c[u][1], s1[u][hh]);
          s1[u][hh] = fmaf(q.z, c[u][2], s1[u][hh]);
          s1[u][hh] = fmaf(q.w, c[u][3], s1[u][hh]);
        }
      }
    }
    float score[PP][GMAX];
#pragma unroll
    for (int u = 0; u < PP; ++u)
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) score[u][hh] = nk[u] * s1[u][hh];
    if (a.with_sketch) {
      uint32_t sk[PP][D / 32];
      float gm[PP];
#pragma unroll
      for (int u = 0; u < PP; ++u) {
        const uint2* pk = reinterpret_cast<const uint2*>(a.sketch + row[u] * (D / 8));
#pragma unroll
        for (int k = 0; k < D / 64; ++k) {
          const uint2 v = __ldg(pk + k);
          sk[u][2 * k] = v.x;
          sk[u][2 * k + 1] = v.y;
        }
        gm[u] = __half2float(__ushort_as_half(a.gamma[row[u]]));
      }
      float s2[PP][GMAX];
#pragma unroll
      for (int u = 0; u < PP; ++u)
#pragma unroll
        for (int hh = 0; hh < GMAX; ++hh) s2[u][hh] = 0.f;
#pragma unroll
      for (int i4 = 0; i4 < D / 4; ++i4) {
        float bit[PP][4];
#pragma unroll
        for (int u = 0; u < PP; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 4 * i4 + e;
            bit[u][e] = ((sk[u][i >> 5] >> (i & 31)) & 1u) ? 1.f : 0.f;
          }
#pragma unroll
        for (int hh = 0; hh < GMAX; ++hh) {
          const float4 pv = ps4[hh * (D / 4) + i4];
#pragma unroll
          for (int u = 0; u < PP; ++u) {
            s2[u][hh] = fmaf(bit[u][0], pv.x, s2[u][hh]);
            s2[u][hh] = fmaf(bit[u][1], pv.y, s2[u][hh]);
            s2[u][hh] = fmaf(bit[u][2], pv.z, s2[u][hh]);
            s2[u][hh] = fmaf(bit[u][3], pv.w, s2[u][hh]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < PP; ++u)
#pragma unroll
        for (int hh = 0; hh < GMAX; ++hh)
          score[u][hh] = fmaf(gm[u], s2[u][hh] - psum[hh], score[u][hh]);
    }
#pragma unroll
    for (int u = 0; u < PP; ++u) {
      if (!ok[u]) continue;
      const int t = tb + u * kScoreThreads;
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh)
        if (hh < G) a.out[((size_t)b * a.n_q_heads + (size_t)g * G + hh) * a.cap_tok + t] = score[u][hh];
    }
  }
}

template <int D, int BITS>
cudaError_t launch_encode_db(const QjlEncodeArgs& a, const Codebook& cb, const SignMask& sm,
                             cudaStream_t stream) {
  using G = QjlEncGeo<D>;
  // the shared-memory opt-in is per device
  // set once per device (idempotent; atomic so that concurrent first calls do not race)
  static std::atomic<bool> configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(qjl_encode_kernel<D, BITS>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)G::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
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
  cfg.blockDim = dim3(kScoreThreads);
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
