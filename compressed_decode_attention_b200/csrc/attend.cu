// tq_attend: decode attention over the packed cache in one persistent,
// load-balanced kernel on the B200 tensor cores.
//
// [ADAPTQ §How it works, item 3]: the query is rotated once; scores are
// formed from the packed indices through the codebook, without materializing
// the dequantized cache. [TQAI §Test Suite]: the target is
// softmax(Q·K^T/sqrt d)·V. [TQPLUS §2 Sparse V]: V rows with negligible
// weight are left out (block-local rule, include/tq.h).
//
// Work decomposition. The cache is a flat list of 64-position blocks in
// (batch, kv head, block) order; CTA c of Geff owns blocks
// [c·NB/Geff, (c+1)·NB/Geff). Geff = min(grid, #blocks), except that when all
// S (batch, kv head) segments have the same block count and S <= grid, Geff
// is the largest multiple of S within the grid (at most one CTA per block),
// so every CTA stays inside one segment. A CTA walks the (batch, kv head)
// segments of its range; its warps split each segment, merge in shared
// memory, and either write the output (segment = whole sequence) or leave a
// partial in a workspace slot; the last CTA to finish a sequence (atomic
// counter, no waiting) merges the partials and writes the output. No separate
// combine launch, no spin-waits.
//
// Per warp and 64-position block (GQA group of g <= 8 query heads), in four
// 16-position steps:
//   stage   cp.async of the packed K/V rows and fp16 norms (per-warp ring)
//   scores  mma.m16n8k16, fp16 in, fp32 accumulate. A = K codebook values of
//           16 positions (rows) x 16 coordinates, read as fp16 high/low pairs
//           from a shared table indexed by the packed byte (one copy per
//           half-warp lane); B = rotated query, fp16 high and low parts in
//           the 8 columns (g <= 4: 4 heads x {high, low}; g <= 8: two column
//           tiles). K high, K low and query low are summed, so scores keep
//           ~22 significant bits (fp16-only operands measured up to 1.2e-2
//           output error with x20 outlier channels).
//   softmax fp32, log2 domain; block maximum = sparse-V reference.
//   PV      mma.m16n8k16: A = V codebook values (fp16), coordinates x
//           positions; B = softmax weight x V norm (fp16), moved from the
//           score layout with movmatrix. V2: position pairs by byte permutes
//           of a 4-entry register table; V3/V4: pair table + movmatrix.
// Output, once per (batch, query head): D⊙(H·(acc/l))/d with shuffles.
#include <math.h>

#include "device_common.cuh"

namespace tq {
namespace {

constexpr int kWarps = 12;
constexpr int kThreads = 32 * kWarps;
constexpr int kBlk = kGateBlock;                // positions per block
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kKScale = 256.f;                // K codebook scale inside the MMA
constexpr int kSmemBudget = 227 * 1024;

constexpr int ceil_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

template <int BK, int BV>
struct Geo {
  static constexpr int RK = 16 * BK;                    // packed K row bytes
  static constexpr int RV = 16 * BV;
  static constexpr int RVS = BV == 2 ? RV + 16 : RV;    // V row stride in smem
  static constexpr int KB = kBlk * RK;
  static constexpr int VB = kBlk * RVS;
  static constexpr int NKOFF = KB + VB;
  static constexpr int STAGE = KB + VB + 2 * kBlk * 2;
  // K table: uint2 (high pair, low pair) per (pair code, lane & 15): 128 B per code.
  static constexpr int LUTK = (1 << (2 * BK)) * 128;
  // V table (3/4 bits): uint32 fp16 pair per (pair code, lane): 128 B per code.
  static constexpr int LUTV = BV == 2 ? 0 : (1 << (2 * BV)) * 128;
  // The V table sits at a power-of-two offset no smaller than either table,
  // so entry addresses are formed with OR.
  static constexpr int LUTV_OFF = BV == 2 ? LUTK : ceil_pow2(LUTK > LUTV ? LUTK : LUTV);
  static constexpr int QOFF = LUTV_OFF + LUTV;
  static constexpr int QS = kMaxGroup * kHeadDim * 2 * 2;  // q~ high and low, fp16
  static constexpr int MISC = 1024;                     // kMiscWords words
  static constexpr int FIXED = QOFF + QS + MISC;
  static constexpr int NFIT = (kSmemBudget - FIXED) / (kWarps * STAGE);
  static constexpr int NSTAGE = NFIT > 3 ? 3 : NFIT;
  static constexpr int MERGE = kWarps * (kMaxGroup * kHeadDim + 2 * kMaxGroup) * 4;
  static constexpr int RING = NSTAGE * kWarps * STAGE;
  static constexpr int SMEM = FIXED + (RING > MERGE ? RING : MERGE);
  static_assert(NSTAGE >= 1, "stage ring does not fit");
  static_assert(SMEM <= kSmemBudget, "shared memory budget");
};

// misc words
constexpr int kMiscSeg = 0;      // b, g, blk0, nseg, nb, L
constexpr int kMiscLast = 8;     // last-CTA flag
constexpr int kMiscNB = 9;       // flat block count (lo, hi), common length
constexpr int kMiscState = 12;   // scan state: sb, sP (lo, hi)
constexpr int kMiscQInv = 16;    // 8 floats: 1/(query scale · kKScale)
constexpr int kMiscM = 32;       // 8 floats: merged max
constexpr int kMiscL = 40;       // 8 floats: merged sum
constexpr int kMiscCb = 64;      // 32 words: staged codebooks
constexpr int kMiscWt = 128;     // kWarps x 8 floats: per-warp merge weights
constexpr int kMiscWords = 256;  // Geo::MISC / 4
static_assert(kMiscWt + kWarps * kMaxGroup <= kMiscWords, "misc words");

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ float fast_exp2(float x) {   // ex2.approx: -inf -> 0
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

template <typename T>
__device__ __forceinline__ T lds(const uint8_t* base, uint32_t off) {
  return *reinterpret_cast<const T*>(base + off);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float load_elem(const void* p, int dtype, size_t i) {
  if (dtype == TQ_F32) return reinterpret_cast<const float*>(p)[i];
  const uint16_t v = reinterpret_cast<const uint16_t*>(p)[i];
  if (dtype == TQ_BF16) return __uint_as_float((uint32_t)v << 16);
  return __half2float(__ushort_as_half(v));
}

__device__ __forceinline__ int seq_blocks(const AttendArgs& a, int b) {
  const int L = min(max(a.ctx_lens[b], 0), a.cap_tok);
  return (L + kBlk - 1) / kBlk;
}

// CTA owning flat block `blk` when NB blocks are split over G CTAs as
// [c·NB/G, (c+1)·NB/G): the largest c with floor(c·NB/G) <= blk.
__device__ __forceinline__ int cta_of(long long blk, long long nb, int g) {
  return (int)(((blk + 1) * g - 1) / nb);
}

// Walsh-Hadamard transform of 128 values spread as 4 per lane (coordinate
// 4·lane + k in x[k]): two in-register stages, five shuffle stages.
__device__ __forceinline__ void fwht128_warp(float (&x)[4], int lane) {
#pragma unroll
  for (int s = 1; s < 4; s <<= 1)
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (!(k & s)) {
        const float u = x[k], v = x[k + s];
        x[k] = u + v;
        x[k + s] = u - v;
      }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const bool upper = lane & o;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float p = __shfl_xor_sync(0xFFFFFFFFu, x[k], o);
      x[k] = upper ? p - x[k] : x[k] + p;
    }
  }
}

// Output coordinate held by accumulator register (m-tile r, m-slot m) of PV.
template <int BV>
__device__ __forceinline__ int pv_coord(int r, int m) {
  if (BV == 2) return 16 * (m & 7) + 2 * r + (m >> 3);
  return 32 * ((m & 7) >> 1) + 4 * r + (m & 1) + 2 * (m >> 3);
}

// (pair code p of a lane's chunk of packed words) << SHIFT, for a table
// whose entries are 2^SHIFT bytes apart. Codes are 2·BITS bits wide
// (coordinates 2p, 2p+1), little-endian in the chunk.
template <int BITS, int SHIFT>
__device__ __forceinline__ uint32_t pair_code_shifted(const uint32_t* w, int p) {
  constexpr int FB = 2 * BITS;
  constexpr uint32_t MASK = ((1u << FB) - 1u) << SHIFT;
  const int bit = p * FB;
  const int k = bit >> 5, off = bit & 31;
  if (off + FB > 32) return (__funnelshift_r(w[k], w[k + 1], off) << SHIFT) & MASK;
  if (off >= SHIFT) return (w[k] >> (off - SHIFT)) & MASK;
  return (w[k] << (SHIFT - off)) & MASK;
}

template <int BK, int BV, int NT>
__global__ void __launch_bounds__(kThreads, 1)
attend_kernel(const __grid_constant__ AttendArgs a,
              const __grid_constant__ Codebook cbk,
              const __grid_constant__ Codebook cbv,
              const __grid_constant__ SignMask sm) {
  using Gm = Geo<BK, BV>;
  constexpr int NR = NT == 1 ? 1 : 2;       // score rows (positions) per lane and step
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* lutK = smem;                                   // offset 0
  uint8_t* lutV = smem + Gm::LUTV_OFF;
  __half* qhi = reinterpret_cast<__half*>(smem + Gm::QOFF);
  __half* qlo = qhi + kMaxGroup * kHeadDim;
  float* fin = reinterpret_cast<float*>(qhi);             // reuses q~ after a segment
  int* misc = reinterpret_cast<int*>(smem + Gm::QOFF + Gm::QS);
  float* miscf = reinterpret_cast<float*>(misc);
  float* merge = reinterpret_cast<float*>(smem + Gm::FIXED);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int H = a.n_kv_heads, GQ = a.gqa, B = a.batch;
  const int Gc = gridDim.x, cta = blockIdx.x;   // Gc <= kMaxCtas (host check)
  const uint32_t lbK = (lane & 15) * 8;                   // K table lane offset
  const uint32_t lbV = Gm::LUTV_OFF | (lane * 4);         // V table lane base

  // Lengths of the first 32 sequences, loaded by warp 0 now so the latency
  // overlaps the table build; the block count and the first segment search
  // reuse them.
  const int len0 = (warp == 0 && lane < B) ? min(max(a.ctx_lens[lane], 0), a.cap_tok) : 0;

  // ---- codebook tables: fp16 high/low parts of the scaled K levels and the
  // fp16 V levels are staged in misc first (uniform lookups afterwards).
  uint32_t* cbs = reinterpret_cast<uint32_t*>(misc) + kMiscCb;
  if (tid < 16) {
    const float c = cbk.centroid[tid] * kKScale;
    const __half h = __float2half_rn(c), l = __float2half_rn(c - __half2float(h));
    cbs[tid] = (uint32_t)__half_as_ushort(h) | ((uint32_t)__half_as_ushort(l) << 16);
    cbs[16 + tid] = __half_as_ushort(__float2half_rn(cbv.centroid[tid]));
  }
  __syncthreads();
  for (int e = tid; e < (1 << (2 * BK)) * 16; e += kThreads) {
    const int code = e >> 4, copy = e & 15;
    const uint32_t c0 = cbs[code & ((1 << BK) - 1)], c1 = cbs[code >> BK];
    uint2 v;
    v.x = (c0 & 0xFFFFu) | (c1 << 16);              // high parts (even, odd coord)
    v.y = (c0 >> 16) | (c1 & 0xFFFF0000u);          // low parts
    *reinterpret_cast<uint2*>(lutK + code * 128 + copy * 8) = v;
  }
  if (BV != 2) {
    for (int e = tid; e < (1 << (2 * BV)) * 32; e += kThreads) {
      const int code = e >> 5, copy = e & 31;
      *reinterpret_cast<uint32_t*>(lutV + code * 128 + copy * 4) =
          cbs[16 + (code & ((1 << BV) - 1))] | (cbs[16 + (code >> BV)] << 16);
    }
  }
  // V2 byte tables: low bytes of the 4 fp16 levels, then their high bytes.
  uint32_t vt_lo = 0, vt_hi = 0;
  if (BV == 2) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t h = __half_as_ushort(__float2half_rn(cbv.centroid[j]));
      vt_lo |= (h & 0xFFu) << (8 * j);
      vt_hi |= (h >> 8) << (8 * j);
    }
  }

  // ---- status words and empty sequences (CTA 0)
  if (cta == 0) {
    for (int b = 0; b < B; ++b) {
      const int raw = a.ctx_lens[b];
      if (tid == 0 && a.dev_status) {
        if (raw > a.cap_tok) atomicOr(a.dev_status, TQ_DEV_CTX_CLAMPED);
        if (raw <= 0) atomicOr(a.dev_status, TQ_DEV_CTX_EMPTY);
      }
      if (raw <= 0) {
        const size_t n = (size_t)a.n_q_heads * kHeadDim, base = (size_t)b * n;
        for (size_t i = tid; i < n; i += kThreads) {
          if (a.out_dtype == TQ_F32) reinterpret_cast<float*>(a.out)[base + i] = 0.f;
          else reinterpret_cast<uint16_t*>(a.out)[base + i] = 0;
        }
      }
    }
  }

  // ---- flat block count, and whether all sequences have the same length
  if (warp == 0) {
    long long tot = 0;
    int nmin = 0x7FFFFFFF, nmax = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const bool in = b0 + lane < B;
      const int nb = b0 == 0 ? (len0 + kBlk - 1) / kBlk : (in ? seq_blocks(a, b0 + lane) : 0);
      int sum = nb, lo = in ? nb : 0x7FFFFFFF, hi = nb;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
      }
      tot += sum;
      nmin = min(nmin, lo);
      nmax = max(nmax, hi);
    }
    if (lane == 0) {
      const long long nbt = tot * H;
      misc[kMiscNB] = (int)(nbt & 0xFFFFFFFF);
      misc[kMiscNB + 1] = (int)(nbt >> 32);
      misc[kMiscNB + 2] = nmin == nmax ? nmax : -1;   // common length in blocks
      misc[kMiscState] = 0;
      misc[kMiscState + 1] = 0;
      misc[kMiscState + 2] = 0;
    }
  }
  __syncthreads();
  const long long NB = (long long)(unsigned)misc[kMiscNB] | ((long long)misc[kMiscNB + 1] << 32);
  // Balance over Geff CTAs, each owning at least one block (the partial count
  // of a sequence relies on it): min(grid, NB), or, when every (sequence, kv
  // head) segment has the same length and there are no more segments than
  // CTAs, a multiple of the segment count so that no CTA spans two segments.
  int Geff = (int)min((long long)Gc, NB);
  {
    const int common = misc[kMiscNB + 2];
    const long long S = (long long)B * H;
    if (common > 0 && S <= Gc) Geff = (int)(S * min((long long)(Gc / S), (long long)common));
  }
  const long long r0 = cta < Geff ? NB * cta / Geff : 0;
  const long long r1 = cta < Geff ? NB * (cta + 1) / Geff : 0;
  long long pos = r0;
  unsigned nskip = 0;
  const float log2tau = a.tau > 0.f ? log2f(a.tau) : -INFINITY;

  // Lane roles in the score / softmax layout:
  //   NT = 1: the lane holds position gq (tq < 2) or gq + 8 (tq >= 2) of each
  //           16-position step, for heads hs0 = 2·(tq & 1) and hs0 + 1;
  //   NT = 2: positions gq and gq + 8, heads hs0 = 2·tq and hs0 + 1.
  const int hs0 = NT == 1 ? 2 * (tq & 1) : 2 * tq;
  const bool hv0 = hs0 < GQ, hv1 = hs0 + 1 < GQ;
  auto pos_of = [&](int mt, int rr) {
    return 16 * mt + gq + (NT == 1 ? 8 * (tq >> 1) : 8 * rr);
  };

  while (pos < r1) {
    // ---- next segment (warp 0): first sequence whose flat range holds pos
    if (warp == 0) {
      int sb = misc[kMiscState];
      long long sP = (long long)(unsigned)misc[kMiscState + 1] | ((long long)misc[kMiscState + 2] << 32);
      while (true) {
        if (sb >= B) {                    // inconsistent lengths: stop this CTA
          if (lane == 0) misc[kMiscSeg + 3] = 0;
          break;
        }
        const int b = sb + lane;
        const int len = sb == 0 ? len0 : (b < B ? min(max(a.ctx_lens[b], 0), a.cap_tok) : 0);
        const int nb = (len + kBlk - 1) / kBlk;
        int incl = nb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += v;
        }
        const long long end = (long long)H * (sP + incl);
        const unsigned hit = __ballot_sync(0xFFFFFFFFu, end > pos && b < B);
        if (hit) {
          const int l = __ffs(hit) - 1;
          const int nbl = __shfl_sync(0xFFFFFFFFu, nb, l);
          const int lenl = __shfl_sync(0xFFFFFFFFu, len, l);
          const int excl = __shfl_sync(0xFFFFFFFFu, incl - nb, l);
          sb += l;
          sP += excl;
          if (lane == 0) {
            const long long rel = pos - (long long)H * sP;
            const int g = (int)(rel / nbl), blk0 = (int)(rel % nbl);
            misc[kMiscSeg + 0] = sb;
            misc[kMiscSeg + 1] = g;
            misc[kMiscSeg + 2] = blk0;
            misc[kMiscSeg + 3] = (int)min((long long)(nbl - blk0), r1 - pos);
            misc[kMiscSeg + 4] = nbl;
            misc[kMiscSeg + 5] = lenl;
            misc[kMiscState] = sb;
            misc[kMiscState + 1] = (int)(sP & 0xFFFFFFFF);
            misc[kMiscState + 2] = (int)(sP >> 32);
          }
          break;
        }
        sP += __shfl_sync(0xFFFFFFFFu, incl, 31);
        sb += 32;
      }
    }
    __syncthreads();
    const int b = misc[kMiscSeg + 0], g = misc[kMiscSeg + 1], blk0 = misc[kMiscSeg + 2];
    const int nseg = misc[kMiscSeg + 3], nbl = misc[kMiscSeg + 4], L = misc[kMiscSeg + 5];
    if (nseg <= 0) break;
    const long long sP_seg = (long long)(unsigned)misc[kMiscState + 1] | ((long long)misc[kMiscState + 2] << 32);
    const long long seg_first = (long long)H * sP_seg + (long long)g * nbl;

    // query values of the group (warp h < g loads head h), issued before the
    // block loads so that both latencies overlap
    float qraw[4] = {0.f, 0.f, 0.f, 0.f};
    if (warp < GQ) {
      const size_t qo = ((size_t)b * a.n_q_heads + (size_t)g * GQ + warp) * kHeadDim + 4 * lane;
#pragma unroll
      for (int k = 0; k < 4; ++k) qraw[k] = load_elem(a.q, a.q_dtype, qo + k);
    }

    // ---- this warp's blocks of the segment; their first loads go out
    // before the query rotation so that the two overlap
    const int wb0 = blk0 + (int)((long long)nseg * warp / kWarps);
    const int wb1 = blk0 + (int)((long long)nseg * (warp + 1) / kWarps);
    const int nw = wb1 - wb0;

    float acc[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

    const size_t seq_row = ((size_t)b * H + g) * a.cap_tok;
    const uint8_t* gk = a.packed_k + seq_row * Gm::RK;
    const uint8_t* gv = a.packed_v + seq_row * Gm::RV;
    const uint16_t* gnk = a.norms_k + seq_row;
    const uint16_t* gnv = a.norms_v + seq_row;
    const uint32_t wring = Gm::FIXED + warp * Gm::NSTAGE * Gm::STAGE;   // smem offset
    const uint32_t wring_s = smem_addr(smem) + wring;                    // shared address

    // cp.async of block `blk` into ring slot `slot`. K and V blocks are
    // contiguous in global memory; chunk c of K lands at byte 16c, chunk c of
    // V at row (c / BV) · RVS + (c % BV) · 16. Chunks past the sequence are
    // zero-filled without reading.
    auto issue = [&](int blk, int slot) {
      const int t0 = blk * kBlk;
      const int kvalid = min(kBlk, L - t0) * BK;
      const int vvalid = min(kBlk, L - t0) * BV;
      const uint32_t dst = wring_s + slot * Gm::STAGE;
      const uint8_t* ksrc = gk + (size_t)t0 * Gm::RK;
      const uint8_t* vsrc = gv + (size_t)t0 * Gm::RV;
#pragma unroll
      for (int i = 0; i < BK * 2; ++i) {
        const int ch = lane + 32 * i;
        const bool ok = ch < kvalid;
        cp_async16(dst + 16 * ch, ksrc + (ok ? 16 * ch : 0), ok ? 16 : 0);
      }
#pragma unroll
      for (int i = 0; i < BV * 2; ++i) {
        const int ch = lane + 32 * i;
        const bool ok = ch < vvalid;
        cp_async16(dst + Gm::KB + (ch / BV) * Gm::RVS + (ch % BV) * 16,
                   vsrc + (ok ? 16 * ch : 0), ok ? 16 : 0);
      }
      if (lane < 16) {
        const int c8 = lane & 7;
        const bool ok = t0 + 8 * c8 < L;
        const uint16_t* src = (lane < 8 ? gnk : gnv) + t0 + (ok ? 8 * c8 : 0);
        cp_async16(dst + Gm::NKOFF + (lane >> 3) * (2 * kBlk) + 16 * c8, src, ok ? 16 : 0);
      }
    };

#pragma unroll
    for (int p = 0; p < Gm::NSTAGE - 1; ++p) {
      if (p < nw) issue(wb0 + p, p);
      cp_async_commit();
    }
    // ---- rotated query of the group: warp h handles query head h
    if (warp < GQ) {
      float x[4];
      const uint32_t m = sm.w[lane >> 3];
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = apply_sign(qraw[k], m, (4 * lane + k) & 31);
      fwht128_warp(x, lane);
      // log2(e)/d^{3/2} folds the rotation normalization, the codebook's
      // 1/sqrt(d) and the softmax 1/sqrt(d); a power-of-two scale keeps the
      // fp16 high part near 2^14 so that the low part stays normal.
      float amax = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        x[k] *= kLog2e / (128.0f * 11.3137084989847603904f);
        amax = fmaxf(amax, fabsf(x[k]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      const int e = amax > 0.f ? ilogbf(amax) : 0;
      const float qs = ldexpf(1.f, min(14 - e, 120));
      uint32_t hi2[2], lo2[2];
#pragma unroll
      for (int k = 0; k < 4; k += 2) {
        const float v0 = x[k] * qs, v1 = x[k + 1] * qs;
        const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
        hi2[k / 2] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
        lo2[k / 2] = pack_half2(v0 - __half2float(h0), v1 - __half2float(h1));
      }
      *reinterpret_cast<uint2*>(qhi + warp * kHeadDim + 4 * lane) = make_uint2(hi2[0], hi2[1]);
      *reinterpret_cast<uint2*>(qlo + warp * kHeadDim + 4 * lane) = make_uint2(lo2[0], lo2[1]);
      if (lane == 0) miscf[kMiscQInv + warp] = 1.f / (qs * kKScale);
    }
    __syncthreads();

    // ---- query fragments (B operand of the score MMA), column n = gq.
    //   NT = 1: columns 0-3 hold the high part of heads 0-3, 4-7 their low part.
    //   NT = 2: tile 0 column n = high part of head n, tile 1 = low part.
    // The K-low product reuses tile 0 (for NT = 1 it also picks up the
    // negligible query-low x K-low term).
    uint32_t qb[NT][8][2];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int head = NT == 1 ? (gq & 3) : gq;
      const __half* src = (NT == 1 ? (gq < 4) : (t == 0)) ? qhi : qlo;
      const bool ok = head < GQ;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int c0 = 32 * tq + 4 * s;
        qb[t][s][0] = ok ? *reinterpret_cast<const uint32_t*>(src + head * kHeadDim + c0) : 0u;
        qb[t][s][1] = ok ? *reinterpret_cast<const uint32_t*>(src + head * kHeadDim + c0 + 2) : 0u;
      }
    }
    const float sinv0 = hv0 ? miscf[kMiscQInv + hs0] : 0.f;
    const float sinv1 = hv1 ? miscf[kMiscQInv + hs0 + 1] : 0.f;

    for (int i = 0; i < nw; ++i) {
      {
        const int nxt = i + Gm::NSTAGE - 1;
        if (nxt < nw) issue(wb0 + nxt, nxt % Gm::NSTAGE);
        cp_async_commit();
      }
      cp_async_wait<Gm::NSTAGE - 1>();
      __syncwarp();
      const uint32_t st = wring + (i % Gm::NSTAGE) * Gm::STAGE;         // smem offset
      const int t0 = (wb0 + i) * kBlk;
      const bool partial = t0 + kBlk > L;

      // -- scores: 4 steps of 16 positions
      float sc[4][NR][2];               // [step][row][head hs0 + e]
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t kw0[BK + 1], kw1[BK + 1];   // rows gq and gq + 8, chunk tq
        const uint32_t r0 = st + (16 * mt + gq) * Gm::RK + 4 * BK * tq;
        const uint32_t r1 = r0 + 8 * Gm::RK;
        if (BK == 4) {                       // one 16-byte load per row chunk
          const uint4 u0 = lds<uint4>(smem, r0), u1 = lds<uint4>(smem, r1);
          kw0[0] = u0.x; kw0[1] = u0.y; kw0[2 % (BK + 1)] = u0.z; kw0[3 % (BK + 1)] = u0.w;
          kw1[0] = u1.x; kw1[1] = u1.y; kw1[2 % (BK + 1)] = u1.z; kw1[3 % (BK + 1)] = u1.w;
        } else if (BK == 2) {
          const uint2 u0 = lds<uint2>(smem, r0), u1 = lds<uint2>(smem, r1);
          kw0[0] = u0.x; kw0[1] = u0.y;
          kw1[0] = u1.x; kw1[1] = u1.y;
        } else {
#pragma unroll
          for (int w = 0; w < BK; ++w) {
            kw0[w] = lds<uint32_t>(smem, r0 + 4 * w);
            kw1[w] = lds<uint32_t>(smem, r1 + 4 * w);
          }
        }
        kw0[BK] = kw1[BK] = 0;
        // two accumulator sets (even / odd k-steps) halve the MMA chains
        float dh[2][NT][4], dl[2][4];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int t = 0; t < NT; ++t) dh[c][t][0] = dh[c][t][1] = dh[c][t][2] = dh[c][t][3] = 0.f;
          dl[c][0] = dl[c][1] = dl[c][2] = dl[c][3] = 0.f;
        }
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2) {
          const uint2 e00 = lds<uint2>(smem, pair_code_shifted<BK, 7>(kw0, 2 * s2) | lbK);
          const uint2 e10 = lds<uint2>(smem, pair_code_shifted<BK, 7>(kw1, 2 * s2) | lbK);
          const uint2 e01 = lds<uint2>(smem, pair_code_shifted<BK, 7>(kw0, 2 * s2 + 1) | lbK);
          const uint2 e11 = lds<uint2>(smem, pair_code_shifted<BK, 7>(kw1, 2 * s2 + 1) | lbK);
#pragma unroll
          for (int t = 0; t < NT; ++t)
            mma16816(dh[s2 & 1][t], e00.x, e10.x, e01.x, e11.x, qb[t][s2][0], qb[t][s2][1]);
          mma16816(dl[s2 & 1], e00.y, e10.y, e01.y, e11.y, qb[0][s2][0], qb[0][s2][1]);
        }
        float dsum[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dsum[t][k] = (dh[0][t][k] + dh[1][t][k]) + (t == 0 ? dl[0][k] + dl[1][k] : 0.f);
        // d[0], d[1]: position gq, columns 2tq, 2tq+1; d[2], d[3]: position gq+8
        if (NT == 1) {
          // Columns 2tq, 2tq+1 are the high part of heads 2tq, 2tq+1 (tq < 2)
          // or the low part of heads 2(tq-2), +1 (tq >= 2); lane ^ 2 holds
          // the other part. Lanes tq < 2 keep position gq, tq >= 2 keep gq+8.
          const float d0 = dsum[0][0], d1 = dsum[0][1];
          const float d2 = dsum[0][2], d3 = dsum[0][3];
          const bool lowq = tq >= 2;
          const float s0 = __shfl_xor_sync(0xFFFFFFFFu, lowq ? d0 : d2, 2);
          const float s1 = __shfl_xor_sync(0xFFFFFFFFu, lowq ? d1 : d3, 2);
          sc[mt][0][0] = (lowq ? d2 : d0) + s0;
          sc[mt][0][1] = (lowq ? d3 : d1) + s1;
        } else {
          sc[mt][0][0] = dsum[0][0] + dsum[NT - 1][0];
          sc[mt][0][1] = dsum[0][1] + dsum[NT - 1][1];
          sc[mt][NR - 1][0] = dsum[0][2] + dsum[NT - 1][2];
          sc[mt][NR - 1][1] = dsum[0][3] + dsum[NT - 1][3];
        }
      }

      // -- scale by the K norm and query scale, mask, block maximum per head
      float mb0 = -INFINITY, mb1 = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int rr = 0; rr < NR; ++rr) {
          const int p = pos_of(mt, rr);
          const float nk = __half2float(__ushort_as_half(lds<uint16_t>(smem, st + Gm::NKOFF + 2 * p)));
          float v0 = sc[mt][rr][0] * (sinv0 * nk);
          float v1 = sc[mt][rr][1] * (sinv1 * nk);
          if (partial && t0 + p >= L) v0 = v1 = -INFINITY;
          sc[mt][rr][0] = v0;
          sc[mt][rr][1] = v1;
          mb0 = fmaxf(mb0, v0);
          mb1 = fmaxf(mb1, v1);
        }
      // lanes holding the same heads: NT = 1 -> lane bits 1-4; NT = 2 -> bits 2-4
#pragma unroll
      for (int o = (NT == 1 ? 2 : 4); o < 32; o <<= 1) {
        mb0 = fmaxf(mb0, __shfl_xor_sync(0xFFFFFFFFu, mb0, o));
        mb1 = fmaxf(mb1, __shfl_xor_sync(0xFFFFFFFFu, mb1, o));
      }
      const float mn0 = fmaxf(m_run[0], mb0), mn1 = fmaxf(m_run[1], mb1);
      const float al0 = fast_exp2(m_run[0] - mn0), al1 = fast_exp2(m_run[1] - mn1);
      m_run[0] = mn0;
      m_run[1] = mn1;
      l_run[0] *= al0;
      l_run[1] *= al1;

      // -- weights, gate, P' = w · nV packed as fp16 pairs (heads hs0, hs0+1)
      uint32_t pk[4][NR];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int rr = 0; rr < NR; ++rr) {
          const int p = pos_of(mt, rr);
          const float nv = __half2float(__ushort_as_half(lds<uint16_t>(smem, st + Gm::NKOFF + 2 * kBlk + 2 * p)));
          const float s0 = sc[mt][rr][0], s1 = sc[mt][rr][1];
          const float w0 = fast_exp2(s0 - mn0), w1 = fast_exp2(s1 - mn1);
          l_run[0] += w0;
          l_run[1] += w1;
          float p0 = w0 * nv, p1 = w1 * nv;
          const bool g0 = s0 - mb0 < log2tau, g1 = s1 - mb1 < log2tau;   // exp(s - M_blk) < tau
          if (g0) p0 = 0.f;
          if (g1) p1 = 0.f;
          nskip += (g0 && hv0 && s0 != -INFINITY) + (g1 && hv1 && s1 != -INFINITY);
          pk[mt][rr] = pack_half2(hv0 ? p0 : 0.f, hv1 ? p1 : 0.f);
        }
      // rescale the PV accumulators (PV layout: heads 2tq, 2tq+1)
      {
        float a0 = al0, a1 = al1;
        if (NT == 1 && tq >= 2) a0 = a1 = 1.f;      // heads 4-7: padding
        if (__any_sync(0xFFFFFFFFu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            acc[r][0] *= a0;
            acc[r][1] *= a1;
            acc[r][2] *= a0;
            acc[r][3] *= a1;
          }
        }
      }

      // -- P·V over the four 16-position steps
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t x0, x1;   // P' of positions 0-7 / 8-15 x heads 0-7, standard layout
        if (NT == 1) {
          const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, pk[mt][0], 2);
          x0 = tq < 2 ? pk[mt][0] : 0u;
          x1 = tq < 2 ? other : 0u;
        } else {
          x0 = pk[mt][0];
          x1 = pk[mt][NR - 1];
        }
        if (!__any_sync(0xFFFFFFFFu, (x0 | x1) != 0u)) continue;   // whole step gated
        const uint32_t b0 = transpose8x8(x0), b1 = transpose8x8(x1);
        if (BV == 2) {
          const uint32_t vrow = st + Gm::KB + (16 * mt + 2 * tq) * Gm::RVS + 4 * gq;
          const uint32_t wA = lds<uint32_t>(smem, vrow), wB = lds<uint32_t>(smem, vrow + Gm::RVS);
          const uint32_t wC = lds<uint32_t>(smem, vrow + 8 * Gm::RVS);
          const uint32_t wD = lds<uint32_t>(smem, vrow + 9 * Gm::RVS);
          const uint32_t xab[2] = {__byte_perm(wA, wB, 0x5140), __byte_perm(wA, wB, 0x7362)};
          const uint32_t xcd[2] = {__byte_perm(wC, wD, 0x5140), __byte_perm(wC, wD, 0x7362)};
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int odd = 0; odd < 2; ++odd) {
              const int f0 = 4 * odd, f1 = 4 * odd + 2;   // codes of coords 2r, 2r+1
              const uint32_t s0 = ((xab[half] >> f0) & 0x03030303u) * 0x11u + 0x40404040u;
              const uint32_t s1 = ((xab[half] >> f1) & 0x03030303u) * 0x11u + 0x40404040u;
              const uint32_t s2 = ((xcd[half] >> f0) & 0x03030303u) * 0x11u + 0x40404040u;
              const uint32_t s3 = ((xcd[half] >> f1) & 0x03030303u) * 0x11u + 0x40404040u;
#pragma unroll
              for (int hb = 0; hb < 2; ++hb) {
                const int r = 2 * (2 * half + hb) + odd;
                const int sh = 16 * hb;
                mma16816(acc[r], __byte_perm(vt_lo, vt_hi, s0 >> sh),
                         __byte_perm(vt_lo, vt_hi, s1 >> sh), __byte_perm(vt_lo, vt_hi, s2 >> sh),
                         __byte_perm(vt_lo, vt_hi, s3 >> sh), b0, b1);
              }
            }
          }
        } else {
          uint32_t v0[BV + 1], v1[BV + 1];
          const uint32_t r0p = st + Gm::KB + (16 * mt + gq) * Gm::RVS + 4 * BV * tq;
          const uint32_t r1p = r0p + 8 * Gm::RVS;
#pragma unroll
          for (int w = 0; w < BV; ++w) {
            v0[w] = lds<uint32_t>(smem, r0p + 4 * w);
            v1[w] = lds<uint32_t>(smem, r1p + 4 * w);
          }
          v0[BV] = v1[BV] = 0;
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const uint32_t y0 = lds<uint32_t>(smem, pair_code_shifted<BV, 7>(v0, 2 * r) | lbV);
            const uint32_t y1 = lds<uint32_t>(smem, pair_code_shifted<BV, 7>(v0, 2 * r + 1) | lbV);
            const uint32_t y2 = lds<uint32_t>(smem, pair_code_shifted<BV, 7>(v1, 2 * r) | lbV);
            const uint32_t y3 = lds<uint32_t>(smem, pair_code_shifted<BV, 7>(v1, 2 * r + 1) | lbV);
            mma16816(acc[r], transpose8x8(y0), transpose8x8(y1), transpose8x8(y2),
                     transpose8x8(y3), b0, b1);
          }
        }
      }
      __syncwarp();
    }
    cp_async_wait<0>();

    // ---- per-warp softmax sums over the lanes holding the same heads
#pragma unroll
    for (int o = (NT == 1 ? 2 : 4); o < 32; o <<= 1) {
      l_run[0] += __shfl_xor_sync(0xFFFFFFFFu, l_run[0], o);
      l_run[1] += __shfl_xor_sync(0xFFFFFFFFu, l_run[1], o);
    }

    // ---- merge the warps of this segment
    constexpr int WS = kMaxGroup * kHeadDim + 2 * kMaxGroup;
    __syncthreads();                                  // all warps done with the ring
    {
      float* wm = merge + warp * WS;
      if (gq == 0 && (NT == 2 || tq < 2)) {
        if (hv0) {
          wm[kMaxGroup * kHeadDim + hs0] = nw > 0 ? m_run[0] : -INFINITY;
          wm[kMaxGroup * kHeadDim + kMaxGroup + hs0] = nw > 0 ? l_run[0] : 0.f;
        }
        if (hv1) {
          wm[kMaxGroup * kHeadDim + hs0 + 1] = nw > 0 ? m_run[1] : -INFINITY;
          wm[kMaxGroup * kHeadDim + kMaxGroup + hs0 + 1] = nw > 0 ? l_run[1] : 0.f;
        }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int c0 = pv_coord<BV>(r, gq), c1 = pv_coord<BV>(r, gq + 8);
        const int h0 = 2 * tq, h1 = 2 * tq + 1;
        if (h0 < GQ) {
          wm[h0 * kHeadDim + c0] = acc[r][0];
          wm[h0 * kHeadDim + c1] = acc[r][2];
        }
        if (h1 < GQ) {
          wm[h1 * kHeadDim + c0] = acc[r][1];
          wm[h1 * kHeadDim + c1] = acc[r][3];
        }
      }
    }
    __syncthreads();
    // per-head maximum and sum over the warps, then per-(warp, head) weights
    float* wt = miscf + kMiscWt;                      // [kWarps][GQ] <= 96 floats
    if (tid < GQ) {
      float mx = -INFINITY;
      for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, merge[w * WS + kMaxGroup * kHeadDim + tid]);
      float ls = 0.f;
      for (int w = 0; w < kWarps; ++w) {
        const float mw = merge[w * WS + kMaxGroup * kHeadDim + tid];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - mx);
        wt[w * GQ + tid] = f;
        ls += merge[w * WS + kMaxGroup * kHeadDim + kMaxGroup + tid] * f;
      }
      miscf[kMiscM + tid] = mx;
      miscf[kMiscL + tid] = ls;
    }
    __syncthreads();
    for (int i = tid; i < GQ * kHeadDim; i += kThreads) {
      const int h = i / kHeadDim;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = wt[w * GQ + h];
        if (f != 0.f) s += merge[w * WS + i] * f;
      }
      fin[i] = s;
    }
    __syncthreads();

    bool finalize = nseg == nbl;                      // this CTA saw the whole sequence
    if (!finalize) {
      const int sigma = b * H + g;
      const long long last = seg_first + nbl - 1;
      const int c_first = cta_of(seg_first, NB, Geff), c_last = cta_of(last, NB, Geff);
      const int n_parts = c_last - c_first + 1;
      float* slot = a.slots + (size_t)(cta + sigma) * GQ * kSlotFloats;
      for (int i = tid; i < GQ * kHeadDim; i += kThreads) slot[i] = fin[i];
      if (tid < GQ) {
        slot[GQ * kHeadDim + 2 * tid] = miscf[kMiscM + tid];
        slot[GQ * kHeadDim + 2 * tid + 1] = miscf[kMiscL + tid];
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        const int prev = atomicAdd(a.counters + sigma, 1);
        misc[kMiscLast] = prev == n_parts - 1;
      }
      __syncthreads();
      finalize = misc[kMiscLast] != 0;
      if (finalize) {
        // Merge the n_parts partials of this sequence. Their (max, sum) pairs
        // are read in one parallel pass and turned into weights in shared
        // memory (the ring area is free here: n_parts <= 1024 CTAs x 8 heads
        // x 2 floats = 64 KB); the accumulators are then summed with up to 16
        // independent loads in flight per thread.
        __threadfence();
        const float* s0 = a.slots + (size_t)(c_first + sigma) * GQ * kSlotFloats;
        const size_t stride = (size_t)GQ * kSlotFloats;
        float* pm = merge;                       // [n_parts][GQ] max, then weight
        float* pl = merge + n_parts * GQ;        // [n_parts][GQ] sum
        for (int j = tid; j < n_parts * GQ; j += kThreads) {
          const int p = j / GQ, h = j - p * GQ;
          pm[j] = __ldcg(s0 + p * stride + GQ * kHeadDim + 2 * h);
          pl[j] = __ldcg(s0 + p * stride + GQ * kHeadDim + 2 * h + 1);
        }
        __syncthreads();
        if (tid < GQ) {
          float mx = -INFINITY;
          for (int p = 0; p < n_parts; ++p) mx = fmaxf(mx, pm[p * GQ + tid]);
          float ls = 0.f;
          for (int p = 0; p < n_parts; ++p) ls += pl[p * GQ + tid] * exp2f(pm[p * GQ + tid] - mx);
          miscf[kMiscM + tid] = mx;
          miscf[kMiscL + tid] = ls;
        }
        __syncthreads();
        for (int j = tid; j < n_parts * GQ; j += kThreads)
          pm[j] = exp2f(pm[j] - miscf[kMiscM + j % GQ]);
        __syncthreads();
        for (int i = tid; i < GQ * kHeadDim; i += kThreads) {
          const int h = i / kHeadDim;
          float sum = 0.f;
          int p = 0;
          for (; p + 16 <= n_parts; p += 16) {
            float v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = __ldcg(s0 + (p + k) * stride + i);
#pragma unroll
            for (int k = 0; k < 16; ++k) sum += v[k] * pm[(p + k) * GQ + h];
          }
          for (; p + 4 <= n_parts; p += 4) {
            float v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = __ldcg(s0 + (p + k) * stride + i);
#pragma unroll
            for (int k = 0; k < 4; ++k) sum += v[k] * pm[(p + k) * GQ + h];
          }
          for (; p < n_parts; ++p) sum += __ldcg(s0 + p * stride + i) * pm[p * GQ + h];
          fin[i] = sum;
        }
        if (tid == 0) atomicExch(a.counters + sigma, 0);
        __syncthreads();
      }
    }
    if (finalize && warp < GQ) {
      const float inv_l = 1.f / miscf[kMiscL + warp];
      float x[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = fin[warp * kHeadDim + 4 * lane + k] * inv_l;
      fwht128_warp(x, lane);
      const uint32_t m = sm.w[lane >> 3];
      const size_t ob = ((size_t)b * a.n_q_heads + (size_t)g * GQ + warp) * kHeadDim + 4 * lane;
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = apply_sign(x[k], m, (4 * lane + k) & 31) * (1.f / kHeadDim);
      if (a.out_dtype == TQ_F32) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + ob) = make_float4(x[0], x[1], x[2], x[3]);
      } else {
        uint16_t h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          h[k] = a.out_dtype == TQ_BF16 ? f32_to_bf16_bits(x[k]) : f32_to_f16_bits(x[k]);
        *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.out) + ob) =
            make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
      }
    }
    pos += nseg;
    __syncthreads();                                  // misc / fin / q~ reuse
  }

  if (a.skipped) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nskip += __shfl_xor_sync(0xFFFFFFFFu, nskip, o);
    if (lane == 0 && nskip) atomicAdd(a.skipped, (unsigned long long)nskip);
  }
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int BK, int BV, int NT>
cudaError_t launch_one(const AttendArgs& a, const Codebook& cbk, const Codebook& cbv,
                       const SignMask& sm, int n_ctas, cudaStream_t stream) {
  using Gm = Geo<BK, BV>;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(attend_kernel<BK, BV, NT>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  const int grid = n_ctas > 0 ? n_ctas : sm_count();
  attend_kernel<BK, BV, NT><<<grid, kThreads, Gm::SMEM, stream>>>(a, cbk, cbv, sm);
  return cudaGetLastError();
}

template <int BK, int BV>
cudaError_t launch_pair(const AttendArgs& a, const Codebook& cbk, const Codebook& cbv,
                        const SignMask& sm, int n_ctas, cudaStream_t stream) {
  return a.gqa <= 4 ? launch_one<BK, BV, 1>(a, cbk, cbv, sm, n_ctas, stream)
                    : launch_one<BK, BV, 2>(a, cbk, cbv, sm, n_ctas, stream);
}

}  // namespace

cudaError_t launch_attend(const AttendArgs& a, const Codebook& cbk,
                          const Codebook& cbv, const SignMask& sm, int n_ctas,
                          cudaStream_t stream) {
  if (n_ctas > kMaxCtas) return cudaErrorInvalidValue;
  switch (a.bits_k * 8 + a.bits_v) {
    case 4 * 8 + 2: return launch_pair<4, 2>(a, cbk, cbv, sm, n_ctas, stream);
    case 3 * 8 + 2: return launch_pair<3, 2>(a, cbk, cbv, sm, n_ctas, stream);
    case 4 * 8 + 3: return launch_pair<4, 3>(a, cbk, cbv, sm, n_ctas, stream);
    case 2 * 8 + 2: return launch_pair<2, 2>(a, cbk, cbv, sm, n_ctas, stream);
    case 3 * 8 + 3: return launch_pair<3, 3>(a, cbk, cbv, sm, n_ctas, stream);
    case 4 * 8 + 4: return launch_pair<4, 4>(a, cbk, cbv, sm, n_ctas, stream);
    case 2 * 8 + 3: return launch_pair<2, 3>(a, cbk, cbv, sm, n_ctas, stream);
    case 2 * 8 + 4: return launch_pair<2, 4>(a, cbk, cbv, sm, n_ctas, stream);
    case 3 * 8 + 4: return launch_pair<3, 4>(a, cbk, cbv, sm, n_ctas, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tq
