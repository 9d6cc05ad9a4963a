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
// (batch, kv head, block) order; CTA c of G (one per SM) owns blocks
// [c·NB/G, (c+1)·NB/G). A CTA walks the (batch, kv head) segments of its range;
// its 8 warps split each segment, merge in shared memory, and either write
// the output directly (segment = whole sequence) or leave a partial in a
// workspace slot; the last CTA to finish a sequence (atomic counter, no
// waiting) merges the partials and writes the output. No separate combine
// launch, no spin-waits.
//
// Per warp and 64-position block (GQA group of g <= 8 query heads):
//   stage   cp.async of the packed K/V rows and fp16 norms (per-warp ring)
//   scores  mma.m16n8k16 (fp16 in, fp32 accumulate). A = rotated query:
//           rows 0-7 its fp16 high part, rows 8-15 its fp16 low part (the
//           group fills at most 8 rows), B = K codebook values as fp16
//           high/low pairs from a shared-memory table indexed by the packed
//           byte (one copy per lane, conflict-free). score = row h + row h+8,
//           so the query and codebook keep ~22 significant bits.
//   softmax fp32, log2 domain; block maximum = sparse-V reference
//   PV      mma.m16n8k16: A = V codebook values (fp16) as the transposed
//           tile, B = softmax weights · V norm (fp16) taken straight from the
//           score accumulators. V2: token pairs by byte permutes of a 4-entry
//           register table; V3/V4: pair table + movmatrix transpose.
// Output, once per (batch, query head): D⊙(H·(acc/l))/d with shuffles.
#include <math.h>

#include "device_common.cuh"

namespace tq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kBlk = kGateBlock;                // positions per block
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kKScale = 256.f;                // K codebook scale inside the MMA
constexpr int kSmemBudget = 227 * 1024;

template <int BK, int BV>
struct Geo {
  static constexpr int RK = 16 * BK;                    // packed K row bytes
  static constexpr int RV = 16 * BV;
  static constexpr int RVS = BV == 2 ? RV + 16 : RV;    // V row stride in smem
  static constexpr int KB = kBlk * RK;
  static constexpr int VB = kBlk * RVS;
  static constexpr int NKOFF = KB + VB;
  static constexpr int STAGE = KB + VB + 2 * kBlk * 2;
  static constexpr int LUTK = (1 << (2 * BK)) * 32 * 8;  // uint2 per (pair, lane)
  static constexpr int LUTV = BV == 2 ? 0 : (1 << (2 * BV)) * 32 * 4;
  static constexpr int QS = kMaxGroup * kHeadDim * 2 * 2;  // q~ high and low, fp16
  static constexpr int MISC = 512;                      // 128 words
  static constexpr int FIXED = LUTK + LUTV + QS + MISC;
  static constexpr int NFIT = (kSmemBudget - FIXED) / (kWarps * STAGE);
  static constexpr int NSTAGE = NFIT > 3 ? 3 : NFIT;
  static constexpr int MERGE = kWarps * (kMaxGroup * kHeadDim + 2 * kMaxGroup) * 4;
  static constexpr int RING = NSTAGE * kWarps * STAGE;
  static constexpr int SMEM = FIXED + (RING > MERGE ? RING : MERGE);
  static_assert(NSTAGE >= 1, "stage ring does not fit");
  static_assert(SMEM <= kSmemBudget, "shared memory budget");
};

// misc words
constexpr int kMiscSeg = 0;      // b, g, blk0, nseg, nb, L, flat0 (7 ints)
constexpr int kMiscLast = 8;     // last-CTA flag
constexpr int kMiscNB = 9;       // flat block count (2 ints: lo, hi)
constexpr int kMiscState = 12;   // scan state: sb, sP (lo, hi)
constexpr int kMiscQInv = 16;    // 8 floats: 1/(query scale · kKScale)
constexpr int kMiscM = 32;       // 8 floats: merged max
constexpr int kMiscL = 40;       // 8 floats: merged sum

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
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

// Plain shared-memory loads at a byte offset from the dynamic smem base, so
// the compiler can schedule them (the cp.async waits carry memory clobbers).
__device__ __forceinline__ uint2 lds64(const uint8_t* base, uint32_t off) {
  return *reinterpret_cast<const uint2*>(base + off);
}
__device__ __forceinline__ uint32_t lds32(const uint8_t* base, uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(base + off);
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

// Shared-memory address of pair-table entry `field` in this lane's copy
// (lane_base = table address + lane · entry size).
template <int ENTRY_SHIFT>
__device__ __forceinline__ uint32_t lut_off(uint32_t field, uint32_t lane_base) {
  return (field << ENTRY_SHIFT) + lane_base;
}

// Field p (2·BITS bits: coordinates 2p, 2p+1) of a lane's chunk of packed words.
template <int BITS>
__device__ __forceinline__ uint32_t pair_field(const uint32_t* w, int p) {
  constexpr int FB = 2 * BITS;
  const int bit = p * FB;
  const int k = bit >> 5, off = bit & 31;
  uint32_t v;
  if (off + FB <= 32) v = w[k] >> off;
  else v = __funnelshift_r(w[k], w[k + 1], off);
  return v & ((1u << FB) - 1u);
}

template <int BK, int BV>
__global__ void __launch_bounds__(kThreads, 1)
attend_kernel(const __grid_constant__ AttendArgs a,
              const __grid_constant__ Codebook cbk,
              const __grid_constant__ Codebook cbv,
              const __grid_constant__ SignMask sm) {
  using Gm = Geo<BK, BV>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* lutK = smem;
  uint8_t* lutV = smem + Gm::LUTK;
  __half* qhi = reinterpret_cast<__half*>(smem + Gm::LUTK + Gm::LUTV);
  __half* qlo = qhi + kMaxGroup * kHeadDim;
  float* fin = reinterpret_cast<float*>(qhi);             // reuses q~ after a segment
  int* misc = reinterpret_cast<int*>(smem + Gm::LUTK + Gm::LUTV + Gm::QS);
  float* miscf = reinterpret_cast<float*>(misc);
  uint8_t* ring = smem + Gm::FIXED;
  float* merge = reinterpret_cast<float*>(ring);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int H = a.n_kv_heads, GQ = a.gqa, B = a.batch;
  const int Gc = gridDim.x, cta = blockIdx.x;   // Gc <= kMaxCtas (host check)
  const uint32_t lutK_base = 0, lutV_base = Gm::LUTK;    // byte offsets in smem

  // ---- codebook tables: fp16 high/low parts of the scaled K levels and
  // fp16 V levels are staged in misc first (uniform lookups afterwards).
  uint32_t* cbs = reinterpret_cast<uint32_t*>(misc) + 64;   // 16 K (hi|lo<<16), 16 V
  if (tid < 16) {
    const float c = cbk.centroid[tid] * kKScale;
    const __half h = __float2half_rn(c), l = __float2half_rn(c - __half2float(h));
    cbs[tid] = (uint32_t)__half_as_ushort(h) | ((uint32_t)__half_as_ushort(l) << 16);
    cbs[16 + tid] = __half_as_ushort(__float2half_rn(cbv.centroid[tid]));
  }
  __syncthreads();
  for (int e = tid; e < (1 << (2 * BK)) * 32; e += kThreads) {
    const int entry = e >> 5, copy = e & 31;
    const uint32_t c0 = cbs[entry & ((1 << BK) - 1)], c1 = cbs[entry >> BK];
    uint2 v;
    v.x = (c0 & 0xFFFFu) | (c1 << 16);
    v.y = (c0 >> 16) | (c1 & 0xFFFF0000u);
    *reinterpret_cast<uint2*>(lutK + entry * 256 + copy * 8) = v;
  }
  if (BV != 2) {
    for (int e = tid; e < (1 << (2 * BV)) * 32; e += kThreads) {
      const int entry = e >> 5, copy = e & 31;
      *reinterpret_cast<uint32_t*>(lutV + entry * 128 + copy * 4) =
          cbs[16 + (entry & ((1 << BV) - 1))] | (cbs[16 + (entry >> BV)] << 16);
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

  // ---- flat block count
  if (warp == 0) {
    long long tot = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      int nb = (b0 + lane < B) ? seq_blocks(a, b0 + lane) : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) nb += __shfl_xor_sync(0xFFFFFFFFu, nb, o);
      tot += nb;
    }
    if (lane == 0) {
      const long long nbt = tot * H;
      misc[kMiscNB] = (int)(nbt & 0xFFFFFFFF);
      misc[kMiscNB + 1] = (int)(nbt >> 32);
      misc[kMiscState] = 0;       // sb
      misc[kMiscState + 1] = 0;   // sP low word
      misc[kMiscState + 2] = 0;   // sP high word
    }
  }
  __syncthreads();
  const long long NB = (long long)(unsigned)misc[kMiscNB] | ((long long)misc[kMiscNB + 1] << 32);
  // Balance over Geff = min(grid, NB) CTAs so every participating CTA owns at
  // least one block; the partial count of a sequence relies on it.
  const int Geff = (int)min((long long)Gc, NB);
  const long long r0 = cta < Geff ? NB * cta / Geff : 0;
  const long long r1 = cta < Geff ? NB * (cta + 1) / Geff : 0;
  long long pos = r0;
  unsigned nskip = 0;
  const float log2tau = a.tau > 0.f ? log2f(a.tau) : -INFINITY;

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
        const int nb = b < B ? seq_blocks(a, b) : 0;
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
          const int excl = __shfl_sync(0xFFFFFFFFu, incl - nb, l);
          sb += l;
          sP += excl;
          if (lane == 0) {
            const long long start = (long long)H * sP;
            const long long rel = pos - start;
            const int g = (int)(rel / nbl), blk0 = (int)(rel % nbl);
            const int nseg = (int)min((long long)(nbl - blk0), r1 - pos);
            misc[kMiscSeg + 0] = sb;
            misc[kMiscSeg + 1] = g;
            misc[kMiscSeg + 2] = blk0;
            misc[kMiscSeg + 3] = nseg;
            misc[kMiscSeg + 4] = nbl;
            misc[kMiscSeg + 5] = min(max(a.ctx_lens[sb], 0), a.cap_tok);
            misc[kMiscState] = sb;
            misc[kMiscState + 1] = (int)(sP & 0xFFFFFFFF);
            misc[kMiscState + 2] = (int)(sP >> 32);
          }
          break;
        }
        const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
        sP += total;
        sb += 32;
      }
    }
    __syncthreads();
    const int b = misc[kMiscSeg + 0], g = misc[kMiscSeg + 1], blk0 = misc[kMiscSeg + 2];
    const int nseg = misc[kMiscSeg + 3], nbl = misc[kMiscSeg + 4], L = misc[kMiscSeg + 5];
    if (nseg <= 0) break;
    const long long sP_seg = (long long)(unsigned)misc[kMiscState + 1] | ((long long)misc[kMiscState + 2] << 32);
    const long long seg_first = (long long)H * sP_seg + (long long)g * nbl;

    // ---- rotated query of the group: warp h handles query head h
    if (warp < GQ) {
      const size_t qb = ((size_t)b * a.n_q_heads + (size_t)g * GQ + warp) * kHeadDim + 4 * lane;
      float x[4];
      const uint32_t m = sm.w[lane >> 3];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        x[k] = apply_sign(load_elem(a.q, a.q_dtype, qb + k), m, (4 * lane + k) & 31);
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

    // ---- this warp's blocks of the segment
    const int wb0 = blk0 + (int)((long long)nseg * warp / kWarps);
    const int wb1 = blk0 + (int)((long long)nseg * (warp + 1) / kWarps);
    const int nw = wb1 - wb0;
    const bool hv = gq < GQ;                       // this lane's score row is a real head
    uint32_t qa[8][4];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int c0 = 32 * tq + 4 * s;
      if (hv) {
        qa[s][0] = *reinterpret_cast<const uint32_t*>(qhi + gq * kHeadDim + c0);
        qa[s][1] = *reinterpret_cast<const uint32_t*>(qlo + gq * kHeadDim + c0);
        qa[s][2] = *reinterpret_cast<const uint32_t*>(qhi + gq * kHeadDim + c0 + 2);
        qa[s][3] = *reinterpret_cast<const uint32_t*>(qlo + gq * kHeadDim + c0 + 2);
      } else {
        qa[s][0] = qa[s][1] = qa[s][2] = qa[s][3] = 0u;
      }
    }
    const float sinv = hv ? miscf[kMiscQInv + gq] : 0.f;

    float acc[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    const size_t seq_row = ((size_t)b * H + g) * a.cap_tok;
    const uint8_t* gk = a.packed_k + seq_row * Gm::RK;
    const uint8_t* gv = a.packed_v + seq_row * Gm::RV;
    const uint16_t* gnk = a.norms_k + seq_row;
    const uint16_t* gnv = a.norms_v + seq_row;
    const uint32_t wring = Gm::FIXED + warp * Gm::NSTAGE * Gm::STAGE;   // smem offset
    const uint32_t wring_s = smem_addr(smem) + wring;                    // shared address

    auto issue = [&](int blk, int slot) {
      const int t0 = blk * kBlk;
      const int nvalid = min(kBlk, L - t0);
      const uint32_t dst = wring_s + slot * Gm::STAGE;
      for (int ch = lane; ch < kBlk * BK; ch += 32) {
        const int row = ch / BK, col = ch % BK;
        const bool ok = row < nvalid;
        const uint8_t* src = gk + (size_t)(t0 + (ok ? row : 0)) * Gm::RK + col * 16;
        cp_async16(dst + row * Gm::RK + col * 16, src, ok ? 16 : 0);
      }
      for (int ch = lane; ch < kBlk * BV; ch += 32) {
        const int row = ch / BV, col = ch % BV;
        const bool ok = row < nvalid;
        const uint8_t* src = gv + (size_t)(t0 + (ok ? row : 0)) * Gm::RV + col * 16;
        cp_async16(dst + Gm::KB + row * Gm::RVS + col * 16, src, ok ? 16 : 0);
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
    for (int i = 0; i < nw; ++i) {
      {
        const int nxt = i + Gm::NSTAGE - 1;
        if (nxt < nw) issue(wb0 + nxt, nxt % Gm::NSTAGE);
        cp_async_commit();
      }
      cp_async_wait<Gm::NSTAGE - 1>();
      __syncwarp();
      const uint32_t st = wring + (i % Gm::NSTAGE) * Gm::STAGE;          // smem offset
      const int t0 = (wb0 + i) * kBlk;

      // -- scores for 8 tiles of 8 positions; high and low codebook parts
      //    accumulate in separate chains
      float sc[8][2];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t kw[BK + 1];
        const uint32_t krow = st + (8 * j + gq) * Gm::RK + 4 * BK * tq;
#pragma unroll
        for (int w = 0; w < BK; ++w) kw[w] = lds32(smem, krow + 4 * w);
        kw[BK] = 0;
        float dh[4] = {0.f, 0.f, 0.f, 0.f}, dl[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t lo = lutK_base + lane * 8;
        uint2 e[16];
#pragma unroll
        for (int p = 0; p < 16; ++p) e[p] = lds64(smem, lut_off<8>(pair_field<BK>(kw, p), lo));
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2) {
          mma16816(dh, qa[s2][0], qa[s2][1], qa[s2][2], qa[s2][3], e[2 * s2].x, e[2 * s2 + 1].x);
          mma16816(dl, qa[s2][0], qa[s2][1], qa[s2][2], qa[s2][3], e[2 * s2].y, e[2 * s2 + 1].y);
        }
        const uint32_t n2 = lds32(smem, st + Gm::NKOFF + (8 * j + 2 * tq) * 2);
        const float n0 = __half2float(__ushort_as_half((uint16_t)(n2 & 0xFFFF)));
        const float n1 = __half2float(__ushort_as_half((uint16_t)(n2 >> 16)));
        const int tok = t0 + 8 * j + 2 * tq;
        sc[j][0] = tok < L ? ((dh[0] + dl[0]) + (dh[2] + dl[2])) * sinv * n0 : -INFINITY;
        sc[j][1] = tok + 1 < L ? ((dh[1] + dl[1]) + (dh[3] + dl[3])) * sinv * n1 : -INFINITY;
      }

      // -- softmax statistics of the block (head = gq)
      float mb = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) mb = fmaxf(mb, fmaxf(sc[j][0], sc[j][1]));
      mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 1));
      mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 2));
      const float m_new = fmaxf(m_run, mb);
      const float alpha = exp2f(m_run - m_new);
      l_run *= alpha;
      m_run = m_new;
      uint32_t pb[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t n2 = lds32(smem, st + Gm::NKOFF + 2 * kBlk + (8 * j + 2 * tq) * 2);
        float p[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float w = exp2f(sc[j][e] - m_new);
          l_run += w;
          const float nv = __half2float(__ushort_as_half((uint16_t)(e ? n2 >> 16 : n2 & 0xFFFF)));
          float pv = w * nv;
          if (sc[j][e] - mb < log2tau) {       // exp(s - M_blk) < tau, log2 domain
            if (hv && sc[j][e] != -INFINITY) ++nskip;
            pv = 0.f;
          }
          p[e] = hv ? pv : 0.f;
        }
        pb[j] = pack_half2(p[0], p[1]);
      }
      // rescale the accumulators of heads 2tq, 2tq+1
      const float a0 = __shfl_sync(0xFFFFFFFFu, alpha, 8 * tq);
      const float a1 = __shfl_sync(0xFFFFFFFFu, alpha, 8 * tq + 4);
      if (__any_sync(0xFFFFFFFFu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          acc[r][0] *= a0;
          acc[r][1] *= a1;
          acc[r][2] *= a0;
          acc[r][3] *= a1;
        }
      }

      // -- P·V over four 16-position k-steps
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t b0 = pb[2 * kk], b1 = pb[2 * kk + 1];
        if (!__any_sync(0xFFFFFFFFu, (b0 | b1) != 0u)) continue;   // whole step gated
        if (BV == 2) {
          const uint32_t vrow = st + Gm::KB + (16 * kk + 2 * tq) * Gm::RVS + 4 * gq;
          const uint32_t wA = lds32(smem, vrow), wB = lds32(smem, vrow + Gm::RVS);
          const uint32_t wC = lds32(smem, vrow + 8 * Gm::RVS), wD = lds32(smem, vrow + 9 * Gm::RVS);
          const uint32_t xab[2] = {__byte_perm(wA, wB, 0x5140), __byte_perm(wA, wB, 0x7362)};
          const uint32_t xcd[2] = {__byte_perm(wC, wD, 0x5140), __byte_perm(wC, wD, 0x7362)};
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            // original bytes 2·half (low 16 bits) and 2·half+1 (high 16 bits)
#pragma unroll
            for (int odd = 0; odd < 2; ++odd) {
              const int f0 = 4 * odd, f1 = 4 * odd + 2;   // fields of coords 2r, 2r+1
              const uint32_t s0 = ((xab[half] >> f0) & 0x03030303u) * 0x11u + 0x40404040u;
              const uint32_t s1 = ((xab[half] >> f1) & 0x03030303u) * 0x11u + 0x40404040u;
              const uint32_t s2 = ((xcd[half] >> f0) & 0x03030303u) * 0x11u + 0x40404040u;
              const uint32_t s3 = ((xcd[half] >> f1) & 0x03030303u) * 0x11u + 0x40404040u;
#pragma unroll
              for (int hb = 0; hb < 2; ++hb) {
                const int r = 2 * (2 * half + hb) + odd;
                const int sh = 16 * hb;
                const uint32_t va0 = __byte_perm(vt_lo, vt_hi, s0 >> sh);
                const uint32_t va1 = __byte_perm(vt_lo, vt_hi, s1 >> sh);
                const uint32_t va2 = __byte_perm(vt_lo, vt_hi, s2 >> sh);
                const uint32_t va3 = __byte_perm(vt_lo, vt_hi, s3 >> sh);
                mma16816(acc[r], va0, va1, va2, va3, b0, b1);
              }
            }
          }
        } else {
          uint32_t v0[BV + 1], v1[BV + 1];
          const uint32_t r0p = st + Gm::KB + (16 * kk + gq) * Gm::RVS + 4 * BV * tq;
          const uint32_t r1p = r0p + 8 * Gm::RVS;
#pragma unroll
          for (int w = 0; w < BV; ++w) {
            v0[w] = lds32(smem, r0p + 4 * w);
            v1[w] = lds32(smem, r1p + 4 * w);
          }
          v0[BV] = v1[BV] = 0;
          const uint32_t lo = lutV_base + lane * 4;
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const uint32_t x0 = lds32(smem, lut_off<7>(pair_field<BV>(v0, 2 * r), lo));
            const uint32_t x1 = lds32(smem, lut_off<7>(pair_field<BV>(v0, 2 * r + 1), lo));
            const uint32_t x2 = lds32(smem, lut_off<7>(pair_field<BV>(v1, 2 * r), lo));
            const uint32_t x3 = lds32(smem, lut_off<7>(pair_field<BV>(v1, 2 * r + 1), lo));
            mma16816(acc[r], transpose8x8(x0), transpose8x8(x1), transpose8x8(x2),
                     transpose8x8(x3), b0, b1);
          }
        }
      }
      __syncwarp();
    }
    cp_async_wait<0>();

    // ---- merge the warps of this segment
    l_run += __shfl_xor_sync(0xFFFFFFFFu, l_run, 1);
    l_run += __shfl_xor_sync(0xFFFFFFFFu, l_run, 2);
    __syncthreads();                                  // all warps done with the ring
    {
      float* wm = merge + warp * (kMaxGroup * kHeadDim + 2 * kMaxGroup);
      if (tq == 0 && hv) {
        wm[kMaxGroup * kHeadDim + gq] = nw > 0 ? m_run : -INFINITY;
        wm[kMaxGroup * kHeadDim + kMaxGroup + gq] = nw > 0 ? l_run : 0.f;
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
    constexpr int WS = kMaxGroup * kHeadDim + 2 * kMaxGroup;
    if (tid < GQ) {
      float mx = -INFINITY;
      for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, merge[w * WS + kMaxGroup * kHeadDim + tid]);
      float ls = 0.f;
      for (int w = 0; w < kWarps; ++w)
        ls += merge[w * WS + kMaxGroup * kHeadDim + kMaxGroup + tid] *
              exp2f(merge[w * WS + kMaxGroup * kHeadDim + tid] - mx);
      miscf[kMiscM + tid] = mx;
      miscf[kMiscL + tid] = ls;
    }
    __syncthreads();
    for (int i = tid; i < GQ * kHeadDim; i += kThreads) {
      const int h = i / kHeadDim;
      const float mx = miscf[kMiscM + h];
      float s = 0.f;
      for (int w = 0; w < kWarps; ++w) {
        const float mw = merge[w * WS + kMaxGroup * kHeadDim + h];
        if (mw != -INFINITY) s += merge[w * WS + i] * exp2f(mw - mx);
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
        __threadfence();
        const float* s0 = a.slots + (size_t)(c_first + sigma) * GQ * kSlotFloats;
        const size_t stride = (size_t)GQ * kSlotFloats;
        if (tid < GQ) {
          float mx = -INFINITY;
          for (int p = 0; p < n_parts; ++p) mx = fmaxf(mx, __ldcg(s0 + p * stride + GQ * kHeadDim + 2 * tid));
          float ls = 0.f;
          for (int p = 0; p < n_parts; ++p)
            ls += __ldcg(s0 + p * stride + GQ * kHeadDim + 2 * tid + 1) *
                  exp2f(__ldcg(s0 + p * stride + GQ * kHeadDim + 2 * tid) - mx);
          miscf[kMiscM + tid] = mx;
          miscf[kMiscL + tid] = ls;
        }
        __syncthreads();
        for (int i = tid; i < GQ * kHeadDim; i += kThreads) {
          const int h = i / kHeadDim;
          const float mx = miscf[kMiscM + h];
          float s = 0.f;
          for (int p = 0; p < n_parts; ++p)
            s += __ldcg(s0 + p * stride + i) * exp2f(__ldcg(s0 + p * stride + GQ * kHeadDim + 2 * h) - mx);
          fin[i] = s;
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

template <int BK, int BV>
cudaError_t launch_pair(const AttendArgs& a, const Codebook& cbk, const Codebook& cbv,
                        const SignMask& sm, int n_ctas, cudaStream_t stream) {
  using Gm = Geo<BK, BV>;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(attend_kernel<BK, BV>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, Gm::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  const int grid = n_ctas > 0 ? n_ctas : sm_count();
  attend_kernel<BK, BV><<<grid, kThreads, Gm::SMEM, stream>>>(a, cbk, cbv, sm);
  return cudaGetLastError();
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
